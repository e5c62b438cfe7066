// Router: logits z = W_r^T x, selection key, top-k, gates and the per-chunk
// partial statistics.
//
// "Week 2 Day 2: Mixture of Experts" §1.3 (z = W_r^T x, T = TopK(z, k),
// g_i = exp(z_i) / sum_{j in T} exp(z_j)), §4.2 (selection on z + b, gates from
// the raw z), §3.2 (f_i and P_i of the balance loss); "Stanford CS336 Lecture
// 04" §2.3.3c (bias added to the softmax score). Router arithmetic is fp32
// ("Lecture 21 · LLM: Mixture-of-Experts" §7.1: the router runs in fp32).
#include <algorithm>
#include <cstdlib>

#include "common.cuh"
#include "tc_common.cuh"
#include "warp_mma.cuh"

namespace moe {


// ---- W_r [d, E] -> W_r^T [E, d] ------------------------------------------
template <typename T>
__global__ void transpose_kernel(const T* __restrict__ in, T* __restrict__ out, int d, int E,
                                 int32_t* __restrict__ status) {
    __shared__ T tile[32][33];
    pdl_wait();
    pdl_launch();
    if (status != nullptr && blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0 && threadIdx.y == 0)
        *status = MOE_OK;
    int i0 = blockIdx.x * 32, e0 = blockIdx.y * 32;
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        int i = i0 + r, e = e0 + threadIdx.x;
        if (i < d && e < E) tile[r][threadIdx.x] = in[(size_t)i * E + e];
    }
    __syncthreads();
    for (int r = threadIdx.y; r < 32; r += blockDim.y) {
        int e = e0 + r, i = i0 + threadIdx.x;
        if (i < d && e < E) out[(size_t)e * d + i] = tile[threadIdx.x][r];
    }
}

cudaError_t launch_transpose_wr(int dtype, const void* W_r, void* wrt, int d, int E, cudaStream_t st,
                                int32_t* status) {
    dim3 grid(ceil_div(d, 32), ceil_div(E, 32)), block(32, 8);
    if (dtype == MOE_DTYPE_BF16)
        return launch_k(transpose_kernel<__nv_bfloat16>, grid, block, 0, st, (const __nv_bfloat16*)W_r,
                        (__nv_bfloat16*)wrt, d, E, status);
    return launch_k(transpose_kernel<float>, grid, block, 0, st, (const float*)W_r, (float*)wrt, d, E, status);
}

// ---- logits on CUDA cores -------------------------------------------------
// One block per group of kLgTok tokens; its kLgWarps warps split the row into
// contiguous slices of 8-element chunks (lane l takes chunks l, l + 32, ... of
// its warp's slice). Per chunk a lane loads the tokens' x once and the chunk
// of each of 8 experts' W_r^T rows, accumulating acc[token][expert] in
// ascending chunk order. Lane partials are summed by an xor butterfly, warp
// partials in warp order through shared memory: the summation order is fixed,
// so the same inputs always give the same bits. Experts are taken 8 at a time.
constexpr int kLgTok = 4;
constexpr int kLgWarps = 8;
constexpr int kExpPerPass = 8;

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    float4 a = *reinterpret_cast<const float4*>(p);
    float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x; v[2 * i + 1] = f.y;
    }
}

template <typename T>
__global__ void __launch_bounds__(kLgWarps * 32)
logits_kernel(const T* __restrict__ x, const T* __restrict__ wrt, float* __restrict__ logits, int Tn, int d,
              int E) {
    __shared__ float part[kLgWarps][kLgTok][kExpPerPass];
    pdl_wait();
    pdl_launch();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t0 = blockIdx.x * kLgTok;
    const int nt = min(kLgTok, Tn - t0);
    const int nchunk = d / 8;
    const int per = (nchunk + kLgWarps - 1) / kLgWarps;
    const int c_lo = warp * per, c_hi = min(nchunk, c_lo + per);
    for (int e0 = 0; e0 < E; e0 += kExpPerPass) {
        float acc[kLgTok][kExpPerPass];
#pragma unroll
        for (int q = 0; q < kLgTok; ++q)
#pragma unroll
            for (int e = 0; e < kExpPerPass; ++e) acc[q][e] = 0.f;
        for (int c = c_lo + lane; c < c_hi; c += 32) {
            float xv[kLgTok][8];
#pragma unroll
            for (int q = 0; q < kLgTok; ++q) {
                if (q < nt) {
                    load8(x + (size_t)(t0 + q) * d + (size_t)c * 8, xv[q]);
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) xv[q][j] = 0.f;
                }
            }
#pragma unroll
            for (int e = 0; e < kExpPerPass; ++e) {
                if (e0 + e < E) {
                    float wv[8];
                    load8(wrt + (size_t)(e0 + e) * d + (size_t)c * 8, wv);
#pragma unroll
                    for (int q = 0; q < kLgTok; ++q)
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[q][e] = fmaf(xv[q][j], wv[j], acc[q][e]);
                }
            }
        }
#pragma unroll
        for (int q = 0; q < kLgTok; ++q) {
#pragma unroll
            for (int e = 0; e < kExpPerPass; ++e) {
                float v = acc[q][e];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) part[warp][q][e] = v;
            }
        }
        __syncthreads();
        if (threadIdx.x < kLgTok * kExpPerPass) {
            const int q = threadIdx.x / kExpPerPass, e = threadIdx.x % kExpPerPass;
            if (q < nt && e0 + e < E) {
                float v = 0.f;
                for (int w = 0; w < kLgWarps; ++w) v += part[w][q][e];
                logits[(size_t)(t0 + q) * E + e0 + e] = v;
            }
        }
        __syncthreads();
    }
}

cudaError_t launch_logits_simt(int dtype, const void* x, const void* wrt, float* logits,
                               int T, int d, int E, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int grid = ceil_div(T, kLgTok);
    if (dtype == MOE_DTYPE_BF16)
        return launch_k(logits_kernel<__nv_bfloat16>, dim3(grid), dim3(kLgWarps * 32), 0, st,
                        (const __nv_bfloat16*)x, (const __nv_bfloat16*)wrt, logits, T, d, E);
    return launch_k(logits_kernel<float>, dim3(grid), dim3(kLgWarps * 32), 0, st, (const float*)x,
                    (const float*)wrt, logits, T, d, E);
}

// ---- selection: softmax, key, top-k, gates, chunk statistics -------------
// Grid: one block per chunk of kChunk tokens; 8 warps, 4 tokens per warp.
// Lane l holds experts e = l + 32 i, i < EPL. Every warp reduction is an xor
// butterfly, so all lanes end with the same bits and the order is fixed.
constexpr int kSelWarps = 8;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Per token it also accumulates the router statistics of the warp's tokens:
// (log sum_e exp z)^2 for the z-loss, the entropy log-sum-exp - sum_e p z, and
// the gap between the two largest probabilities, p_(1) - p_(2) =
// (1 - exp(z_(2) - z_(1))) / sum_e exp(z_e - z_(1)).
template <int EPL>
struct SelAcc {
    float b[EPL];      // selection bias of the lane's experts
    float psum[EPL];   // sum of the warp's tokens' probabilities of the lane's experts
    float ex_z, ex_h, ex_g;
};

template <int EPL>
__device__ __forceinline__ void sel_init(SelAcc<EPL>& a, const float* __restrict__ bias, int bias_mode, int E,
                                         int lane) {
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        a.b[i] = (bias_mode != MOE_BIAS_NONE && e < E) ? bias[e] : 0.f;
        a.psum[i] = 0.f;
    }
    a.ex_z = a.ex_h = a.ex_g = 0.f;
}

// One token t whose logits the warp holds (lane l: experts l + 32 i in
// zin[i]): softmax, statistics, key, top-k, gates, and the chunk's counts.
template <int EPL, bool COMPACT = false>
__device__ __forceinline__ void sel_token(const float (&zin)[EPL], int t, int bias_mode, int gate_mode, int kk,
                                          int E, int k, int lane, SelAcc<EPL>& a, int* cnt,
                                          int32_t* __restrict__ idx_out, float* __restrict__ gate_out) {
    float z[EPL], key[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        int e = lane + 32 * i;
        z[i] = e < E ? zin[i] : -INFINITY;
    }
    // full softmax over all E raw logits (for P and the PROB key)
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) m = fmaxf(m, z[i]);
    m = warp_max(m);
    float ex[EPL], s = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        int e = lane + 32 * i;
        ex[i] = e < E ? expf(z[i] - m) : 0.f;
        s += ex[i];
    }
    s = warp_sum(s);
    const float inv_s = 1.f / s;
    // router statistics of this token
    {
        float pz = 0.f, z1 = -INFINITY, z2 = -INFINITY;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            if (lane + 32 * i < E) {
                pz += ex[i] * z[i];
                if (z[i] > z1) { z2 = z1; z1 = z[i]; } else if (z[i] > z2) { z2 = z[i]; }
            }
        }
        pz = warp_sum(pz) * inv_s;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float o1 = __shfl_xor_sync(0xffffffffu, z1, o);
            const float o2 = __shfl_xor_sync(0xffffffffu, z2, o);
            const float hi = fmaxf(z1, o1);
            z2 = fmaxf(fminf(z1, o1), fmaxf(z2, o2));
            z1 = hi;
        }
        const float lse = m + logf(s);
        a.ex_z += lse * lse;
        a.ex_h += lse - pz;
        a.ex_g += (1.f - expf(z2 - m)) * inv_s;
    }
    unsigned valid = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        int e = lane + 32 * i;
        float p = ex[i] * inv_s;
        if (e < E) {
            a.psum[i] += p;
            valid |= 1u << i;
        }
        key[i] = bias_mode == MOE_BIAS_NONE ? z[i]
               : bias_mode == MOE_BIAS_LOGIT ? z[i] + a.b[i]
               : p + a.b[i];
    }
    // top-k: k rounds of a warp arg-max over (key desc, index asc); the
    // compact form keeps the rounds a loop (small code for kernels that run
    // the selection beside other work), the other unrolls them
    unsigned taken = 0;
    float zsel[MOE_MAX_K];
    int esel[MOE_MAX_K];
    auto round = [&](int j) {
        float bk = -INFINITY, bz = 0.f;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            bool ok = ((valid >> i) & 1u) && !((taken >> i) & 1u);
            if (ok && (key[i] > bk || be == 0x7fffffff)) {
                bk = key[i]; be = lane + 32 * i; bz = z[i];
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            float ok_ = __shfl_xor_sync(0xffffffffu, bk, o);
            int oe = __shfl_xor_sync(0xffffffffu, be, o);
            float oz = __shfl_xor_sync(0xffffffffu, bz, o);
            bool better = (oe != 0x7fffffff) &&
                          (be == 0x7fffffff || ok_ > bk || (ok_ == bk && oe < be));
            if (better) { bk = ok_; be = oe; bz = oz; }
        }
        if ((be & 31) == lane) taken |= 1u << (be >> 5);
        zsel[j] = bz;
        esel[j] = be;
    };
    float zm = -INFINITY, gs = 0.f, ge[MOE_MAX_K];
    if constexpr (COMPACT) {
#pragma unroll 1
        for (int j = 0; j < k; ++j) round(j);
        // gates: softmax over the selected raw logits, slot order
#pragma unroll 1
        for (int j = 0; j < k; ++j) zm = fmaxf(zm, zsel[j]);
#pragma unroll 1
        for (int j = 0; j < k; ++j) { ge[j] = expf(zsel[j] - zm); gs += ge[j]; }
    } else {
#pragma unroll
        for (int j = 0; j < MOE_MAX_K; ++j)
            if (j < k) round(j);
        // gates: softmax over the selected raw logits, slot order
#pragma unroll
        for (int j = 0; j < MOE_MAX_K; ++j) if (j < k) zm = fmaxf(zm, zsel[j]);
#pragma unroll
        for (int j = 0; j < MOE_MAX_K; ++j) {
            if (j < k) { ge[j] = expf(zsel[j] - zm); gs += ge[j]; }
        }
    }
    const float inv_g = 1.f / gs;
    if (lane == 0) {
        auto emit = [&](int j) {
            idx_out[(size_t)t * k + j] = esel[j];
            // selected softmax, or the full-softmax probability (Switch gate)
            gate_out[(size_t)t * k + j] = gate_mode == MOE_GATE_FULL ? expf(zsel[j] - m) * inv_s : ge[j] * inv_g;
            atomicAdd(&cnt[esel[j] * kk + (kk > 1 ? j : 0)], 1);   // integer: order does not matter
        };
        if constexpr (COMPACT) {
#pragma unroll 1
            for (int j = 0; j < k; ++j) emit(j);
        } else {
#pragma unroll
            for (int j = 0; j < MOE_MAX_K; ++j)
                if (j < k) emit(j);
        }
    }
}

// Q tokens at once (lane l holds the logits of experts l + 32 i of each):
// per token the same arithmetic as sel_token (compact form) in the same
// order, with the Q tokens' steps interleaved so that their shuffle chains
// overlap instead of running one token after another. Only tokens q < nt
// are counted and emitted (the others run on zeros); the statistics take
// the tokens in order, so the bits are those of sel_token called token by
// token.
template <int EPL, int Q>
__device__ __forceinline__ void sel_tokens(const float (&zin)[Q][EPL], int nt, int t0, int bias_mode, int gate_mode,
                                           int kk, int E, int k, int lane, SelAcc<EPL>& a, int* cnt,
                                           int32_t* __restrict__ idx_out, float* __restrict__ gate_out) {
    float z[Q][EPL], ex[Q][EPL], key[Q][EPL], m[Q], s[Q], inv_s[Q];
#pragma unroll
    for (int q = 0; q < Q; ++q)
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            z[q][i] = e < E ? (q < nt ? zin[q][i] : 0.f) : -INFINITY;
        }
    // full softmax over all E raw logits
#pragma unroll
    for (int q = 0; q < Q; ++q) {
        m[q] = -INFINITY;
#pragma unroll
        for (int i = 0; i < EPL; ++i) m[q] = fmaxf(m[q], z[q][i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int q = 0; q < Q; ++q) m[q] = fmaxf(m[q], __shfl_xor_sync(0xffffffffu, m[q], o));
#pragma unroll
    for (int q = 0; q < Q; ++q) {
        s[q] = 0.f;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            ex[q][i] = e < E ? expf(z[q][i] - m[q]) : 0.f;
            s[q] += ex[q][i];
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int q = 0; q < Q; ++q) s[q] += __shfl_xor_sync(0xffffffffu, s[q], o);
#pragma unroll
    for (int q = 0; q < Q; ++q) inv_s[q] = 1.f / s[q];
    // router statistics
    {
        float pz[Q], z1[Q], z2[Q];
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            pz[q] = 0.f; z1[q] = -INFINITY; z2[q] = -INFINITY;
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                if (lane + 32 * i < E) {
                    pz[q] += ex[q][i] * z[q][i];
                    if (z[q][i] > z1[q]) { z2[q] = z1[q]; z1[q] = z[q][i]; } else if (z[q][i] > z2[q]) { z2[q] = z[q][i]; }
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int q = 0; q < Q; ++q) pz[q] += __shfl_xor_sync(0xffffffffu, pz[q], o);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int q = 0; q < Q; ++q) {
                const float o1 = __shfl_xor_sync(0xffffffffu, z1[q], o);
                const float o2 = __shfl_xor_sync(0xffffffffu, z2[q], o);
                const float hi = fmaxf(z1[q], o1);
                z2[q] = fmaxf(fminf(z1[q], o1), fmaxf(z2[q], o2));
                z1[q] = hi;
            }
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            if (q < nt) {
                const float pzq = pz[q] * inv_s[q];
                const float lse = m[q] + logf(s[q]);
                a.ex_z += lse * lse;
                a.ex_h += lse - pzq;
                a.ex_g += (1.f - expf(z2[q] - m[q])) * inv_s[q];
            }
        }
    }
    unsigned valid = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i)
        if (lane + 32 * i < E) valid |= 1u << i;
#pragma unroll
    for (int q = 0; q < Q; ++q)
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const float p = ex[q][i] * inv_s[q];
            if (q < nt && ((valid >> i) & 1u)) a.psum[i] += p;
            key[q][i] = bias_mode == MOE_BIAS_NONE ? z[q][i]
                      : bias_mode == MOE_BIAS_LOGIT ? z[q][i] + a.b[i]
                      : p + a.b[i];
        }
    // top-k: k rounds of a warp arg-max over (key desc, index asc), on one
    // 64-bit value per candidate: the key mapped to an unsigned integer of
    // the same order (-0 taken as +0, as a float compare does) above the
    // complemented index, so the larger value is the larger key and, among
    // equal keys, the lower index; 0 stands for no candidate. Lane j keeps
    // the winner of round j (its raw logit and index) in registers.
    unsigned taken[Q];
    float zmine[Q];
    int emine[Q];
#pragma unroll
    for (int q = 0; q < Q; ++q) { taken[q] = 0; zmine[q] = 0.f; emine[q] = 0; }
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
        unsigned long long best[Q];
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            best[q] = 0ull;
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                if (((valid >> i) & 1u) && !((taken[q] >> i) & 1u)) {
                    const uint32_t b = __float_as_uint(key[q][i] + 0.f);
                    const uint32_t o = (b & 0x80000000u) ? ~b : (b | 0x80000000u);
                    const unsigned long long c = ((unsigned long long)o << 32) | (uint32_t)(~(lane + 32 * i));
                    best[q] = c > best[q] ? c : best[q];
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int q = 0; q < Q; ++q) {
                const unsigned long long c = __shfl_xor_sync(0xffffffffu, best[q], o);
                best[q] = c > best[q] ? c : best[q];
            }
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            const int be = (int)(~(uint32_t)best[q]);
            float zc = z[q][0];
#pragma unroll
            for (int i = 1; i < EPL; ++i)
                if ((be >> 5) == i) zc = z[q][i];
            const float bz = __shfl_sync(0xffffffffu, zc, be & 31);   // the raw logit, from its lane
            if ((be & 31) == lane) taken[q] |= 1u << (be >> 5);
            if (lane == j) { zmine[q] = bz; emine[q] = be; }
        }
    }
    // gates: softmax over the selected raw logits, slot order (every lane
    // reads slot j from lane j, in order); lane j < k emits slot j
    float zm[Q], gs[Q];
#pragma unroll
    for (int q = 0; q < Q; ++q) { zm[q] = -INFINITY; gs[q] = 0.f; }
#pragma unroll 1
    for (int j = 0; j < k; ++j)
#pragma unroll
        for (int q = 0; q < Q; ++q) zm[q] = fmaxf(zm[q], __shfl_sync(0xffffffffu, zmine[q], j));
#pragma unroll 1
    for (int j = 0; j < k; ++j)
#pragma unroll
        for (int q = 0; q < Q; ++q) gs[q] += expf(__shfl_sync(0xffffffffu, zmine[q], j) - zm[q]);
    if (lane < k) {
#pragma unroll
        for (int q = 0; q < Q; ++q) {
            if (q < nt) {
                const size_t o = (size_t)(t0 + q) * k + lane;
                idx_out[o] = emine[q];
                // selected softmax, or the full-softmax probability (Switch gate)
                gate_out[o] = gate_mode == MOE_GATE_FULL ? expf(zmine[q] - m[q]) * inv_s[q]
                                                         : expf(zmine[q] - zm[q]) * (1.f / gs[q]);
                atomicAdd(&cnt[emine[q] * kk + (kk > 1 ? lane : 0)], 1);   // integer: order does not matter
            }
        }
    }
}

// The chunk's statistics: probability sums over warps in warp order, counts,
// and the z-loss / entropy / gap sums.
template <int EPL>
__device__ __forceinline__ void sel_finish(const SelAcc<EPL>& a, int chunk, int NB, int E, int kk, int warp, int lane,
                                           const int* cnt, float (*ps)[MOE_MAX_E], float (*ext)[3],
                                           int32_t* __restrict__ blockcnt, float* __restrict__ blockpsum,
                                           float* __restrict__ blockextra) {
    if (lane == 0) {
        ext[warp][0] = a.ex_z;
        ext[warp][1] = a.ex_h;
        ext[warp][2] = a.ex_g;
    }
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        int e = lane + 32 * i;
        if (e < E) ps[warp][e] = a.psum[i];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float acc = 0.f;
        for (int w = 0; w < kSelWarps; ++w) acc += ps[w][e];   // fixed order over warps
        blockpsum[(size_t)chunk * E + e] = acc;
    }
    for (int i = threadIdx.x; i < E * kk; i += blockDim.x) blockcnt[(size_t)i * NB + chunk] = cnt[i];
    if (threadIdx.x < 3 && blockextra != nullptr) {
        float acc = 0.f;
        for (int w = 0; w < kSelWarps; ++w) acc += ext[w][threadIdx.x];
        blockextra[(size_t)chunk * 3 + threadIdx.x] = acc;
    }
}

template <int EPL>
__global__ void __launch_bounds__(kSelWarps * 32)
select_kernel(const float* __restrict__ logits, const float* __restrict__ bias, int bias_mode, int gate_mode,
              int kk, int Tn, int E, int k, int32_t* __restrict__ idx_out, float* __restrict__ gate_out,
              int32_t* __restrict__ blockcnt, float* __restrict__ blockpsum, float* __restrict__ blockextra) {
    __shared__ int cnt[kMaxSlotCounts];
    __shared__ float ps[kSelWarps][MOE_MAX_E];
    __shared__ float ext[kSelWarps][3];
    pdl_wait();
    pdl_launch();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int chunk = blockIdx.x, NB = gridDim.x;
    for (int e = threadIdx.x; e < E * kk; e += blockDim.x) cnt[e] = 0;
    SelAcc<EPL> a;
    sel_init(a, bias, bias_mode, E, lane);
    __syncthreads();

    constexpr int kTokPerWarp = kChunk / kSelWarps;
    for (int q = 0; q < kTokPerWarp; ++q) {
        const int t = chunk * kChunk + warp * kTokPerWarp + q;
        if (t >= Tn) break;
        float z[EPL];
        const float* zr = logits + (size_t)t * E;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            int e = lane + 32 * i;
            z[i] = e < E ? zr[e] : -INFINITY;
        }
        sel_token<EPL>(z, t, bias_mode, gate_mode, kk, E, k, lane, a, cnt, idx_out, gate_out);
    }
    sel_finish<EPL>(a, chunk, NB, E, kk, warp, lane, cnt, ps, ext, blockcnt, blockpsum, blockextra);
}

// ---- fused router: logits and selection in one kernel ----------------------
// One block per chunk of kChunk tokens, the same warp-to-token assignment as
// select_kernel (warp w: tokens 4w .. 4w + 3 of the chunk). Experts are taken
// eight per pass: the block first copies W_r^T of the pass's experts into
// shared memory (W_r [d, E] as given: a row holds the E weights of one input
// feature). A warp then computes its four tokens' logits itself: lane l
// takes the 8-element chunks c = l, l + 32, ... of the row (16-byte loads of
// x straight from global memory, several chunks of every token in flight),
// multiplies them with the pass's W_r^T from shared memory in fp32 FMAs, and
// an xor butterfly leaves every lane with the sums, in a fixed order. The
// logits are written out (the workspace keeps them) and, still in registers,
// go through the same per-token selection as select_kernel. E <= 64. This
// is the fp32 router, and the bf16 one where the MMA form below does not
// fit; its speed is set by FMA issue (8 FMAs per element of x per pass).
template <typename T>
struct RawVec8 {   // 8 elements of a row as loaded: one 16-byte vector (bf16) or two (fp32)
    uint4 v[sizeof(T) == 2 ? 1 : 2];
};
template <typename T>
__device__ __forceinline__ void raw_load8(const T* p, RawVec8<T>& r) {
#pragma unroll
    for (int i = 0; i < (sizeof(T) == 2 ? 1 : 2); ++i) r.v[i] = __ldg(reinterpret_cast<const uint4*>(p) + i);
}
__device__ __forceinline__ void unpack8(const RawVec8<__nv_bfloat16>& r, float (&v)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r.v[0]);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x; v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ void unpack8(const RawVec8<float>& r, float (&v)[8]) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        v[4 * i] = __uint_as_float(r.v[i].x); v[4 * i + 1] = __uint_as_float(r.v[i].y);
        v[4 * i + 2] = __uint_as_float(r.v[i].z); v[4 * i + 3] = __uint_as_float(r.v[i].w);
    }
}

// The selection half of both fused routers: the warp's nt tokens t0, t0 + 1,
// ... (lane l holds the logits of experts l + 32 i) are written out and go
// through the per-token selection.
template <int EPL>
__device__ __forceinline__ void fused_select(const float (&zt)[kChunk / kSelWarps][EPL], int nt, int t0,
                                             int bias_mode, int gate_mode, int kk, int E, int k, int lane,
                                             SelAcc<EPL>& a, int* cnt, float* __restrict__ logits,
                                             int32_t* __restrict__ idx_out, float* __restrict__ gate_out) {
#pragma unroll
    for (int q = 0; q < kChunk / kSelWarps; ++q) {
        if (q < nt) {
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int e = lane + 32 * i;
                if (e < E) logits[(size_t)(t0 + q) * E + e] = zt[q][i];
            }
        }
    }
    sel_tokens<EPL, kChunk / kSelWarps>(zt, nt, t0, bias_mode, gate_mode, kk, E, k, lane, a, cnt, idx_out, gate_out);
}

// Shared memory of the fused router: W_r^T of one pass's eight experts over
// the whole row (64 KB for bf16 at d = 4096); wider rows take the
// three-kernel router.
constexpr size_t kFusedWtMaxBytes = 160 * 1024;
template <typename T>
size_t fused_smem_bytes(int d) {
    return (size_t)kExpPerPass * (size_t)d * sizeof(T);
}

template <typename T, int EPL>
__global__ void __launch_bounds__(kSelWarps * 32)
route_fused_kernel(const T* __restrict__ x, const T* __restrict__ W_r, const float* __restrict__ bias,
                   int bias_mode, int gate_mode, int kk, int Tn, int d, int E, int k, float* __restrict__ logits,
                   int32_t* __restrict__ idx_out, float* __restrict__ gate_out, int32_t* __restrict__ blockcnt,
                   float* __restrict__ blockpsum, float* __restrict__ blockextra, int32_t* __restrict__ status) {
    static_assert(EPL <= 2, "fused router: E <= 64");
    constexpr int kTokPerWarp = kChunk / kSelWarps;   // 4
    __shared__ int cnt[kMaxSlotCounts];
    __shared__ float ps[kSelWarps][MOE_MAX_E];
    __shared__ float ext[kSelWarps][3];
    extern __shared__ __align__(128) uint8_t fused_dsm[];
    T* wt = reinterpret_cast<T*>(fused_dsm);                      // [kExpPerPass][d]: W_r^T of the pass
    pdl_wait();
    pdl_launch();
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *status = MOE_OK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int chunk = blockIdx.x, NB = gridDim.x;
    for (int e = threadIdx.x; e < E * kk; e += blockDim.x) cnt[e] = 0;
    SelAcc<EPL> a;
    sel_init(a, bias, bias_mode, E, lane);
    const int c0tok = chunk * kChunk;
    const int ntok = min(kChunk, Tn - c0tok);                     // tokens of the block
    const int q0 = warp * kTokPerWarp;                            // the warp's first token in the block
    const int nt = max(0, min(kTokPerWarp, ntok - q0));
    float zt[kTokPerWarp][EPL];
#pragma unroll
    for (int q = 0; q < kTokPerWarp; ++q)
#pragma unroll
        for (int i = 0; i < EPL; ++i) zt[q][i] = -INFINITY;
    const int nchunk = d / 8;                                     // 8-element chunks of a row
    for (int e0 = 0; e0 < E; e0 += kExpPerPass) {
        __syncthreads();   // the previous pass's W_r^T is consumed
        // W_r^T [e0 .. e0 + 7][0 .. d) (zeros past E): the rows of W_r are one
        // contiguous run of d E elements, requested as 16-byte vectors, eight
        // per thread, before any is written, transposed, into shared memory
        if (e0 + kExpPerPass > E)
            for (int i = threadIdx.x; i < kExpPerPass * d; i += blockDim.x) wt[i] = T(0.f);
        __syncthreads();
        {
            const int ng = d * E / 8;
            for (int g0 = threadIdx.x; g0 < ng; g0 += blockDim.x * 8) {
                RawVec8<T> wr[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int g = g0 + (int)blockDim.x * j;
                    if (g < ng) raw_load8(W_r + (size_t)g * 8, wr[j]);
                }
#pragma unroll 1
                for (int j = 0; j < 8; ++j) {
                    const int g = g0 + (int)blockDim.x * j;
                    if (g >= ng) break;
                    float v[8];
                    unpack8(wr[j], v);
                    if (E % kExpPerPass == 0) {
                        // the group is experts [eb, eb + 8) of one input feature r
                        const int r = (g * 8) / E, eb = g * 8 - r * E;
                        if (eb == e0) {
#pragma unroll
                            for (int i = 0; i < 8; ++i) wt[i * d + r] = T(v[i]);
                        }
                    } else {
#pragma unroll 1
                        for (int i = 0; i < 8; ++i) {
                            const int idx = g * 8 + i, r = idx / E, e = idx - r * E - e0;
                            if (e >= 0 && e < kExpPerPass) wt[e * d + r] = T(v[i]);
                        }
                    }
                }
            }
        }
        __syncthreads();   // W_r^T written
        // lane l takes the row's 8-element chunks l, l + 32, ...: the warp's
        // tokens' x straight from global memory (512 contiguous bytes a row
        // per warp load, kXUnroll chunks of every token in flight), the eight
        // experts' weights of the chunk's input features from shared memory
        float acc[kTokPerWarp][kExpPerPass];
#pragma unroll
        for (int q = 0; q < kTokPerWarp; ++q)
#pragma unroll
            for (int e = 0; e < kExpPerPass; ++e) acc[q][e] = 0.f;
        constexpr int kXUnroll = sizeof(T) == 2 ? 4 : 2;
#pragma unroll 1
        for (int cb = lane; cb < nchunk; cb += 32 * kXUnroll) {
            RawVec8<T> xr[kXUnroll][kTokPerWarp];
#pragma unroll
            for (int u = 0; u < kXUnroll; ++u) {
                const int c = cb + 32 * u;
#pragma unroll
                for (int q = 0; q < kTokPerWarp; ++q)
                    if (c < nchunk && q < nt) raw_load8(x + (size_t)(c0tok + q0 + q) * d + (size_t)c * 8, xr[u][q]);
            }
#pragma unroll
            for (int u = 0; u < kXUnroll; ++u) {
                const int c = cb + 32 * u;
                if (c >= nchunk) break;
                float xv[kTokPerWarp][8];
#pragma unroll
                for (int q = 0; q < kTokPerWarp; ++q) {
                    if (q < nt) {
                        unpack8(xr[u][q], xv[q]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j) xv[q][j] = 0.f;
                    }
                }
#pragma unroll
                for (int e = 0; e < kExpPerPass; ++e) {
                    float wv[8];
                    load8(wt + (size_t)e * d + (size_t)c * 8, wv);
#pragma unroll
                    for (int q = 0; q < kTokPerWarp; ++q)
#pragma unroll
                        for (int j = 0; j < 8; ++j) acc[q][e] = fmaf(xv[q][j], wv[j], acc[q][e]);
                }
            }
        }
    // butterfly sums: every lane ends with the same bits
#pragma unroll
        for (int q = 0; q < kTokPerWarp; ++q)
#pragma unroll
            for (int e = 0; e < kExpPerPass; ++e) {
                float v = acc[q][e];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                acc[q][e] = v;
            }
        // expert e0 + e belongs to lane (e0 + e) % 32, register (e0 + e) / 32
        const int ir = e0 >> 5;
#pragma unroll
        for (int e = 0; e < kExpPerPass; ++e) {
            if (lane == ((e0 + e) & 31) && e0 + e < E) {
#pragma unroll
                for (int q = 0; q < kTokPerWarp; ++q) {
#pragma unroll
                    for (int i = 0; i < EPL; ++i)
                        if (i == ir) zt[q][i] = acc[q][e];
                }
            }
        }
    }
    __syncthreads();   // the chunk's counters are zeroed
    fused_select<EPL>(zt, nt, c0tok + q0, bias_mode, gate_mode, kk, E, k, lane, a, cnt, logits, idx_out, gate_out);
    sel_finish<EPL>(a, chunk, NB, E, kk, warp, lane, cnt, ps, ext, blockcnt, blockpsum, blockextra);
}

// ---- fused router, bf16: the logits on the warp-level MMA ------------------
// The same block and selection as route_fused_kernel (one block of 8 warps
// per chunk of kChunk tokens), with the dot products of the logits done by
// mma.sync (m16n8k16, bf16 products exact in fp32, fp32 accumulate) instead
// of fp32 FMAs: less than half the instructions. With one block of 8 warps
// per SM, its time goes to three latency-bound phases in turn: staging
// W_r^T, streaming x through the MMAs, and the selection.
//
// Operands. A is W_r^T of the pass's experts (16 expert rows per MMA; an
// 8-row half past the pass's experts is fed as zeros, and the rows of a
// partial half are zero-filled), kept in shared memory for the whole pass.
// B is 8 token rows of x. Warp w takes token octet w % 4 of the chunk and
// the 128-element items h, h + 2, h + 4, ... of the row, h = w / 4;
// each warp streams its items through its own ring of kRmStages shared-memory
// buffers with 16-byte cp.async copies (a half-warp copies 256 contiguous
// bytes of one row). For a 32-element chunk at kb, lane (g, t) takes the 8
// values at kb + 8t of A row g (and g + 8) and of token row g: values 0-3 feed
// one MMA, 4-7 a second, so each k of the chunk is multiplied once (the order
// of k inside an MMA is not memory order; a dot product does not see it).
// Piece p of staged token row r sits at position p ^ sw(r) in its 256-byte
// row, W_r^T rows are 2d + 64 bytes apart: the fragment reads of a quarter
// warp fall in eight different bank groups.
//
// The two K halves of each octet meet in shared memory: half 1 stores its
// partial logits, half 0 adds its own (a fixed order), and the selection
// reads the chunk's logits from there. Passes of P experts (P a multiple of
// 8, W_r^T of P experts within kRmWtMaxBytes) cover E <= 64; each pass reads
// x again (from L2 after the first).
constexpr int kRmItemK = 128;                                        // K elements per staged item
constexpr int kRmItemBytes = 8 * kRmItemK * 2;                       // 8 token rows of it
constexpr int kRmStages = 6;                                         // items in each warp's ring
constexpr int kRmZStride = 64;                                       // logits tile: up to 64 experts a token
constexpr size_t kRmRingBytes = (size_t)kSelWarps * kRmStages * kRmItemBytes;   // 96 KB
constexpr size_t kRmZBytes = (size_t)kChunk * kRmZStride * sizeof(float);         // 8 KB
constexpr size_t kRmWtMaxBytes = 84 * 1024;
constexpr size_t kRmSmemMax = kRmRingBytes + kRmZBytes + kRmWtMaxBytes;

int rm_row_bytes(int d) { return 2 * d + 64; }
// experts per pass (0: not even eight rows of W_r^T fit)
int rm_pass_experts(int d, int E) {
    const int fit = (int)(kRmWtMaxBytes / (size_t)rm_row_bytes(d)) / 8 * 8;
    return std::min(fit, std::min(64, ceil_div(E, 8) * 8));
}
bool route_fused_mma_ok(int d, int E) {
    static const bool enabled = [] {
        const char* v = std::getenv("MOE_ROUTER_MMA");
        return !(v != nullptr && v[0] == '0');
    }();
    return enabled && E <= 64 && d % 8 == 0 && rm_pass_experts(d, E) >= 8;
}

__device__ __forceinline__ int rm_swz(int r) { return ((r & 1) << 2) | ((r >> 1) & 3); }

template <int EPL, int GM>
__global__ void __launch_bounds__(kSelWarps * 32, 1)
route_fused_mma_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ W_r,
                       const float* __restrict__ bias, int bias_mode, int gate_mode, int kk, int Tn, int d, int E,
                       int k, int P, float* __restrict__ logits, int32_t* __restrict__ idx_out,
                       float* __restrict__ gate_out, int32_t* __restrict__ blockcnt, float* __restrict__ blockpsum,
                       float* __restrict__ blockextra, int32_t* __restrict__ status) {
    static_assert(EPL <= 2, "fused router: E <= 64");
    constexpr int kTokPerWarp = kChunk / kSelWarps;   // 4
    constexpr int NS = kRmStages;
    __shared__ int cnt[kMaxSlotCounts];
    __shared__ float ps[kSelWarps][MOE_MAX_E];
    __shared__ float ext[kSelWarps][3];
    extern __shared__ __align__(128) uint8_t rm_smem[];
    // [kSelWarps][NS] item buffers, the chunk's logits [kChunk][kRmZStride],
    // then W_r^T of the pass [P][2d + 64 bytes]
    float* zl = reinterpret_cast<float*>(rm_smem + kRmRingBytes);
    const uint32_t wt = smem_addr(rm_smem + kRmRingBytes + kRmZBytes);
    pdl_wait();
    pdl_launch();
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *status = MOE_OK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int chunk = blockIdx.x, NB = gridDim.x;
    for (int e = threadIdx.x; e < E * kk; e += blockDim.x) cnt[e] = 0;
    SelAcc<EPL> a;
    sel_init(a, bias, bias_mode, E, lane);
    const int c0tok = chunk * kChunk;
    const int ntok = min(kChunk, Tn - c0tok);
    const int rs = 2 * d + 64;

    const int gid = lane >> 2, tig = lane & 3;
    const int oct = warp & 3, half = warp >> 2;
    const int S = (d + kRmItemK - 1) / kRmItemK;
    const int nmine = (S - half + 1) / 2;                 // this warp's items: half, half + 2, ...
    const uint32_t ring = smem_addr(rm_smem + (size_t)warp * NS * kRmItemBytes);

    // the lane's four copies of an item: piece lane % 16 of rows 2i + lane / 16
    const int pc = lane & 15;
    const __nv_bfloat16* xsrc[4];
    uint32_t xdst[4];
    bool xrow[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int r = 2 * i + (lane >> 4);
        xrow[i] = oct * 8 + r < ntok;
        xsrc[i] = x + (size_t)(xrow[i] ? c0tok + oct * 8 + r : c0tok) * d + pc * 8;
        xdst[i] = (uint32_t)(r * (kRmItemK * 2) + ((pc ^ rm_swz(r)) << 4));
    }
    // copy this warp's item m into ring slot `slot`; always one commit group
    // (empty past the end), so the wait counts stay aligned
    auto issue = [&](int slot, int m) {
        if (m < nmine) {
            const int k0 = (half + 2 * m) * kRmItemK;
            const bool pin = pc * 8 < d - k0;   // the piece lies inside the row
            const uint32_t dst = ring + (uint32_t)slot * kRmItemBytes;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (pin && xrow[i]) cp_async16(dst + xdst[i], xsrc[i] + k0);
        }
        cp_async_commit();
    };

    for (int e0 = 0; e0 < E; e0 += P) {
        const int pe = min(P, E - e0);
#pragma unroll
        for (int s = 0; s < NS - 1; ++s) issue(s, s);
        __syncthreads();   // the previous pass's W_r^T and logits are consumed
        // W_r^T [e0, e0 + pe) x [0, d): the rows of W_r hold the E weights of
        // one input feature each
        if (E % 8 == 0) {
            // features (r, r + 1) x 8 experts: two 16-byte loads, eight
            // 4-byte stores of (feature r, feature r + 1) pairs
            // (kStage pairs of loads in flight per thread)
            constexpr int kStage = 8;
            const int hd = d / 2;
            const int n = hd * (pe / 8);
            for (int it0 = threadIdx.x; it0 < n; it0 += kStage * blockDim.x) {
                uint4 u0[kStage], u1[kStage];
#pragma unroll
                for (int b = 0; b < kStage; ++b) {
                    const int it = it0 + b * (int)blockDim.x;
                    if (it < n) {
                        const int c = it / hd, r = 2 * (it - c * hd);
                        const __nv_bfloat16* src = W_r + (size_t)r * E + e0 + 8 * c;
                        u0[b] = __ldg(reinterpret_cast<const uint4*>(src));
                        u1[b] = __ldg(reinterpret_cast<const uint4*>(src + E));
                    }
                }
#pragma unroll
                for (int b = 0; b < kStage; ++b) {
                    const int it = it0 + b * (int)blockDim.x;
                    if (it < n) {
                        const int c = it / hd, r = 2 * (it - c * hd);
                        const uint32_t w0[4] = {u0[b].x, u0[b].y, u0[b].z, u0[b].w};
                        const uint32_t w1[4] = {u1[b].x, u1[b].y, u1[b].z, u1[b].w};
                        const uint32_t base = wt + (uint32_t)(8 * c) * rs + (uint32_t)r * 2;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            sts32(base + (uint32_t)(2 * i) * rs, __byte_perm(w0[i], w1[i], 0x5410));
                            sts32(base + (uint32_t)(2 * i + 1) * rs, __byte_perm(w0[i], w1[i], 0x7632));
                        }
                    }
                }
            }
        } else {
            // rows pe .. pe8 - 1 are zeros, so that 8-row halves are whole
            __nv_bfloat16* wtp = reinterpret_cast<__nv_bfloat16*>(rm_smem + kRmRingBytes + kRmZBytes);
            const int pe8 = (pe + 7) / 8 * 8;
            for (int it = threadIdx.x; it < pe8 * d; it += blockDim.x) {
                const int e = it / d, r = it - e * d;
                wtp[(size_t)e * (rs / 2) + r] = e < pe ? W_r[(size_t)r * E + e0 + e] : __float2bfloat16(0.f);
            }
        }
        __syncthreads();   // W_r^T written

        // independent accumulator sets (with one 16-row group, one per MMA of
        // an item: 8; otherwise one per 32-element chunk: 4), so that no MMA
        // waits for the one before it; the sets are summed in a fixed order
        // at the end of the pass
        constexpr int NSET = GM == 1 ? 2 * (kRmItemK / 32) : kRmItemK / 32;
        float accu[GM][NSET][4];
#pragma unroll
        for (int G = 0; G < GM; ++G)
#pragma unroll
            for (int u = 0; u < NSET; ++u) accu[G][u][0] = accu[G][u][1] = accu[G][u][2] = accu[G][u][3] = 0.f;
        const int g16 = (pe + 15) / 16;
        const int pe8 = (pe + 7) / 8 * 8;   // W^T rows present (zeros past pe)
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
        for (int m = 0; m < nmine; ++m) {
            issue((m + NS - 1) % NS, m + NS - 1);
            cp_async_wait<NS - 1>();
            __syncwarp();
            const uint32_t buf = ring + (uint32_t)(m % NS) * kRmItemBytes;
            const int k0 = (half + 2 * m) * kRmItemK;
            // the lane's 8 elements of chunk u start at kb(u) = k0 + 32u + 8t
            // (d % 8 == 0: all inside the row or all outside); a whole item
            // needs no checks. Rows of the item past the chunk's tokens hold
            // stale data: they only feed their own columns of D, which are
            // never read. Expert halves are whole (8 rows, zeros past pe).
            const bool full = k0 + kRmItemK <= d;
            uint4 xb[kRmItemK / 32];
#pragma unroll
            for (int u = 0; u < kRmItemK / 32; ++u) {
                const uint32_t a = buf + (uint32_t)(gid * (kRmItemK * 2) + (((4 * u + tig) ^ rm_swz(gid)) << 4));
                xb[u] = (full || k0 + 32 * u + 8 * tig < d) ? lds128(a) : z4;
            }
#pragma unroll
            for (int G = 0; G < GM; ++G) {
                if (G < g16) {
                    const int ea = 16 * G + gid, eb = ea + 8;
                    const bool hi = 16 * G + 8 < pe8;   // the upper 8-row half holds experts
                    uint4 wa[kRmItemK / 32], wb[kRmItemK / 32];
#pragma unroll
                    for (int u = 0; u < kRmItemK / 32; ++u) {
                        const int kb = k0 + 32 * u + 8 * tig;
                        const bool kin = full || kb < d;
                        wa[u] = kin ? lds128(wt + (uint32_t)ea * rs + (uint32_t)kb * 2) : z4;
                        wb[u] = (hi && kin) ? lds128(wt + (uint32_t)eb * rs + (uint32_t)kb * 2) : z4;
                    }
#pragma unroll
                    for (int u = 0; u < kRmItemK / 32; ++u)
                        mma_bf16(accu[G][u], wa[u].x, wb[u].x, wa[u].y, wb[u].y, xb[u].x, xb[u].y);
#pragma unroll
                    for (int u = 0; u < kRmItemK / 32; ++u)
                        mma_bf16(accu[G][(u + kRmItemK / 32) % NSET], wa[u].z, wb[u].z, wa[u].w, wb[u].w, xb[u].z,
                                 xb[u].w);
                }
            }
            __syncwarp();   // the buffer is refilled by a later issue()
        }
        cp_async_wait<0>();
        float acc[GM][4];
#pragma unroll
        for (int G = 0; G < GM; ++G)
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v = accu[G][0][c];
#pragma unroll
                for (int u = 1; u < NSET; ++u) v += accu[G][u][c];
                acc[G][c] = v;
            }
        // D element (expert e0 + 16G + g (+ 8), token 8 oct + 2t (+ 1)):
        // half 1 stores its partial sums, half 0 adds its own to them
        auto zat = [&](int G, int c) -> float* {
            const int e = 16 * G + gid + ((c & 2) ? 8 : 0);
            const int tok = oct * 8 + 2 * tig + (c & 1);
            return zl + tok * kRmZStride + e0 + e;
        };
        if (half == 1) {
#pragma unroll
            for (int G = 0; G < GM; ++G)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (G < g16 && 16 * G + gid + ((c & 2) ? 8 : 0) < pe) *zat(G, c) = acc[G][c];
        }
        __syncthreads();
        if (half == 0) {
#pragma unroll
            for (int G = 0; G < GM; ++G)
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (G < g16 && 16 * G + gid + ((c & 2) ? 8 : 0) < pe) {
                        float* q = zat(G, c);
                        *q = acc[G][c] + *q;
                    }
        }
    }
    __syncthreads();   // the chunk's logits are complete (and its counters zeroed)
    const int q0 = warp * kTokPerWarp;
    const int nt = max(0, min(kTokPerWarp, ntok - q0));
    float zt[kTokPerWarp][EPL];
#pragma unroll
    for (int q = 0; q < kTokPerWarp; ++q)
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            const int e = lane + 32 * i;
            zt[q][i] = e < E ? zl[(q0 + q) * kRmZStride + e] : -INFINITY;
        }
    fused_select<EPL>(zt, nt, c0tok + q0, bias_mode, gate_mode, kk, E, k, lane, a, cnt, logits, idx_out, gate_out);
    sel_finish<EPL>(a, chunk, NB, E, kk, warp, lane, cnt, ps, ext, blockcnt, blockpsum, blockextra);
}

bool route_fused_ok(int dtype, int d, int E) {
    return E <= 64 && d % 8 == 0 && (dtype == MOE_DTYPE_F32 || dtype == MOE_DTYPE_BF16) &&
           fused_smem_bytes<float>(d) / (dtype == MOE_DTYPE_BF16 ? 2 : 1) <= kFusedWtMaxBytes;
}

cudaError_t launch_route_fused(int dtype, const void* x, const void* W_r, const float* bias, int bias_mode,
                               int gate_mode, int kk, int T, int d, int E, int k, float* logits, int32_t* idx,
                               float* gate, int32_t* blockcnt, float* blockpsum, float* blockextra, int32_t* status,
                               cudaStream_t st) {
    const int NB = ceil_div(T, kChunk);
    if (NB == 0) return cudaSuccess;
    dim3 grid(NB), block(kSelWarps * 32);
    // the staged operands (up to 160 KB; 188 KB for the MMA form) are dynamic
    // shared memory beside the selection's static arrays: opted in once per
    // device and variant
    static bool attr_set[64][8] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (dtype == MOE_DTYPE_BF16 && route_fused_mma_ok(d, E)) {
        const int P = rm_pass_experts(d, E);
        const size_t smem = kRmRingBytes + kRmZBytes + (size_t)P * rm_row_bytes(d);
#define MOE_FUSED_MMA(EPLV, GMV, SLOT)                                                                               \
    do {                                                                                                             \
        if (!attr_set[dev][SLOT]) {                                                                                  \
            cudaError_t e_ = cudaFuncSetAttribute(route_fused_mma_kernel<EPLV, GMV>,                                 \
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kRmSmemMax);     \
            if (e_ != cudaSuccess) return e_;                                                                        \
            attr_set[dev][SLOT] = true;                                                                              \
        }                                                                                                            \
        return launch_k(route_fused_mma_kernel<EPLV, GMV>, grid, block, smem, st, (const __nv_bfloat16*)x,           \
                        (const __nv_bfloat16*)W_r, bias, bias_mode, gate_mode, kk, T, d, E, k, P, logits, idx, gate, \
                        blockcnt, blockpsum, blockextra, status);                                                    \
    } while (0)
        // GM: 16-row expert groups a pass needs (one up to 16 experts a pass)
        if (E <= 32) {
            if (P <= 16) MOE_FUSED_MMA(1, 1, 4);
            MOE_FUSED_MMA(1, 4, 5);
        }
        if (P <= 16) MOE_FUSED_MMA(2, 1, 6);
        MOE_FUSED_MMA(2, 4, 7);
#undef MOE_FUSED_MMA
    }
#define MOE_FUSED(TYPE, EPLV, SLOT)                                                                                  \
    do {                                                                                                             \
        if (!attr_set[dev][SLOT]) {                                                                                  \
            cudaError_t e_ = cudaFuncSetAttribute(route_fused_kernel<TYPE, EPLV>,                                    \
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize,                       \
                                                  (int)kFusedWtMaxBytes);                                            \
            if (e_ != cudaSuccess) return e_;                                                                        \
            attr_set[dev][SLOT] = true;                                                                              \
        }                                                                                                            \
        return launch_k(route_fused_kernel<TYPE, EPLV>, grid, block, fused_smem_bytes<TYPE>(d), st, (const TYPE*)x, \
                        (const TYPE*)W_r,                                                                            \
                        bias, bias_mode, gate_mode, kk, T, d, E, k, logits, idx, gate, blockcnt, blockpsum,         \
                        blockextra, status);                                                                         \
    } while (0)
    if (dtype == MOE_DTYPE_BF16) {
        if (E <= 32) MOE_FUSED(__nv_bfloat16, 1, 0);
        MOE_FUSED(__nv_bfloat16, 2, 1);
    }
    if (E <= 32) MOE_FUSED(float, 1, 2);
    MOE_FUSED(float, 2, 3);
#undef MOE_FUSED
}

cudaError_t launch_select(const float* logits, const float* bias, int bias_mode, int gate_mode, int kk, int T,
                          int E, int k, int32_t* idx, float* gate, int32_t* blockcnt, float* blockpsum,
                          float* blockextra, cudaStream_t st) {
    int NB = ceil_div(T, kChunk);
    if (NB == 0) return cudaSuccess;
    dim3 grid(NB), block(kSelWarps * 32);
    int epl = ceil_div(E, 32);
#define MOE_SELECT(EPLV)                                                                                        \
    return launch_k(select_kernel<EPLV>, grid, block, 0, st, logits, bias, bias_mode, gate_mode, kk, T, E, k, idx, \
                    gate, blockcnt, blockpsum, blockextra)
    if (epl <= 1) MOE_SELECT(1);
    if (epl <= 2) MOE_SELECT(2);
    if (epl <= 4) MOE_SELECT(4);
    if (epl <= 8) MOE_SELECT(8);
    MOE_SELECT(16);
#undef MOE_SELECT
}

// ---- per-chunk histogram of given selections (standalone permutation) ----
__global__ void hist_kernel(const int32_t* __restrict__ idx, int Tn, int k, int kk, int E,
                            int32_t* __restrict__ blockcnt) {
    __shared__ int cnt[kMaxSlotCounts];
    pdl_wait();
    pdl_launch();
    const int chunk = blockIdx.x, NB = gridDim.x;
    for (int e = threadIdx.x; e < E * kk; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    const int t0 = chunk * kChunk;
    const int n = min(kChunk, Tn - t0) * k;
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        int e = idx[(size_t)t0 * k + i];
        if (e >= 0 && e < E) atomicAdd(&cnt[e * kk + (kk > 1 ? i % k : 0)], 1);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < E * kk; i += blockDim.x) blockcnt[(size_t)i * NB + chunk] = cnt[i];
}

cudaError_t launch_hist(const int32_t* idx, int T, int k, int kk, int E, int32_t* blockcnt, cudaStream_t st) {
    int NB = ceil_div(T, kChunk);
    if (NB == 0) return cudaSuccess;
    return launch_k(hist_kernel, dim3(NB), dim3(256), 0, st, idx, T, k, kk, E, blockcnt);
}

}  // namespace moe
