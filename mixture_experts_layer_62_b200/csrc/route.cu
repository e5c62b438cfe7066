// Router: logits z = W_r^T x, selection key, top-k, gates and the per-chunk
// partial statistics.
//
// "Week 2 Day 2: Mixture of Experts" §1.3 (z = W_r^T x, T = TopK(z, k),
// g_i = exp(z_i) / sum_{j in T} exp(z_j)), §4.2 (selection on z + b, gates from
// the raw z), §3.2 (f_i and P_i of the balance loss); "Stanford CS336 Lecture
// 04" §2.3.3c (bias added to the softmax score). Router arithmetic is fp32
// ("Lecture 21 · LLM: Mixture-of-Experts" §7.1: the router runs in fp32).
#include "common.cuh"
#include "tc_common.cuh"

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
// select_kernel (warp w: tokens 4w .. 4w + 3 of the chunk). A warp computes
// its four tokens' logits itself: lane l takes the 8-element chunks c = l,
// l + 32, ... of the row (16-byte loads of x, four chunks in flight per
// token), multiplies them with the matching rows of W_r [d, E] as given (no
// transposed copy: a row of W_r holds the E weights of one input feature),
// eight experts per pass, and an xor butterfly leaves every lane with the
// sums, in a fixed order. The logits are written out (the workspace keeps
// them) and, still in registers, go through the same per-token selection as
// select_kernel. x is read once from HBM; W_r (d E elements) is re-read from
// L1/L2 by each warp. E <= 64.
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

// Rows of W_r (input features) a block stages at a time: 4 KB of x per token
// for the chunk's 32 tokens (128 KB; a whole Mixtral-sized row block would
// not fit), and W_r^T of those rows for eight experts (32 KB for bf16).
template <typename T>
constexpr int fused_slab() { return 4096 / (int)sizeof(T); }
template <typename T>
constexpr size_t fused_smem_bytes() {
    return (size_t)kChunk * fused_slab<T>() * sizeof(T) + (size_t)kExpPerPass * fused_slab<T>() * sizeof(T) + 64;
}

template <typename T, int EPL>
__global__ void __launch_bounds__(kSelWarps * 32)
route_fused_kernel(const T* __restrict__ x, const T* __restrict__ W_r, const float* __restrict__ bias,
                   int bias_mode, int gate_mode, int kk, int Tn, int d, int E, int k, float* __restrict__ logits,
                   int32_t* __restrict__ idx_out, float* __restrict__ gate_out, int32_t* __restrict__ blockcnt,
                   float* __restrict__ blockpsum, float* __restrict__ blockextra, int32_t* __restrict__ status) {
    static_assert(EPL <= 2, "fused router: E <= 64");
    constexpr int kTokPerWarp = kChunk / kSelWarps;   // 4
    constexpr int SLAB = fused_slab<T>();             // rows of W_r (columns of x) per slab
    __shared__ int cnt[kMaxSlotCounts];
    __shared__ float ps[kSelWarps][MOE_MAX_E];
    __shared__ float ext[kSelWarps][3];
    extern __shared__ __align__(128) uint8_t fused_dsm[];
    T* xs = reinterpret_cast<T*>(fused_dsm);                      // [kChunk][SLAB]: x of the slab
    T* wt = xs + (size_t)kChunk * SLAB;                           // [kExpPerPass][SLAB]: W_r^T of the slab
    uint64_t* xbar = reinterpret_cast<uint64_t*>(wt + (size_t)kExpPerPass * SLAB);
    pdl_wait();
    pdl_launch();
    if (status != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *status = MOE_OK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int chunk = blockIdx.x, NB = gridDim.x;
    for (int e = threadIdx.x; e < E * kk; e += blockDim.x) cnt[e] = 0;
    if (threadIdx.x == 0) {
        tc::mbar_init(xbar, 1);
        tc::fence_mbar_init();
    }
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
    uint32_t xph = 0;
    for (int e0 = 0; e0 < E; e0 += kExpPerPass) {
        float acc[kTokPerWarp][kExpPerPass];
#pragma unroll
        for (int q = 0; q < kTokPerWarp; ++q)
#pragma unroll
            for (int e = 0; e < kExpPerPass; ++e) acc[q][e] = 0.f;
        for (int d0 = 0; d0 < d; d0 += SLAB) {
            const int ns = min(SLAB, d - d0);
            __syncthreads();   // the previous slab is consumed (and the barrier initialised)
            // x of the block's tokens, columns [d0, d0 + ns): one bulk copy per
            // token row into the slab
            if (threadIdx.x == 0) {
                tc::fence_proxy_async_smem();   // the slab's earlier generic reads precede the copies
                tc::mbar_arrive_expect_tx(xbar, (uint32_t)(ntok * ns * (int)sizeof(T)));
                for (int q = 0; q < ntok; ++q)
                    tc::bulk_load(tc::smem_u32(xs + (size_t)q * SLAB), x + (size_t)(c0tok + q) * d + d0,
                                  (uint32_t)(ns * (int)sizeof(T)), xbar);
            }
            // W_r^T [e0 .. e0 + 7][d0 .. d0 + ns) (zeros past E): the rows
            // [d0, d0 + ns) of W_r are one contiguous run of ns E elements,
            // requested as 16-byte vectors, eight per thread, before any is
            // written, transposed, into the slab
            if (e0 + kExpPerPass > E)
                for (int i = threadIdx.x; i < kExpPerPass * ns; i += blockDim.x) wt[(i / ns) * SLAB + i % ns] = T(0.f);
            __syncthreads();
            {
                const T* src = W_r + (size_t)d0 * E;
                const int ng = ns * E / 8;
                for (int g0 = threadIdx.x; g0 < ng; g0 += blockDim.x * 8) {
                    RawVec8<T> wr[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int g = g0 + (int)blockDim.x * j;
                        if (g < ng) raw_load8(src + (size_t)g * 8, wr[j]);
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
                                for (int i = 0; i < 8; ++i) wt[i * SLAB + r] = T(v[i]);
                            }
                        } else {
#pragma unroll 1
                            for (int i = 0; i < 8; ++i) {
                                const int idx = g * 8 + i, r = idx / E, e = idx - r * E - e0;
                                if (e >= 0 && e < kExpPerPass) wt[e * SLAB + r] = T(v[i]);
                            }
                        }
                    }
                }
            }
            __syncthreads();   // W_r^T slab written
            // the x slab has landed (bulk copies of this block's own rows, which
            // complete on their own; the wait is still bounded)
            if (!tc::mbar_try_wait(xbar, xph)) {
                const uint64_t t0 = tc::global_timer_ns();
                while (!tc::mbar_try_wait(xbar, xph)) {
                    if (tc::global_timer_ns() - t0 > static_cast<uint64_t>(kDrainLimitNs)) {
                        if (status != nullptr) atomicExch(status, MOE_ERR_TIMEOUT);
                        break;
                    }
                }
            }
            xph ^= 1u;
            // lane l takes the slab's 8-element chunks l, l + 32, ...: the four
            // tokens' x and the eight experts' weights of the chunk's 8 input
            // features, all from shared memory
            const int nchunk = ns / 8;
#pragma unroll 1
            for (int c = lane; c < nchunk; c += 32) {
                float xv[kTokPerWarp][8];
#pragma unroll
                for (int q = 0; q < kTokPerWarp; ++q) {
                    if (q < nt) {
                        load8(xs + (size_t)(q0 + q) * SLAB + c * 8, xv[q]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j) xv[q][j] = 0.f;
                    }
                }
#pragma unroll
                for (int e = 0; e < kExpPerPass; ++e) {
                    float wv[8];
                    load8(wt + e * SLAB + c * 8, wv);
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
#pragma unroll
    for (int q = 0; q < kTokPerWarp; ++q) {
        if (q < nt) {
            const int t = c0tok + q0 + q;
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const int e = lane + 32 * i;
                if (e < E) logits[(size_t)t * E + e] = zt[q][i];
            }
            sel_token<EPL, true>(zt[q], t, bias_mode, gate_mode, kk, E, k, lane, a, cnt, idx_out, gate_out);
        }
    }
    sel_finish<EPL>(a, chunk, NB, E, kk, warp, lane, cnt, ps, ext, blockcnt, blockpsum, blockextra);
}

bool route_fused_ok(int dtype, int d, int E) {
    return E <= 64 && d % 8 == 0 && (dtype == MOE_DTYPE_F32 || dtype == MOE_DTYPE_BF16);
}

cudaError_t launch_route_fused(int dtype, const void* x, const void* W_r, const float* bias, int bias_mode,
                               int gate_mode, int kk, int T, int d, int E, int k, float* logits, int32_t* idx,
                               float* gate, int32_t* blockcnt, float* blockpsum, float* blockextra, int32_t* status,
                               cudaStream_t st) {
    const int NB = ceil_div(T, kChunk);
    if (NB == 0) return cudaSuccess;
    dim3 grid(NB), block(kSelWarps * 32);
    // the staged x and W_r slabs (160 KB) are dynamic shared memory beside
    // the selection's static arrays: opted in once per device and variant
    static bool attr_set[64][4] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
#define MOE_FUSED(TYPE, EPLV, SLOT)                                                                                  \
    do {                                                                                                             \
        if (!attr_set[dev][SLOT]) {                                                                                  \
            cudaError_t e_ = cudaFuncSetAttribute(route_fused_kernel<TYPE, EPLV>,                                    \
                                                  cudaFuncAttributeMaxDynamicSharedMemorySize,                       \
                                                  (int)fused_smem_bytes<TYPE>());                                    \
            if (e_ != cudaSuccess) return e_;                                                                        \
            attr_set[dev][SLOT] = true;                                                                              \
        }                                                                                                            \
        return launch_k(route_fused_kernel<TYPE, EPLV>, grid, block, fused_smem_bytes<TYPE>(), st, (const TYPE*)x,  \
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
