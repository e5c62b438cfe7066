// Backward pass of the MoE layer outside the grouped GEMMs: the gate-scaled
// gather of the output gradient, the router-logit gradient, the router
// weight gradient, the input gradient and the auxiliary-loss-free bias
// update. The loss is L = <dy, y> + alpha L_aux + beta L_z.
//
//  * combine y_t = sum_j g_{t,j} o_{t,j} ("Lecture 21 · LLM: Mixture-of-
//    Experts" §3.2 step 4): dO[pos] = g dy_t, dgate_{t,j} = <dy_t, o_{t,j}>;
//  * gates, softmax of the selected raw logits ("Week 2 Day 2: Mixture of
//    Experts" §1.3): dz_{e_j} += g_j (dg_j - sum_l g_l dg_l); full-softmax
//    gates: dz += p (v - <p, v>), v_{e_j} = dg_j;
//  * balance loss with f frozen (same page §3.2): dz_{t,i} += alpha E/T
//    p_{t,i} (f_i - sum_j p_{t,j} f_j); z-loss (§3.4): dz += beta 2/T lse p;
//  * router z = W_r^T x: dW_r = x^T dz, dx += W_r dz;
//  * bias update ("Lecture 21" §2.4): above-mean experts b -= gamma, below
//    b += gamma, decided exactly by the sign of c_e E - T k.
// Every reduction runs in a fixed order; no atomics.
#include <algorithm>

#include "common.cuh"

namespace moe {

namespace {

__device__ __forceinline__ float wsum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float wmax(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ void unpack8(const uint4& u, float (&v)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

constexpr int kWarps = 8;

// One warp per (token, slot): the gate-scaled gradient row and the gate's
// gradient (lane-strided partial dot products, then a butterfly).
__global__ void __launch_bounds__(kWarps * 32)
bwd_gather_kernel(const __nv_bfloat16* __restrict__ dy, const __nv_bfloat16* __restrict__ o,
                  const int32_t* __restrict__ pos, const float* __restrict__ gate, int npairs, int d, int k,
                  __nv_bfloat16* __restrict__ dO, float* __restrict__ dgate) {
    pdl_wait();
    pdl_launch();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pr = blockIdx.x * kWarps + warp;
    if (pr >= npairs) return;
    const int t = pr / k;
    const int r = pos[pr];
    if (r < 0) {
        if (lane == 0) dgate[pr] = 0.f;
        return;
    }
    const float g = gate[pr];
    const int nvec = d / 8;
    const uint4* dyv = reinterpret_cast<const uint4*>(dy + static_cast<size_t>(t) * d);
    const uint4* ov = reinterpret_cast<const uint4*>(o + static_cast<size_t>(r) * d);
    uint4* dov = reinterpret_cast<uint4*>(dO + static_cast<size_t>(r) * d);
    float acc = 0.f;
    for (int v = lane; v < nvec; v += 32) {
        float a[8], b[8];
        unpack8(dyv[v], a);
        unpack8(ov[v], b);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc = fmaf(a[i], b[i], acc);
        dov[v] = make_uint4(pack2(g * a[0], g * a[1]), pack2(g * a[2], g * a[3]), pack2(g * a[4], g * a[5]),
                            pack2(g * a[6], g * a[7]));
    }
    acc = wsum(acc);
    if (lane == 0) dgate[pr] = acc;
}

constexpr int kMaxEPL = MOE_MAX_E / 32;   // experts per lane

// One warp per token: softmax of its logits, then the three terms of dz.
__global__ void __launch_bounds__(kWarps * 32)
router_bwd_kernel(const float* __restrict__ logits, const int32_t* __restrict__ idx, const float* __restrict__ gate,
                  const float* __restrict__ dgate, const void* __restrict__ stats, int T, int E, int k,
                  int gate_mode, float alpha, float beta, float* __restrict__ dz, __nv_bfloat16* __restrict__ dz16) {
    pdl_wait();
    pdl_launch();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * kWarps + warp;
    if (t >= T) return;
    const float* f = MOE_STATS_F(stats, E);
    const int epl = (E + 31) / 32;
    float z[kMaxEPL], p[kMaxEPL], g[kMaxEPL];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kMaxEPL; ++i) {
        const int e = lane + 32 * i;
        z[i] = (i < epl && e < E) ? logits[static_cast<size_t>(t) * E + e] : -INFINITY;
        m = fmaxf(m, z[i]);
    }
    m = wmax(m);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kMaxEPL; ++i) {
        const int e = lane + 32 * i;
        p[i] = (i < epl && e < E) ? expf(z[i] - m) : 0.f;
        s += p[i];
    }
    s = wsum(s);
    const float inv = 1.f / s;
#pragma unroll
    for (int i = 0; i < kMaxEPL; ++i) {
        p[i] *= inv;
        g[i] = 0.f;
    }
    const int32_t* it = idx + static_cast<size_t>(t) * k;
    const float* gt = gate + static_cast<size_t>(t) * k;
    const float* dgt = dgate + static_cast<size_t>(t) * k;
    if (gate_mode == MOE_GATE_SELECTED) {
        float sg = 0.f;   // sum_l g_l dg_l, slot order
        for (int j = 0; j < k; ++j) sg += gt[j] * dgt[j];
        for (int j = 0; j < k; ++j) {
            const int e = it[j];
            if ((e & 31) == lane) {
                const float add = gt[j] * (dgt[j] - sg);
#pragma unroll
                for (int i = 0; i < kMaxEPL; ++i)
                    if ((e >> 5) == i) g[i] += add;
            }
        }
    } else {
        float v[kMaxEPL];
#pragma unroll
        for (int i = 0; i < kMaxEPL; ++i) v[i] = 0.f;
        for (int j = 0; j < k; ++j) {
            const int e = it[j];
            if ((e & 31) == lane) {
#pragma unroll
                for (int i = 0; i < kMaxEPL; ++i)
                    if ((e >> 5) == i) v[i] += dgt[j];
            }
        }
        float pv = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxEPL; ++i) pv += p[i] * v[i];
        pv = wsum(pv);
#pragma unroll
        for (int i = 0; i < kMaxEPL; ++i) g[i] += p[i] * (v[i] - pv);
    }
    if (alpha != 0.f) {
        float pf = 0.f;
#pragma unroll
        for (int i = 0; i < kMaxEPL; ++i) {
            const int e = lane + 32 * i;
            if (i < epl && e < E) pf += p[i] * f[e];
        }
        pf = wsum(pf);
        const float c = alpha * static_cast<float>(E) / static_cast<float>(T);
#pragma unroll
        for (int i = 0; i < kMaxEPL; ++i) {
            const int e = lane + 32 * i;
            if (i < epl && e < E) g[i] += c * p[i] * (f[e] - pf);
        }
    }
    if (beta != 0.f) {
        const float lse = m + logf(s);
        const float c = beta * 2.f / static_cast<float>(T) * lse;
#pragma unroll
        for (int i = 0; i < kMaxEPL; ++i) g[i] += c * p[i];
    }
#pragma unroll
    for (int i = 0; i < kMaxEPL; ++i) {
        const int e = lane + 32 * i;
        if (i < epl && e < E) {
            dz[static_cast<size_t>(t) * E + e] = g[i];
            if (dz16 != nullptr) dz16[static_cast<size_t>(t) * E + e] = __float2bfloat16_rn(g[i]);
        }
    }
}

// dW_r[i][e] = sum_t x[t][i] dz[t][e] in two fixed-order passes: block
// (i-block, token chunk, expert group) sums its kDwrTok tokens into a
// partial, then the partials are summed over chunks in order. A thread owns
// two columns and a group of experts; the chunk's dz rows are staged in
// shared memory.
constexpr int kDwrTok = 128;   // tokens per chunk

template <int EB>   // experts per block (grid z): 8 for routers of 8, 32 otherwise
__global__ void __launch_bounds__(256)
dwr_partial_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ dz, int T, int d, int E,
                   float* __restrict__ part) {
    __shared__ float dzs[kDwrTok][EB];
    pdl_wait();
    pdl_launch();
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);   // two consecutive columns
    const int t0 = blockIdx.y * kDwrTok;
    const int e0 = blockIdx.z * EB;
    const int ne = min(EB, E - e0);
    const int nt = min(kDwrTok, T - t0);
    for (int q = threadIdx.x; q < kDwrTok * EB; q += blockDim.x) {
        const int tt = q / EB, ee = q % EB;
        dzs[tt][ee] = (tt < nt && ee < ne) ? dz[static_cast<size_t>(t0 + tt) * E + e0 + ee] : 0.f;
    }
    __syncthreads();
    if (i >= d) return;
    float a0[EB], a1[EB];
#pragma unroll
    for (int e = 0; e < EB; ++e) a0[e] = a1[e] = 0.f;
    const __nv_bfloat162* xc = reinterpret_cast<const __nv_bfloat162*>(x + static_cast<size_t>(t0) * d + i);
#pragma unroll 4
    for (int tt = 0; tt < nt; ++tt) {
        const float2 xv = __bfloat1622float2(xc[static_cast<size_t>(tt) * (d / 2)]);
#pragma unroll
        for (int e = 0; e < EB; ++e) {
            a0[e] = fmaf(xv.x, dzs[tt][e], a0[e]);
            a1[e] = fmaf(xv.y, dzs[tt][e], a1[e]);
        }
    }
    float* out = part + (static_cast<size_t>(blockIdx.y) * d + i) * E + e0;
#pragma unroll
    for (int e = 0; e < EB; ++e)
        if (e < ne) {
            out[e] = a0[e];
            out[E + e] = a1[e];
        }
}

__global__ void __launch_bounds__(256)
dwr_reduce_kernel(const float* __restrict__ part, int nchunks, int d, int E, float* __restrict__ dW_r) {
    pdl_wait();
    pdl_launch();
    const size_t n = static_cast<size_t>(d) * E;
    for (size_t q = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x; q < n;
         q += static_cast<size_t>(gridDim.x) * blockDim.x) {
        float s = 0.f;
        for (int c = 0; c < nchunks; ++c) s += part[static_cast<size_t>(c) * n + q];
        dW_r[q] = s;
    }
}

// dx_t = sum_j dXp[pos_{t,j}] + W_r dz_t (+ the shared expert's dXs_t). A
// thread owns 8 consecutive columns of dx for a tile of kDxTok tokens. The
// router term reads the thread's 8 rows of W_r [d][E] once per tile: with
// E <= 16 they are held in registers; wider routers walk the experts 8 at a
// time (one 16-byte load per row) and accumulate the tile's tokens from each
// load. (Rows of neighbouring threads are 8 E bytes apart, so reading them
// per token was bound by L1 wavefronts.) The tile's dz rows are staged in
// shared memory.
constexpr int kDxTok = 16;

template <int EG>   // E / 8 when E <= 16 (rows in registers), 0: E % 8 == 0, walked in groups of 8,
                   // -1: the router term is given (dxr [T][d] fp32, from the tensor cores)
__global__ void __launch_bounds__(256)
bwd_dx_kernel(const __nv_bfloat16* __restrict__ dXp, const int32_t* __restrict__ pos,
              const __nv_bfloat16* __restrict__ W_r, const float* __restrict__ dz,
              const __nv_bfloat16* __restrict__ dXs, const float* __restrict__ dxr, int T, int d, int E, int k,
              __nv_bfloat16* __restrict__ dx) {
    constexpr int TT = EG > 0 ? kDxTok : 8;   // tokens per tile
    extern __shared__ float dzs[];             // [TT][E]
    pdl_wait();
    pdl_launch();
    const int t0 = blockIdx.x * TT;
    const int nt = min(TT, T - t0);
    for (int q = threadIdx.x; q < nt * E; q += blockDim.x) dzs[q] = dz[static_cast<size_t>(t0) * E + q];
    __syncthreads();
    const int v = blockIdx.y * blockDim.x + threadIdx.x;   // 8 consecutive columns
    if (v >= d / 8) return;
    // sum of the token's kept rows of dXp, plus the shared expert's input
    // gradient when there is one
    auto expert_terms = [&](int t, float (&sum)[8]) {
        for (int j = 0; j < k; ++j) {
            const int r = pos[static_cast<size_t>(t) * k + j];
            if (r < 0) continue;
            float a[8];
            unpack8(reinterpret_cast<const uint4*>(dXp + static_cast<size_t>(r) * d)[v], a);
#pragma unroll
            for (int c = 0; c < 8; ++c) sum[c] += a[c];
        }
        if (dXs != nullptr) {
            float a[8];
            unpack8(reinterpret_cast<const uint4*>(dXs + static_cast<size_t>(t) * d)[v], a);
#pragma unroll
            for (int c = 0; c < 8; ++c) sum[c] += a[c];
        }
    };
    auto store = [&](int t, const float (&sum)[8]) {
        reinterpret_cast<uint4*>(dx + static_cast<size_t>(t) * d)[v] =
            make_uint4(pack2(sum[0], sum[1]), pack2(sum[2], sum[3]), pack2(sum[4], sum[5]), pack2(sum[6], sum[7]));
    };
    if constexpr (EG > 0) {
        // few experts: rows 8v .. 8v+7 of W_r stay packed in registers, the
        // router term is formed token by token
        uint4 w[8][EG > 0 ? EG : 1];
#pragma unroll
        for (int c = 0; c < 8; ++c)
#pragma unroll
            for (int g = 0; g < EG; ++g)
                w[c][g] = reinterpret_cast<const uint4*>(W_r + static_cast<size_t>(8 * v + c) * E)[g];
        for (int tt = 0; tt < nt; ++tt) {
            const float* zt = dzs + tt * E;
            float sum[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                float acc = 0.f;
#pragma unroll
                for (int g = 0; g < EG; ++g) {
                    float wf[8];
                    unpack8(w[c][g], wf);
#pragma unroll
                    for (int q = 0; q < 8; ++q) acc = fmaf(wf[q], zt[8 * g + q], acc);
                }
                sum[c] = acc;
            }
            expert_terms(t0 + tt, sum);
            store(t0 + tt, sum);
        }
    } else {
        // router term of every token of the tile, acc[tt][c]: each group of
        // 8 experts' W_r rows is loaded once for the TT tokens
        float acc[TT][8];
#pragma unroll
        for (int tt = 0; tt < TT; ++tt)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[tt][c] = 0.f;
        const int groups = EG == 0 ? E / 8 : 0;
        for (int g = 0; g < groups; ++g) {
            float w[8][8];   // rows 8v .. 8v+7, experts 8g .. 8g+7
#pragma unroll
            for (int c = 0; c < 8; ++c)
                unpack8(reinterpret_cast<const uint4*>(W_r + static_cast<size_t>(8 * v + c) * E)[g], w[c]);
#pragma unroll
            for (int tt = 0; tt < TT; ++tt) {
                if (tt < nt) {
                    const float* zt = dzs + tt * E + 8 * g;
#pragma unroll
                    for (int c = 0; c < 8; ++c)
#pragma unroll
                        for (int q = 0; q < 8; ++q) acc[tt][c] = fmaf(w[c][q], zt[q], acc[tt][c]);
                }
            }
        }
#pragma unroll
        for (int tt = 0; tt < TT; ++tt) {
            if (tt >= nt) break;
            const int t = t0 + tt;
            float sum[8];
            if (EG == 0) {
#pragma unroll
                for (int c = 0; c < 8; ++c) sum[c] = acc[tt][c];
            } else {   // the router term comes from the tensor cores
                const float4* pr = reinterpret_cast<const float4*>(dxr + static_cast<size_t>(t) * d + 8 * v);
                const float4 r0 = pr[0], r1 = pr[1];
                sum[0] = r0.x; sum[1] = r0.y; sum[2] = r0.z; sum[3] = r0.w;
                sum[4] = r1.x; sum[5] = r1.y; sum[6] = r1.z; sum[7] = r1.w;
            }
            expert_terms(t, sum);
            store(t, sum);
        }
    }
}

__global__ void single_group_kernel(int32_t* indptr, int T) {
    pdl_wait();
    pdl_launch();
    if (threadIdx.x == 0) {
        indptr[0] = 0;
        indptr[1] = T;
    }
}

__global__ void bias_update_kernel(const void* __restrict__ stats, int T, int E, int k, float gamma,
                                   float* __restrict__ bias) {
    pdl_wait();
    pdl_launch();
    const int32_t* c = MOE_STATS_COUNTS(stats, E);
    const long long tk = static_cast<long long>(T) * k;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const long long s = static_cast<long long>(c[e]) * E - tk;   // sign of c_e - T k / E, exactly
        if (s > 0) bias[e] -= gamma;
        else if (s < 0) bias[e] += gamma;
    }
}

}  // namespace

cudaError_t launch_bwd_gather(const void* dy, const void* o, const int32_t* pos, const float* gate, int T, int d,
                              int k, void* dO, float* dgate, cudaStream_t st) {
    const int np = T * k;
    if (np == 0) return cudaSuccess;
    return launch_k(bwd_gather_kernel, dim3(ceil_div(np, kWarps)), dim3(kWarps * 32), 0, st,
                    static_cast<const __nv_bfloat16*>(dy), static_cast<const __nv_bfloat16*>(o), pos, gate, np, d, k,
                    static_cast<__nv_bfloat16*>(dO), dgate);
}

cudaError_t launch_router_bwd(const float* logits, const int32_t* idx, const float* gate, const float* dgate,
                              const void* stats, int T, int E, int k, int gate_mode, float alpha, float beta,
                              float* dz, void* dz16, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    return launch_k(router_bwd_kernel, dim3(ceil_div(T, kWarps)), dim3(kWarps * 32), 0, st, logits, idx, gate, dgate,
                    stats, T, E, k, gate_mode, alpha, beta, dz, static_cast<__nv_bfloat16*>(dz16));
}

cudaError_t launch_dwr(const void* x, const float* dz, int T, int d, int E, float* part, float* dW_r,
                       cudaStream_t st) {
    const int nchunks = ceil_div(T, kDwrTok);
    cudaError_t e;
    if (E <= 8)
        e = launch_k(dwr_partial_kernel<8>, dim3(ceil_div(d, 512), nchunks, 1), dim3(256), 0, st,
                     static_cast<const __nv_bfloat16*>(x), dz, T, d, E, part);
    else
        e = launch_k(dwr_partial_kernel<32>, dim3(ceil_div(d, 512), nchunks, ceil_div(E, 32)), dim3(256), 0, st,
                     static_cast<const __nv_bfloat16*>(x), dz, T, d, E, part);
    if (e != cudaSuccess) return e;
    const long long n = static_cast<long long>(d) * E;
    return launch_k(dwr_reduce_kernel, dim3(static_cast<unsigned>(std::min<long long>(ceil_div((int)n, 256), 1184))),
                    dim3(256), 0, st, static_cast<const float*>(part), nchunks, d, E, dW_r);
}

cudaError_t launch_bwd_dx(const void* dXp, const int32_t* pos, const void* W_r, const float* dz, const void* dXs,
                          const float* dxr, int T, int d, int E, int k, void* dx, cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    auto args = [&](auto kern, int tt) {
        const dim3 grid(ceil_div(T, tt), ceil_div(d / 8, 256));
        const size_t smem = sizeof(float) * tt * E;
        return launch_k(kern, grid, dim3(256), smem, st, static_cast<const __nv_bfloat16*>(dXp), pos,
                        static_cast<const __nv_bfloat16*>(W_r), dz, static_cast<const __nv_bfloat16*>(dXs), dxr, T,
                        d, E, k, static_cast<__nv_bfloat16*>(dx));
    };
    if (dxr != nullptr) return args(bwd_dx_kernel<-1>, 8);
    if (E == 8) return args(bwd_dx_kernel<1>, kDxTok);
    if (E == 16) return args(bwd_dx_kernel<2>, kDxTok);
    if (E % 8 == 0) return args(bwd_dx_kernel<0>, 8);
    return cudaErrorNotSupported;   // the backward requires E % 8 == 0
}

cudaError_t launch_single_group(int32_t* indptr, int T, cudaStream_t st) {
    return launch_k(single_group_kernel, dim3(1), dim3(32), 0, st, indptr, T);
}

cudaError_t launch_bias_update(const void* stats, int T, int E, int k, float gamma, float* bias, cudaStream_t st) {
    return launch_k(bias_update_kernel, dim3(1), dim3(512), 0, st, stats, T, E, k, gamma, bias);
}

}  // namespace moe
