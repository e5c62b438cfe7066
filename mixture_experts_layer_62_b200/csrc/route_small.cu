// Small-batch router: the whole routing and permutation of a decode-sized
// batch (T*k <= 64 pairs) in one block of 512 threads, so a decode step
// spends one launch here instead of five.
//
// It computes the same quantities, with the same definitions, as the general
// path (route.cu, permute.cu): z = W_r^T x in fp32 ("Week 2 Day 2: Mixture of
// Experts" §1.3), the selection key and top-k with the lowest index winning
// ties, the gates as the softmax of the selected raw logits (§1.3, §4.2), the
// per-expert counts and mean probabilities (§3.2), capacity and the ranks of
// the pairs in token order inside each expert ("Lecture 21 · LLM:
// Mixture-of-Experts" §3.3, §3.5), indptr, the tile schedules of the grouped
// GEMMs with their split factors, and the gather of the permuted rows.
// Reductions run in a fixed order (the summation trees differ from the
// general path's, so the two paths agree to fp32 rounding, not bit for bit).
#include "common.cuh"

namespace moe {

namespace {

constexpr int kWarps = 16;
constexpr int kTokPass = 4;   // tokens per logits pass
constexpr int kMaxT = kSmallMaxPairs;

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
__device__ __forceinline__ void bf16x8(const uint4& u, float (&v)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

__global__ void __launch_bounds__(kWarps * 32) route_small_kernel(SmallRouteArgs a) {
    __shared__ float z[kMaxT][kSmallMaxE];
    __shared__ float part[kWarps][kTokPass][8];
    __shared__ float psw[kWarps][kSmallMaxE];
    __shared__ int cnt[kSmallMaxE];
    __shared__ int indptr_s[kSmallMaxE + 1];
    __shared__ int sidx[kSmallMaxPairs];
    __shared__ int spos[kSmallMaxPairs];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int T = a.T, d = a.d, E = a.E, k = a.k;
    const __nv_bfloat16* x = static_cast<const __nv_bfloat16*>(a.x);
    const __nv_bfloat16* W_r = static_cast<const __nv_bfloat16*>(a.W_r);

    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    for (int i = threadIdx.x; i < kWarps * kSmallMaxE; i += blockDim.x) (&psw[0][0])[i] = 0.f;

    // ---- A. logits: warps split the row; 4 tokens x 8 experts per pass ----
    const int nchunk = d / 8;
    const int per = (nchunk + kWarps - 1) / kWarps;
    const int c_lo = warp * per, c_hi = min(nchunk, c_lo + per);
    for (int t0 = 0; t0 < T; t0 += kTokPass) {
        const int nt = min(kTokPass, T - t0);
        for (int e0 = 0; e0 < E; e0 += 8) {
            float acc[kTokPass][8];
#pragma unroll
            for (int q = 0; q < kTokPass; ++q)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[q][e] = 0.f;
            for (int c = c_lo + lane; c < c_hi; c += 32) {
                float xv[kTokPass][8];
#pragma unroll
                for (int q = 0; q < kTokPass; ++q) {
                    if (q < nt) {
                        bf16x8(*reinterpret_cast<const uint4*>(x + (size_t)(t0 + q) * d + (size_t)c * 8), xv[q]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 8; ++j) xv[q][j] = 0.f;
                    }
                }
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    // row c*8 + j of W_r, experts e0 .. e0+7 (16 contiguous bytes)
                    float wv[8];
                    bf16x8(*reinterpret_cast<const uint4*>(W_r + (size_t)(c * 8 + j) * E + e0), wv);
#pragma unroll
                    for (int q = 0; q < kTokPass; ++q)
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[q][e] = fmaf(xv[q][j], wv[e], acc[q][e]);
                }
            }
#pragma unroll
            for (int q = 0; q < kTokPass; ++q)
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    float v = warp_sum(acc[q][e]);
                    if (lane == 0) part[warp][q][e] = v;
                }
            __syncthreads();
            if (threadIdx.x < kTokPass * 8) {
                const int q = threadIdx.x / 8, e = threadIdx.x % 8;
                if (q < nt) {
                    float v = 0.f;
                    for (int w = 0; w < kWarps; ++w) v += part[w][q][e];
                    z[t0 + q][e0 + e] = v;
                    if (a.logits) a.logits[(size_t)(t0 + q) * E + e0 + e] = v;
                }
            }
            __syncthreads();
        }
    }

    // ---- B. selection: one warp per token; lane holds experts lane, lane+32 ----
    for (int t = warp; t < T; t += kWarps) {
        float zz[2], key[2], ex[2];
        unsigned valid = 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int e = lane + 32 * i;
            zz[i] = e < E ? z[t][e] : -INFINITY;
            if (e < E) valid |= 1u << i;
        }
        float m = warp_max(fmaxf(zz[0], zz[1]));
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            ex[i] = ((valid >> i) & 1u) ? expf(zz[i] - m) : 0.f;
            s += ex[i];
        }
        s = warp_sum(s);
        const float inv_s = 1.f / s;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int e = lane + 32 * i;
            const float p = ex[i] * inv_s;
            const float b = (a.bias_mode != MOE_BIAS_NONE && e < E) ? a.bias[e] : 0.f;
            if (e < E) psw[warp][e] += p;
            key[i] = a.bias_mode == MOE_BIAS_NONE ? zz[i] : a.bias_mode == MOE_BIAS_LOGIT ? zz[i] + b : p + b;
        }
        unsigned taken = 0;
        float zsel[MOE_MAX_K];
        int esel[MOE_MAX_K];
#pragma unroll
        for (int j = 0; j < MOE_MAX_K; ++j) {
            if (j < k) {
                float bk = -INFINITY, bz = 0.f;
                int be = 0x7fffffff;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const bool ok = ((valid >> i) & 1u) && !((taken >> i) & 1u);
                    if (ok && (key[i] > bk || be == 0x7fffffff)) { bk = key[i]; be = lane + 32 * i; bz = zz[i]; }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ok_ = __shfl_xor_sync(0xffffffffu, bk, o);
                    const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                    const float oz = __shfl_xor_sync(0xffffffffu, bz, o);
                    const bool better = (oe != 0x7fffffff) &&
                                        (be == 0x7fffffff || ok_ > bk || (ok_ == bk && oe < be));
                    if (better) { bk = ok_; be = oe; bz = oz; }
                }
                if ((be & 31) == lane) taken |= 1u << (be >> 5);
                zsel[j] = bz;
                esel[j] = be;
            }
        }
        float zm = -INFINITY;
#pragma unroll
        for (int j = 0; j < MOE_MAX_K; ++j) if (j < k) zm = fmaxf(zm, zsel[j]);
        float gs = 0.f, ge[MOE_MAX_K];
#pragma unroll
        for (int j = 0; j < MOE_MAX_K; ++j) if (j < k) { ge[j] = expf(zsel[j] - zm); gs += ge[j]; }
        const float inv_g = 1.f / gs;
        if (lane == 0) {
#pragma unroll
            for (int j = 0; j < MOE_MAX_K; ++j) {
                if (j < k) {
                    a.idx[(size_t)t * k + j] = esel[j];
                    a.gate[(size_t)t * k + j] = ge[j] * inv_g;
                    sidx[t * k + j] = esel[j];
                    atomicAdd(&cnt[esel[j]], 1);   // integer: order does not matter
                }
            }
        }
    }
    __syncthreads();

    // ---- C. counts, capacity, indptr, statistics, tile schedules (warp 0) ----
    if (warp == 0) {
        int c[2], kp[2];
        float fP = 0.f;
        float* P = MOE_STATS_P(a.stats, E);
        float* f = MOE_STATS_F(a.stats, E);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int e = lane + 32 * i;
            c[i] = e < E ? cnt[e] : 0;
            kp[i] = a.capacity < 0 ? c[i] : min(c[i], a.capacity);
            if (e < E) {
                float acc = 0.f;
                for (int w = 0; w < kWarps; ++w) acc += psw[w][e];   // fixed order over warps
                const float Pe = acc / (float)T;
                const float fe = (float)c[i] / ((float)T * (float)k);
                P[e] = Pe;
                f[e] = fe;
                fP += fe * Pe;
                MOE_STATS_COUNTS(a.stats, E)[e] = c[i];
                MOE_STATS_KEPT(a.stats, E)[e] = kp[i];
            }
        }
        const float laux = (float)E * warp_sum(fP);
        // exclusive scan of kept over experts lane, lane+32
        int run = 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            int incl = kp[i];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n_ = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += n_;
            }
            const int e = lane + 32 * i;
            const int ex = run + incl - kp[i];
            if (e < E) {
                indptr_s[e] = ex;
                a.indptr[e] = ex;
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        // tile schedules: one M-block per expert with rows (kept <= 64 < 128)
        int t13[2], t2[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int mt = kp[i] > 0 ? 1 : 0;
            t13[i] = mt * a.nt13;
            t2[i] = mt * a.nt2;
        }
        int run13 = 0, run2 = 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            int i13 = t13[i], i2 = t2[i];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int n13 = __shfl_up_sync(0xffffffffu, i13, o);
                const int n2 = __shfl_up_sync(0xffffffffu, i2, o);
                if (lane >= o) { i13 += n13; i2 += n2; }
            }
            const int e = lane + 32 * i;
            if (e < E) {
                a.tiles13[e] = run13 + i13 - t13[i];
                a.tiles2[e] = run2 + i2 - t2[i];
            }
            run13 += __shfl_sync(0xffffffffu, i13, 31);
            run2 += __shfl_sync(0xffffffffu, i2, 31);
        }
        int maxc = max(c[0], c[1]);
        int drop = (c[0] - kp[0]) + (c[1] - kp[1]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            maxc = max(maxc, __shfl_xor_sync(0xffffffffu, maxc, o));
            drop += __shfl_xor_sync(0xffffffffu, drop, o);
        }
        if (lane == 0) {
            indptr_s[E] = run;
            a.indptr[E] = run;
            a.tiles13[E] = run13;
            a.tiles2[E] = run2;
            a.tiles13[E + 1] = pick_split(run13, a.nkb13, a.sm_count, a.split_max);
            a.tiles2[E + 1] = pick_split(run2, a.nkb2, a.sm_count, a.split_max);
            moe_stats* st = static_cast<moe_stats*>(a.stats);
            st->capacity = a.capacity;
            st->rows = run;
            st->dropped = drop;
            st->max_count = maxc;
            st->l_aux = laux;
            const float mean = (float)T * (float)k / (float)E;
            st->max_over_mean = (float)maxc / mean;
            st->reserved = 0;
        }
    }
    __syncthreads();

    // ---- D. ranks in token order and destinations ----
    for (int i = threadIdx.x; i < T * k; i += blockDim.x) {
        const int t = i / k;
        const int e = sidx[i];
        int rank = 0;
        for (int i2 = 0; i2 < t * k; ++i2) rank += (sidx[i2] == e);
        const int p = (a.capacity < 0 || rank < a.capacity) ? indptr_s[e] + rank : -1;
        spos[i] = p;
        a.pos[i] = p;
        if (p >= 0 && a.row_token != nullptr) a.row_token[p] = t;
    }
    __syncthreads();

    // ---- E. gather: xp[pos] = x[t], 16-byte vectors, coalesced ----
    const int nvec = d / 8;
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    uint4* xp = static_cast<uint4*>(a.xp);
    for (int i = threadIdx.x; i < T * nvec; i += blockDim.x) {
        const int t = i / nvec, v = i % nvec;
        const uint4 val = xv[(size_t)t * nvec + v];
        for (int j = 0; j < k; ++j) {
            const int p = spos[t * k + j];
            if (p >= 0) xp[(size_t)p * nvec + v] = val;
        }
    }
}

}  // namespace

bool small_route_ok(const moe_problem& p) {
    return p.dtype == MOE_DTYPE_BF16 && p.d_ff_shared == 0 && p.T > 0 && (long long)p.T * p.k <= kSmallMaxPairs &&
           p.E <= kSmallMaxE && p.E % 8 == 0 && p.d % 8 == 0;
}

cudaError_t launch_route_small(const SmallRouteArgs& a, cudaStream_t st) {
    route_small_kernel<<<1, kWarps * 32, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace moe
