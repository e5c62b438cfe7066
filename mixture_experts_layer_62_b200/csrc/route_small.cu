// Small-batch router: the whole routing and permutation of a decode-sized
// batch (T*k <= 64 pairs) in two short launches instead of five: partial
// logits by (token, part of the row) blocks, then one kernel for the
// selection, statistics, destinations, tile schedules and the row gather.
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
#include "route_select.cuh"

namespace moe {

namespace {

using small::warp_max;
using small::warp_sum;
__device__ __forceinline__ void bf16x8(const uint4& u, float (&v)[8]) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 f = __bfloat1622float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// ---- kernel 1: partial logits, one block per (token, part of the row) ---------
// Block (t, part) sums x_t . W_r[:, e] over its slice of the row: 4 warps, lane
// l takes chunks l, l + 32, ... of its warp's sub-slice, xor butterfly over
// lanes, warp order over warps. Output: partial[(t * P + part) * E + e].
constexpr int kPartWarps = 4;

__global__ void __launch_bounds__(kPartWarps * 32) route_logits_kernel(SmallRouteArgs a, int P) {
    __shared__ float wsum[kPartWarps][kSmallMaxE];
    pdl_wait();
    pdl_launch();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x, part = blockIdx.y;
    if (a.status_reset != nullptr && t == 0 && part == 0 && threadIdx.x == 0) *a.status_reset = MOE_OK;
    const int d = a.d, E = a.E;
    const __nv_bfloat16* xr = static_cast<const __nv_bfloat16*>(a.x) + (size_t)t * d;
    const __nv_bfloat16* W_r = static_cast<const __nv_bfloat16*>(a.W_r);
    const int nchunk = d / 8;
    const int per_part = (nchunk + P - 1) / P;
    const int p_lo = part * per_part, p_hi = min(nchunk, p_lo + per_part);
    const int per_warp = (p_hi - p_lo + kPartWarps - 1) / kPartWarps;
    const int c_lo = p_lo + warp * per_warp, c_hi = min(p_hi, c_lo + per_warp);
    for (int e0 = 0; e0 < E; e0 += 8) {
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        for (int c = c_lo + lane; c < c_hi; c += 32) {
            float xv[8];
            bf16x8(*reinterpret_cast<const uint4*>(xr + (size_t)c * 8), xv);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float wv[8];   // row c*8 + j of W_r, experts e0 .. e0+7
                bf16x8(*reinterpret_cast<const uint4*>(W_r + (size_t)(c * 8 + j) * E + e0), wv);
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[e] = fmaf(xv[j], wv[e], acc[e]);
            }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float v = warp_sum(acc[e]);
            if (lane == 0) wsum[warp][e0 + e] = v;
        }
    }
    __syncthreads();
    if (threadIdx.x < E) {
        float v = 0.f;
        for (int w = 0; w < kPartWarps; ++w) v += wsum[w][threadIdx.x];
        a.probs[((size_t)t * P + part) * E + threadIdx.x] = v;   // partial logits
    }
}

// ---- kernel 2: logits, selection, statistics, destinations, gather -----------
// Every block sums the partial logits (part order), selects (one warp per
// token: softmax, key, top-k with the lowest index winning ties, gates over
// the selected raw logits), counts, scans and places the <= 64 pairs (rank =
// earlier pairs of the same expert, token order), then gathers its slice of
// the row vectors. Block 0 alone writes logits, idx, gate, pos, row_token,
// indptr, the statistics and the tile schedules with their split factors.
constexpr int kFinWarps = 16;

__global__ void __launch_bounds__(kFinWarps * 32) route_finish_kernel(const __grid_constant__ SmallRouteArgs a, int P) {
    __shared__ float z[kSmallMaxPairs][kSmallMaxE];
    __shared__ float psw[kFinWarps][kSmallMaxE];
    __shared__ int sidx[kSmallMaxPairs];
    __shared__ int spos[kSmallMaxPairs];
    __shared__ int indptr_s[kSmallMaxE + 1];
    __shared__ float bias_s[kSmallMaxE];
    __shared__ float extw[kFinWarps][3];
    __shared__ float zsel_s[kFinWarps][MOE_MAX_K];
    __shared__ int esel_s[kFinWarps][MOE_MAX_K];
    const int T = a.T, E = a.E, k = a.k;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool writer = blockIdx.x == 0;
    // Before the dependency wait: only inputs of the pass (bias, x), never an
    // output of the preceding kernel. The x vectors this block gathers are
    // loaded now and held in registers.
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        bias_s[e] = a.bias_mode != MOE_BIAS_NONE ? a.bias[e] : 0.f;
    for (int i = threadIdx.x; i < kFinWarps * kSmallMaxE; i += blockDim.x) (&psw[0][0])[i] = 0.f;
    const int nvec = a.d / 8;
    const int vper = (nvec + gridDim.x - 1) / gridDim.x;
    const int v_lo = blockIdx.x * vper, v_hi = min(nvec, v_lo + vper);
    const int span = max(0, v_hi - v_lo);
    const uint4* xv = static_cast<const uint4*>(a.x);
    constexpr int kHeld = 4;
    uint4 held[kHeld];
#pragma unroll
    for (int h = 0; h < kHeld; ++h) {
        const int i = threadIdx.x + h * (int)blockDim.x;
        if (i < T * span) held[h] = xv[(size_t)(i / span) * nvec + v_lo + i % span];
    }
    pdl_wait();
    pdl_launch();
    if (writer)   // split-K arrival counters start at zero on every pass
        for (int i = threadIdx.x; i < a.sem_n; i += blockDim.x) a.sem[i] = 0;
    for (int i = threadIdx.x; i < T * E; i += blockDim.x) {
        const int t = i / E, e = i % E;
        const float v = small::sum_partials(a.probs, t, P, E, e);
        z[t][e] = v;
        if (writer) a.logits[i] = v;
    }
    __syncthreads();

    float ex_z = 0.f, ex_h = 0.f, ex_g = 0.f;
    for (int t = warp; t < T; t += kFinWarps) {
        const small::TokenSoftmax ts =
            small::token_softmax(lane < E ? z[t][lane] : 0.f, lane + 32 < E ? z[t][lane + 32] : 0.f, E, lane);
        const float* zz = ts.zz;
        const float* ex = ts.ex;
        const unsigned valid = ts.valid;
        const float m = ts.m, s = ts.s, inv_s = ts.inv_s;
        {   // router statistics of this token (z-loss, entropy, top-1/top-2 gap)
            float pz = 0.f, z1 = -INFINITY, z2 = -INFINITY;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                if ((valid >> i) & 1u) {
                    pz += ex[i] * zz[i];
                    if (zz[i] > z1) { z2 = z1; z1 = zz[i]; } else if (zz[i] > z2) { z2 = zz[i]; }
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
            ex_z += lse * lse;
            ex_h += lse - pz;
            ex_g += (1.f - expf(z2 - m)) * inv_s;
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int e = lane + 32 * i;
            if (e < E) psw[warp][e] += small::token_prob(ts, i);
        }
        // k rounds of a warp arg-max (the lowest index wins ties); the selected
        // logits and experts go to shared memory, lane j then finishes slot j
        small::token_topk(ts, bias_s, a.bias_mode, E, k, lane, zsel_s[warp], esel_s[warp]);
        __syncwarp();
        if (lane < k) {
            // gates: softmax over the k selected raw logits, summed in slot order
            float zm = -INFINITY;
            for (int j = 0; j < k; ++j) zm = fmaxf(zm, zsel_s[warp][j]);
            float gs = 0.f;
            for (int j = 0; j < k; ++j) gs += expf(zsel_s[warp][j] - zm);
            const float inv_g = 1.f / gs;
            const float zj = zsel_s[warp][lane];
            const int ej = esel_s[warp][lane];
            sidx[t * k + lane] = ej;
            if (writer) {
                a.idx[(size_t)t * k + lane] = ej;
                a.gate[(size_t)t * k + lane] =
                    a.gate_mode == MOE_GATE_FULL ? expf(zj - m) * inv_s : expf(zj - zm) * inv_g;
            }
        }
        __syncwarp();
    }
    if (lane == 0) {
        extw[warp][0] = ex_z;
        extw[warp][1] = ex_h;
        extw[warp][2] = ex_g;
    }
    __syncthreads();

    if (warp == 0) {
        // counts, capacity, kept, indptr (experts lane, lane + 32)
        int c[2], kp[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int e = lane + 32 * i;
            int n_ = 0;
            if (e < E)
                for (int q = 0; q < T * k; ++q) n_ += (sidx[q] == e);
            c[i] = n_;
            kp[i] = a.capacity < 0 ? n_ : min(n_, a.capacity);
        }
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
            if (e < E) indptr_s[e] = run + incl - kp[i];
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) indptr_s[E] = run;
        if (writer) {
            float fP = 0.f;
            int t13[2], t2[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int e = lane + 32 * i;
                t13[i] = (kp[i] > 0 ? 1 : 0) * a.nt13;   // kept <= 64 rows: one M-block
                t2[i] = (kp[i] > 0 ? 1 : 0) * a.nt2;
                if (e < E) {
                    float acc = 0.f;
                    for (int w = 0; w < kFinWarps; ++w) acc += psw[w][e];   // fixed order over warps
                    const float Pe = acc / (float)T;
                    const float fe = (float)c[i] / ((float)T * (float)k);
                    MOE_STATS_P(a.stats, E)[e] = Pe;
                    MOE_STATS_F(a.stats, E)[e] = fe;
                    MOE_STATS_COUNTS(a.stats, E)[e] = c[i];
                    MOE_STATS_KEPT(a.stats, E)[e] = kp[i];
                    a.indptr[e] = indptr_s[e];
                    fP += fe * Pe;
                }
            }
            const float laux = (float)E * warp_sum(fP);
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
            // active experts (<= 64 here) index the host-built split table
            const int n_active = __popc(__ballot_sync(0xffffffffu, kp[0] > 0)) +
                                 __popc(__ballot_sync(0xffffffffu, kp[1] > 0));
            int maxc = max(c[0], c[1]);
            int drop = (c[0] - kp[0]) + (c[1] - kp[1]);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                maxc = max(maxc, __shfl_xor_sync(0xffffffffu, maxc, o));
                drop += __shfl_xor_sync(0xffffffffu, drop, o);
            }
            if (lane == 0) {
                a.indptr[E] = run;
                a.tiles13[E] = run13;
                a.tiles2[E] = run2;
                a.tiles13[E + 1] = a.split_on ? a.split.s13[n_active] : 1;
                a.tiles2[E + 1] = a.split_on ? a.split.s2[n_active] : 1;
                moe_stats* st = static_cast<moe_stats*>(a.stats);
                st->capacity = a.capacity;
                st->rows = run;
                st->dropped = drop;
                st->max_count = maxc;
                st->l_aux = laux;
                st->max_over_mean = (float)maxc / ((float)T * (float)k / (float)E);
                float ez = 0.f, eh = 0.f, eg = 0.f;
                for (int w = 0; w < kFinWarps; ++w) {   // fixed order over warps
                    ez += extw[w][0];
                    eh += extw[w][1];
                    eg += extw[w][2];
                }
                st->z_loss = ez / (float)T;
                st->entropy = eh / (float)T;
                st->top_gap = eg / (float)T;
                st->reserved[0] = 0;
                st->reserved[1] = 0;
            }
        }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < T * k; i += blockDim.x) {
        const int t = i / k, e = sidx[i];
        const int rank = small::pair_rank(sidx, i, T, k, a.drop_slot != 0);
        const int p = (a.capacity < 0 || rank < a.capacity) ? indptr_s[e] + rank : -1;
        spos[i] = p;
        if (writer) {
            a.pos[i] = p;
            if (p >= 0 && a.row_token != nullptr) a.row_token[p] = t;
        }
    }
    __syncthreads();
    // gather this block's slice of every token row (the first kHeld vectors
    // of each thread were loaded before the wait)
    if (span <= 0) return;
    uint4* xp = static_cast<uint4*>(a.xp);
    for (int i = threadIdx.x, h = 0; i < T * span; i += blockDim.x, ++h) {
        const int t = i / span, v = v_lo + i % span;
        uint4 val;
        if (h < kHeld) {
#pragma unroll
            for (int hh = 0; hh < kHeld; ++hh)
                if (hh == h) val = held[hh];
        } else {
            val = xv[(size_t)t * nvec + v];
        }
        for (int j = 0; j < k; ++j) {
            const int p = spos[t * k + j];
            if (p >= 0) xp[(size_t)p * nvec + v] = val;
        }
    }
}

}  // namespace

bool small_route_ok(const moe_problem& p) {
    return p.dtype == MOE_DTYPE_BF16 && p.d_ff_shared == 0 && p.pad_rows == 0 && !p.train && p.T > 0 &&
           (long long)p.T * p.k <= kSmallMaxPairs &&
           p.E <= kSmallMaxE && p.E % 8 == 0 && p.d % 8 == 0;
}

int small_route_parts(int d) {
    const int nchunk = d / 8;
    const int P = (nchunk + 127) / 128;   // ~128 chunks (1 per lane of 4 warps) per block
    return P < 1 ? 1 : (P > kSmallMaxParts ? kSmallMaxParts : P);
}

cudaError_t launch_route_small(const SmallRouteArgs& a, cudaStream_t st) {
    const int nchunk = a.d / 8;
    const int P = small_route_parts(a.d);
    cudaError_t e = launch_k(route_logits_kernel, dim3(a.T, P), dim3(kPartWarps * 32), 0, st, a, P);
    if (e != cudaSuccess) return e;
    g_pdl_after_first();
    int blocks = (nchunk + 63) / 64;   // >= 64 vectors of the gather per block
    blocks = blocks < 1 ? 1 : (blocks > 32 ? 32 : blocks);
    return launch_k(route_finish_kernel, dim3(blocks), dim3(kFinWarps * 32), 0, st, a, P);
}

}  // namespace moe
