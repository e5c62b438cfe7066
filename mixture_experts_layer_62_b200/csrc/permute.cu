// Permutation of token rows by expert ("Lecture 21 · LLM: Mixture-of-Experts"
// §3.3: the N x E selection mask flattened expert-major, an exclusive prefix
// sum giving every selected pair its destination row, indptr from the same
// scan; §3.5: capacity C = ceil(k N / E x cf), overflow pairs dropped).
//
// The mask is never materialised. Per chunk of kChunk tokens the router (or
// hist_kernel) counts pairs per expert; one block scans those counts in
// expert-major order (e outer, chunk inner), which is the order of the
// flattened mask; a pair's rank inside its expert is the scan value of its
// chunk plus the number of earlier pairs of the same expert in the chunk.
// No atomics decide any position, so the permutation is deterministic and
// ranks follow token order.
#include "common.cuh"

namespace moe {

constexpr int kScanThreads = 1024;

// Exclusive block-wide scan of one int per thread; returns the block total.
__device__ int block_exclusive_scan(int v, int* warp_tot, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int nw = blockDim.x >> 5;
        int w = lane < nw ? warp_tot[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int n = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += n;
        }
        if (lane < nw) warp_tot[lane] = wi - w;   // exclusive warp offsets
        if (lane == 31) warp_tot[32] = wi;
    }
    __syncthreads();
    int excl = warp_tot[warp] + incl - v;
    total = warp_tot[32];
    __syncthreads();
    return excl;
}

// Tile schedule of a grouped GEMM: tiles[g] = sum_{g' < g} mtiles(g') * ntiles(g').
__device__ void build_schedule(const int* rows, int G, int E, int tile_m, int nt, int nt_shared,
                               int32_t* tiles, int* warp_tot) {
    int carry = 0;
    for (int base = 0; base < G; base += blockDim.x) {
        int g = base + threadIdx.x;
        int v = 0;
        if (g < G) v = ((rows[g] + tile_m - 1) / tile_m) * (g < E ? nt : nt_shared);
        int tot;
        int ex = block_exclusive_scan(v, warp_tot, tot);
        if (g < G) tiles[g] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) tiles[G] = carry;
}

// CTAs of the small class (the first S of the grid) for one GEMM with the
// grid split: the S minimising the later of the two classes' end times,
// with a large tile's K block of MMAs taken as kLargeKbSec and the small
// tiles as weight streams of kSmallCtaBw per CTA, kSmallHbmShare at most in
// all (the large class keeps the rest of the memory bandwidth). Both rates
// are measured on B200: a large tile's K block in the Mixtral-shaped GEMM
// 1/3 (1.44 ms for 3293 K blocks per CTA), and the small class's stream per
// CTA from a sweep of S on the DeepSeek-shaped layer (about 55 GB/s: four
// stages in flight per CTA bound it).
constexpr double kLargeKbSec = 0.44e-6;
constexpr double kSmallCtaBw = 55e9;
constexpr double kSmallHbmShare = 4.5e12;

__device__ int choose_small_ctas(double large_kb, double small_bytes, int grid) {
    if (small_bytes <= 0.0) return 0;
    if (large_kb <= 0.0) return grid;
    int best = 1;
    double best_t = 1e30;
    for (int S = 1; S < grid; ++S) {
        const double tl = large_kb * kLargeKbSec / (double)(grid - S);
        const double bw = fmin((double)S * kSmallCtaBw, kSmallHbmShare);
        const double ts = small_bytes / bw;
        const double t = fmax(tl, ts);
        if (t < best_t) { best_t = t; best = S; }
    }
    return best;
}

// The schedules of GEMM 1/3 and GEMM 2 from the rows per group (rows[E] =
// T for the shared expert): one class of tiles, or with gs.on the large
// class (groups of more than kSmallRows rows, the shared expert), the small
// class and S. Block-wide; ends synchronised.
__device__ void build_gemm_schedules(int* rows, int G, int E, int tile_m, int nt13, int nt13s, int nt2, int nt2s,
                                     int32_t* tiles13, int32_t* tiles2, const GridSplit& gs, int* warp_tot,
                                     int* srows) {
    if (!gs.on) {
        build_schedule(rows, G, E, tile_m, nt13, nt13s, tiles13, warp_tot);
        __syncthreads();
        build_schedule(rows, G, E, tile_m, nt2, nt2s, tiles2, warp_tot);
        __syncthreads();
        if (threadIdx.x == 0) {
            tiles13[G + 2] = 0;
            tiles2[G + 2] = 0;
        }
        return;
    }
    // small class: one (operand-swapped) M block per group of 1..kSmallRows rows
    for (int g = threadIdx.x; g < G; g += blockDim.x) {
        const bool small = g < E && rows[g] > 0 && rows[g] <= kSmallRows;
        srows[g] = small ? rows[g] : 0;
    }
    __syncthreads();
    for (int g = threadIdx.x; g < G; g += blockDim.x)
        if (srows[g] > 0) rows[g] = 0;   // the large class skips them
    __syncthreads();
    build_schedule(rows, G, E, tile_m, nt13, nt13s, tiles13, warp_tot);
    __syncthreads();
    build_schedule(rows, G, E, tile_m, nt2, nt2s, tiles2, warp_tot);
    __syncthreads();
    build_schedule(srows, G, E, kSmallRows, nt13, nt13s, tiles13 + G + 3, warp_tot);
    __syncthreads();
    build_schedule(srows, G, E, kSmallRows, nt2, nt2s, tiles2 + G + 3, warp_tot);
    __syncthreads();
    if (threadIdx.x == 0) {
        const int kb13 = (gs.k13 + 63) / 64, kb2 = (gs.k2 + 63) / 64;
        const int kb13s = (gs.k13s + 63) / 64, kb2s = (gs.k2s + 63) / 64;
        double l13 = 0, l2 = 0, s13 = 0, s2 = 0;
        for (int g = 0; g < G; ++g) {
            if (rows[g] > 0) {
                const double mt = (double)((rows[g] + tile_m - 1) / tile_m);
                l13 += mt * (g < E ? (double)nt13 * kb13 : (double)nt13s * kb13s);
                l2 += mt * (g < E ? (double)nt2 * kb2 : (double)nt2s * kb2s);
            }
            if (srows[g] > 0) {
                // per K block: the 256 weight rows (32 KB) and the group's 32-row boxes of A
                const double xb = (double)((srows[g] + 31) / 32) * 4096.0;
                s13 += (double)nt13 * kb13 * (32768.0 + xb);
                s2 += (double)nt2 * kb2 * (32768.0 + xb);
            }
        }
        const int f = gs.force_ctas > 0 ? min(gs.force_ctas, gs.grid) : -1;
        tiles13[G + 2] = gs.interleave ? 0 : f > 0 ? (s13 > 0 ? f : 0) : choose_small_ctas(l13, s13, gs.grid);
        tiles2[G + 2] = gs.interleave ? 0 : f > 0 ? (s2 > 0 ? f : 0) : choose_small_ctas(l2, s2, gs.grid);
    }
    __syncthreads();
}

__global__ void __launch_bounds__(kScanThreads) scan_kernel(const __grid_constant__ ScanArgs a, int NB) {
    __shared__ int warp_tot[33];
    __shared__ int start[MOE_MAX_E + 1];
    __shared__ int kept_s[MOE_MAX_E + 1];
    __shared__ float fP[MOE_MAX_E];
    pdl_wait();
    pdl_launch();
    const int E = a.E;

    // 1. per expert row of chunk counts (expert-major order, chunk inner):
    //    exclusive prefix inside the row -> blockoff, row total -> start[e].
    //    One warp per row, 32 consecutive entries per step (coalesced); the
    //    loads of 8 steps are issued before their scans, so a row of a few
    //    hundred chunks costs one or two memory round trips, not one a step.
    {
        const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
        const int len = a.kk * NB;   // (slot, chunk) entries of one expert
        constexpr int U = 8;
        for (int e = warp; e < E; e += nw) {
            const int32_t* row = a.blockcnt + (size_t)e * len;
            int32_t* orow = a.blockoff + (size_t)e * len;
            int carry = 0;
            for (int b0 = 0; b0 < len; b0 += 32 * U) {
                int v[U];
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int b = b0 + 32 * u + lane;
                    v[u] = b < len ? row[b] : 0;
                }
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int b = b0 + 32 * u + lane;
                    int incl = v[u];
#pragma unroll
                    for (int o = 1; o < 32; o <<= 1) {
                        int n_ = __shfl_up_sync(0xffffffffu, incl, o);
                        if (lane >= o) incl += n_;
                    }
                    if (b < len) orow[b] = carry + incl - v[u];
                    carry += __shfl_sync(0xffffffffu, incl, 31);
                }
            }
            if (lane == 0) start[e] = carry;   // c_e (converted to a prefix below)
        }
    }
    __syncthreads();
    // 2. per-expert counts -> exclusive prefix over experts in start[]
    {
        int c_e = threadIdx.x < E ? start[threadIdx.x] : 0;
        int tot;
        int ex = block_exclusive_scan(c_e, warp_tot, tot);
        if (threadIdx.x < E) start[threadIdx.x] = ex;
        if (threadIdx.x == 0) start[E] = tot;
    }
    __syncthreads();

    // 3. counts, capacity, kept and indptr over kept rows
    int c = 0, kp = 0;
    const int e = threadIdx.x;
    if (e < E) {
        c = start[e + 1] - start[e];
        kp = a.capacity < 0 ? c : min(c, a.capacity);
    }
    // rows an expert occupies: its kept pairs, rounded up to a multiple of
    // the block size in the padded (MegaBlocks) layout
    const int kr = a.pad > 0 ? (kp + a.pad - 1) / a.pad * a.pad : kp;
    int tot_rows, tot_kept;
    int ex = block_exclusive_scan(e < E ? kr : 0, warp_tot, tot_rows);
    block_exclusive_scan(e < E ? kp : 0, warp_tot, tot_kept);
    if (e < E) {
        a.indptr[e] = ex;
        kept_s[e] = kp;
    }
    if (threadIdx.x == 0) a.indptr[E] = tot_rows;

    moe_stats* st = (moe_stats*)a.stats;
    int32_t* counts = MOE_STATS_COUNTS(a.stats, E);
    int32_t* kept = MOE_STATS_KEPT(a.stats, E);
    float* P = MOE_STATS_P(a.stats, E);
    float* f = MOE_STATS_F(a.stats, E);
    if (e < E) {
        counts[e] = c;
        kept[e] = kp;
    }

    // 4. P_e = mean router probability over the per-chunk sums [NB][E]: a
    //    warp takes 32 consecutive experts (coalesced rows) and one of
    //    `segs` contiguous ranges of chunks, summed in chunk order with 8
    //    loads in flight; the ranges are then added in range order. Fixed
    //    order throughout.
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __shared__ float psum_s[kScanThreads];
    if (a.blockpsum != nullptr) {
        const int groups = (E + 31) / 32;
        const int segs = max(1, (kScanThreads / 32) / groups);
        if (warp < groups * segs) {
            const int g = warp % groups, sg = warp / groups;
            const int ee = g * 32 + lane;
            const int b_lo = (int)((long long)sg * NB / segs), b_hi = (int)((long long)(sg + 1) * NB / segs);
            float acc = 0.f;
            if (ee < E) {
                int b = b_lo;
                for (; b + 8 <= b_hi; b += 8) {
                    float v[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) v[u] = a.blockpsum[(size_t)(b + u) * E + ee];
#pragma unroll
                    for (int u = 0; u < 8; ++u) acc += v[u];
                }
                for (; b < b_hi; ++b) acc += a.blockpsum[(size_t)b * E + ee];
                psum_s[sg * E + ee] = acc;
            }
        }
        __syncthreads();
        const int ee = threadIdx.x;
        if (ee < E) {
            float acc = 0.f;
            for (int sg = 0; sg < segs; ++sg) acc += psum_s[sg * E + ee];
            float Pe = a.T > 0 ? acc / (float)a.T : 0.f;
            float fe = a.T > 0 ? (float)(start[ee + 1] - start[ee]) / ((float)a.T * (float)a.k) : 0.f;
            P[ee] = Pe;
            f[ee] = fe;
            fP[ee] = fe * Pe;
        }
    }
    // router statistics: per-chunk sums of (z-loss, entropy, gap), one warp
    // each, lane-strided then butterfly (fixed order)
    __shared__ float extra_s[3];
    if (a.blockextra != nullptr && warp < 3) {
        float acc = 0.f;
        for (int b0 = lane; b0 < NB; b0 += 32 * 4) {   // 4 loads in flight, summed in chunk order
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int b = b0 + 32 * u;
                v[u] = b < NB ? a.blockextra[(size_t)b * 3 + warp] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) acc += v[u];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) extra_s[warp] = a.T > 0 ? acc / (float)a.T : 0.f;
    }
    __syncthreads();
    // 5. header: fixed-order sums in one thread
    if (threadIdx.x == 0) {
        int dropped = 0, maxc = 0;
        for (int ee = 0; ee < E; ++ee) {
            int ce = start[ee + 1] - start[ee];
            dropped += ce - kept_s[ee];
            maxc = max(maxc, ce);
        }
        st->status = MOE_OK;
        st->capacity = a.capacity;
        st->rows = tot_kept;
        st->dropped = dropped;
        st->max_count = maxc;
        float mean = a.T > 0 ? (float)a.T * (float)a.k / (float)E : 0.f;
        st->max_over_mean = mean > 0.f ? (float)maxc / mean : 0.f;
        if (a.blockpsum != nullptr) {
            float s = 0.f;
            for (int ee = 0; ee < E; ++ee) s += fP[ee];
            st->l_aux = (float)E * s;
        }
        if (a.blockextra != nullptr) {
            st->z_loss = extra_s[0];
            st->entropy = extra_s[1];
            st->top_gap = extra_s[2];
        }
        st->reserved[0] = 0;
        st->reserved[1] = 0;
    }
    // 6. tile schedules of the grouped GEMMs
    if (a.tiles13 != nullptr) {
        __shared__ int rows[MOE_MAX_E + 1];
        if (threadIdx.x < E) rows[threadIdx.x] = a.pad > 0 ? (kept_s[threadIdx.x] + a.pad - 1) / a.pad * a.pad
                                                           : kept_s[threadIdx.x];
        if (threadIdx.x == 0) rows[E] = a.T;
        __syncthreads();
        const int G = E + a.has_shared;
        __shared__ int srows[MOE_MAX_E + 1];
        build_gemm_schedules(rows, G, E, a.tile_m, a.ntiles13, a.ntiles13_shared, a.ntiles2, a.ntiles2_shared,
                             a.tiles13, a.tiles2, a.gsplit, warp_tot, srows);
        // split factors: with split-K on, every active expert is one M-block,
        // so the host-built table indexed by the active-expert count applies
        int n_active;
        block_exclusive_scan(threadIdx.x < E && kept_s[threadIdx.x] > 0 ? 1 : 0, warp_tot, n_active);
        if (threadIdx.x == 0) {
            const int n = n_active < kSplitMaxRows ? n_active : kSplitMaxRows;
            a.tiles13[G + 1] = a.split_on ? a.split.s13[n] : 1;
            a.tiles2[G + 1] = a.split_on ? a.split.s2[n] : 1;
        }
        // split-K arrival counters start at zero on every pass
        for (int i = threadIdx.x; i < a.sem_n; i += blockDim.x) a.sem[i] = 0;
    }
}

cudaError_t launch_scan(const ScanArgs& a, cudaStream_t st) {
    int NB = ceil_div(a.T, kChunk);
    return launch_k(scan_kernel, dim3(1), dim3(kScanThreads), 0, st, a, NB);
}

// Tile schedule from a given indptr (the standalone expert stages), with the
// same split factors and counter reset as the scan of the forward pass.
__global__ void __launch_bounds__(kScanThreads)
schedule_kernel(const int32_t* __restrict__ indptr, int E, int T, int has_shared, int tile_m,
                int nt13, int nt2, int nt13s, int nt2s, int32_t* tiles13, int32_t* tiles2,
                const __grid_constant__ ScheduleSplit sp) {
    __shared__ int warp_tot[33];
    __shared__ int rows[MOE_MAX_E + 1];
    pdl_wait();
    pdl_launch();
    for (int g = threadIdx.x; g < E; g += blockDim.x) rows[g] = indptr[g + 1] - indptr[g];
    if (threadIdx.x == 0) rows[E] = T;
    __syncthreads();
    if (kDebugChecks) {
        // the given offsets must start at 0 or above, never decrease and end
        // within the permuted rows; otherwise no tile is scheduled
        __shared__ int bad;
        if (threadIdx.x == 0) bad = 0;
        __syncthreads();
        for (int g = threadIdx.x; g < E; g += blockDim.x)
            if (indptr[g] < 0 || indptr[g + 1] < indptr[g] || indptr[g + 1] > sp.rows_max) bad = 1;
        __syncthreads();
        if (bad) {
            for (int g = threadIdx.x; g <= E; g += blockDim.x) rows[g] = 0;
            if (threadIdx.x == 0) debug_record_bounds(sp.status);
        }
        __syncthreads();
    }
    const int G = E + has_shared;
    int n_active;
    block_exclusive_scan(threadIdx.x < E && rows[threadIdx.x] > 0 ? 1 : 0, warp_tot, n_active);
    __shared__ int srows[MOE_MAX_E + 1];
    build_gemm_schedules(rows, G, E, tile_m, nt13, nt13s, nt2, nt2s, tiles13, tiles2, sp.gsplit, warp_tot, srows);
    if (threadIdx.x == 0) {
        const int n = n_active < kSplitMaxRows ? n_active : kSplitMaxRows;
        tiles13[G + 1] = sp.split_on ? sp.split.s13[n] : 1;
        tiles2[G + 1] = sp.split_on ? sp.split.s2[n] : 1;
    }
    for (int i = threadIdx.x; i < sp.sem_n; i += blockDim.x) sp.sem[i] = 0;
}

cudaError_t launch_schedule(const int32_t* indptr, int E, int T, int has_shared, int tile_m,
                            int ntiles13, int ntiles2, int ntiles13_shared, int ntiles2_shared,
                            int32_t* tiles13, int32_t* tiles2, const ScheduleSplit& sp, cudaStream_t st) {
    return launch_k(schedule_kernel, dim3(1), dim3(kScanThreads), 0, st, indptr, E, T, has_shared, tile_m, ntiles13,
                    ntiles2, ntiles13_shared, ntiles2_shared, tiles13, tiles2, sp);
}

// Ranks, destinations and the row gather. Block (chunk, column group): every
// block of a chunk derives the chunk's destinations (a few hundred integer
// compares), the column-group-0 block writes pos and row_token, and each
// block gathers its slice of the row vectors.
// Gather: xp[pos[t, j]] = x[t] for every kept pair, 16-byte vectors; each
// source vector is read once and written to all of the token's kept rows.
__global__ void __launch_bounds__(256)
permute_gather_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ idx,
                      const int32_t* __restrict__ blockoff, const int32_t* __restrict__ indptr,
                      int Tn, int nvec, int E, int k, int kk, int capacity,
                      int32_t* __restrict__ pos, int32_t* __restrict__ row_token,
                      uint4* __restrict__ xp) {
    __shared__ int sidx[kChunk][MOE_MAX_K];
    __shared__ int spos[kChunk][MOE_MAX_K];
    pdl_wait();
    pdl_launch();
    const int chunk = blockIdx.x, NB = gridDim.x;
    const bool writer = blockIdx.y == 0;
    const int vper = (nvec + gridDim.y - 1) / gridDim.y;
    const int v_lo = blockIdx.y * vper, v_hi = min(nvec, v_lo + vper);
    const int t0 = chunk * kChunk;
    const int ntok = min(kChunk, Tn - t0);
    for (int i = threadIdx.x; i < ntok * k; i += blockDim.x)
        sidx[i / k][i % k] = idx[(size_t)t0 * k + i];
    __syncthreads();
    for (int i = threadIdx.x; i < ntok * k; i += blockDim.x) {
        const int q = i / k, j = i % k;
        const int e = sidx[q][j];
        if (e < 0 || e >= E) {   // not an expert: the pair takes no row
            spos[q][j] = -1;
            if (writer) pos[(size_t)(t0 + q) * k + j] = -1;
            continue;
        }
        // pairs of this expert earlier in the chunk: any slot of an earlier
        // token (token order), or the same slot of an earlier token (slot
        // priority, where the chunk's base already counts earlier slots)
        int before = 0;
        if (kk > 1) {
            for (int q2 = 0; q2 < q; ++q2) before += (sidx[q2][j] == e);
        } else {
            for (int q2 = 0; q2 < q; ++q2)
                for (int j2 = 0; j2 < k; ++j2) before += (sidx[q2][j2] == e);
        }
        const int rank = blockoff[((size_t)e * kk + (kk > 1 ? j : 0)) * NB + chunk] + before;
        int p = -1;
        if (capacity < 0 || rank < capacity) p = indptr[e] + rank;
        spos[q][j] = p;
        if (writer) {
            pos[(size_t)(t0 + q) * k + j] = p;
            if (p >= 0 && row_token != nullptr) row_token[p] = t0 + q;
        }
    }
    __syncthreads();
    if (xp == nullptr) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int q = warp; q < ntok; q += blockDim.x >> 5) {
        const uint4* src = x + (size_t)(t0 + q) * nvec;
        int dst[MOE_MAX_K];
        int nd = 0;
        for (int j = 0; j < k; ++j)
            if (spos[q][j] >= 0) dst[nd++] = spos[q][j];
        if (nd == 0) continue;
        // four vectors of the row in flight per lane before any is written
        for (int v0 = v_lo + lane; v0 < v_hi; v0 += 32 * 4) {
            uint4 val[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (v0 + 32 * u < v_hi) val[u] = src[v0 + 32 * u];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                if (v0 + 32 * u < v_hi)
                    for (int j = 0; j < nd; ++j) xp[(size_t)dst[j] * nvec + v0 + 32 * u] = val[u];
            }
        }
    }
}

cudaError_t launch_permute_gather(int dtype, const void* x, const int32_t* idx,
                                  const int32_t* blockoff, const int32_t* indptr,
                                  int T, int d, int E, int k, int kk, int capacity,
                                  int32_t* pos, int32_t* row_token, void* xp, cudaStream_t st) {
    int NB = ceil_div(T, kChunk);
    if (NB == 0) return cudaSuccess;
    int nvec = (int)((size_t)d * elem_bytes(dtype) / 16);
    // column groups so that small batches still cover the GPU (~4 blocks per SM)
    int sms = device_sm_count();
    if (sms <= 0) sms = 148;
    int groups = xp == nullptr ? 1 : ceil_div(4 * sms, NB);
    groups = max(1, min(groups, ceil_div(nvec, 32)));
    dim3 grid(NB, groups);
    return launch_k(permute_gather_kernel, grid, dim3(256), 0, st, (const uint4*)x, idx, blockoff, indptr, T, nvec,
                    E, k, kk, capacity, pos, row_token, (uint4*)xp);
}

// Statistics for T == 0 (nothing routed).
// Padding rows of the padded layout: one block per (expert, slice of the
// row's 16-byte vectors); the expert's last pad-1 rows at most.
__global__ void __launch_bounds__(256)
pad_fill_kernel(const int32_t* __restrict__ indptr, const void* __restrict__ stats, int E, int nvec,
                uint4* __restrict__ xp, int32_t* __restrict__ row_token) {
    pdl_wait();
    pdl_launch();
    const int e = blockIdx.x;
    const int r0 = indptr[e] + MOE_STATS_KEPT(stats, E)[e], r1 = indptr[e + 1];
    const int n = xp != nullptr ? (r1 - r0) * nvec : 0;
    for (int i = blockIdx.y * blockDim.x + threadIdx.x; i < n; i += gridDim.y * blockDim.x)
        xp[(size_t)(r0 + i / nvec) * nvec + i % nvec] = make_uint4(0u, 0u, 0u, 0u);
    if (blockIdx.y == 0 && row_token != nullptr)
        for (int r = r0 + (int)threadIdx.x; r < r1; r += blockDim.x) row_token[r] = -1;
}

cudaError_t launch_pad_fill(int dtype, const int32_t* indptr, const void* stats, int E, int d, void* xp,
                            int32_t* row_token, int pad, cudaStream_t st) {
    const int nvec = (int)((size_t)d * elem_bytes(dtype) / 16);
    // at most pad - 1 rows per expert
    const int per_expert = (pad - 1) * nvec;
    int gy = (per_expert + 256 * 4 - 1) / (256 * 4);
    gy = gy < 1 ? 1 : gy;
    return launch_k(pad_fill_kernel, dim3(E, gy), dim3(256), 0, st, indptr, stats, E, nvec,
                    static_cast<uint4*>(xp), row_token);
}

__global__ void zero_stats_kernel(void* stats, int E, int capacity) {
    pdl_wait();
    pdl_launch();
    moe_stats* st = (moe_stats*)stats;
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        MOE_STATS_COUNTS(stats, E)[e] = 0;
        MOE_STATS_KEPT(stats, E)[e] = 0;
        MOE_STATS_P(stats, E)[e] = 0.f;
        MOE_STATS_F(stats, E)[e] = 0.f;
    }
    if (threadIdx.x == 0) {
        st->status = MOE_OK; st->capacity = capacity; st->rows = 0; st->dropped = 0;
        st->max_count = 0; st->l_aux = 0.f; st->max_over_mean = 0.f;
        st->z_loss = 0.f; st->entropy = 0.f; st->top_gap = 0.f;
        st->reserved[0] = 0; st->reserved[1] = 0;
    }
}

cudaError_t launch_zero_stats(void* stats, int E, int capacity, cudaStream_t st) {
    return launch_k(zero_stats_kernel, dim3(1), dim3(256), 0, st, stats, E, capacity);
}

}  // namespace moe
