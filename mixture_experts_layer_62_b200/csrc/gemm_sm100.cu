// bf16 grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Z = GroupGemm(data, indptr, weights) ("Lecture 21 · LLM: Mixture-of-Experts"
// §3.3): group e multiplies the rows [indptr[e], indptr[e+1]) of the permuted
// activations by expert e's weight matrix; one kernel runs every group
// (§3.7: one kernel for all experts matters most when experts are small).
// Modes:
//   SWIGLU  D tile = [Xp W1_e^T | Xp W3_e^T] for 128 output columns; the
//           epilogue writes H = SiLU(a) * b in bf16 ("Week 2 Day 2" §2.1).
//   PLAIN   D tile = Xp W_e^T for 256 output columns, written as bf16.
//   F32OUT  as PLAIN, written as fp32 (router logits).
//
// Design:
//  * persistent grid (one CTA per SM), static tile list: tile ids are laid
//    out group by group, and inside a group the 128-row M blocks vary
//    fastest, so CTAs that run at the same time share one weight tile (read
//    from HBM once, the others hit L2) and a group's activation rows stay in
//    L2 across its N blocks; a group whose rows would not fit in L2 is cut
//    into bands of M blocks (about 32 MB of rows each) that run one after
//    the other, each over all N blocks;
//  * warp 0: one thread issues TMA loads (A 128x64, B 2 x 128x64, 128-byte
//    swizzle) into a 4-stage ring guarded by full/empty mbarriers;
//  * warp 1: one thread issues tcgen05.mma (M=128, N=256, K=16, bf16 in,
//    fp32 accumulate) into one of two TMEM accumulators (2 x 256 columns)
//    and commits stage releases and accumulator completion to mbarriers;
//  * warps 2-5: epilogue, tcgen05.ld of their 32 TMEM lanes, row masking of
//    the ragged tail of a group, conversion and 16-byte stores; the next
//    tile's MMAs run into the other accumulator meanwhile.
//  * every mbarrier wait is bounded by a wall-clock limit; on expiry the CTA
//    records MOE_ERR_TIMEOUT, drains its in-flight TMA and MMA work, frees
//    TMEM and returns.
// No cluster multicast anywhere: every CTA fetches its own tiles.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "tc_common.cuh"

namespace moe {

namespace {

using namespace tc;

constexpr int BM = 128;
constexpr int BK = 64;                       // 64 bf16 = 128 bytes = one swizzle row
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;         // 16 KB
constexpr int B_HALF_BYTES = 128 * BK * 2;   // 16 KB
constexpr int B_BYTES = 2 * B_HALF_BYTES;    // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int NUM_THREADS = 192;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
#ifndef MOE_RASTER_BYTES
#define MOE_RASTER_BYTES (32ll << 20)   // activation rows of one band of M blocks (0: no bands)
#endif

struct KParams {
    const int32_t* indptr;
    const int32_t* tiles;
    int static_rows;
    int E, has_shared, T;
    int b_rows[2];
    int N[2], K[2];
    void* out[2];
    int32_t* status;
    long long timeout_ns;      // limit of every wait of the work itself
    long long drain_ns;        // limit of the drain after a wait gave up
    float* partial;            // split-K partial rows, or null
    long long partial_stride;  // elements between splits
    int partial_ld;            // elements per partial row
    int32_t* sem;              // split-K arrival counters [tile][kSemPerTile]
    __nv_bfloat16* ab_out;     // SWIGLU: raw gate/up accumulators of routed rows, or null
    __nv_bfloat16* ab_out_s;   // SWIGLU: the same for the shared expert's rows, or null
    int b_before_wait;         // weight tiles of the first stages may load before the dependency wait
    int nt_blk[2];             // N blocks of a group (routed, shared)
    int band_m[2];             // M blocks per band (0: the whole group is one band)
    int split_grid;            // the schedule carries the small/large grid split
    int out_rows[2];           // rows of the output buffers (debug-build bounds checks)
    int interleave;            // with split_grid: both classes in one interleaved order
};

struct Tile {
    int kind, g, rows, row0, m_blk, n_blk, num_kb;
};

__device__ __forceinline__ int total_tiles(const KParams& p, int cols_per_tile) {
    if (p.indptr == nullptr)
        return ((p.static_rows + BM - 1) / BM) * ((p.N[0] + cols_per_tile - 1) / cols_per_tile);
    return p.tiles[p.E + p.has_shared];
}

template <int TM>
__device__ __forceinline__ Tile decode_tile_m(const KParams& p, int tile) {
    Tile t;
    if (p.indptr == nullptr) {
        t.kind = 0; t.g = 0; t.rows = p.static_rows; t.row0 = 0;
    } else {
        int lo = 0, hi = p.E + p.has_shared;   // tiles[lo] <= tile < tiles[hi]
        while (hi - lo > 1) {
            int mid = (lo + hi) >> 1;
            if (p.tiles[mid] <= tile) lo = mid; else hi = mid;
        }
        t.g = lo;
        t.kind = lo >= p.E ? 1 : 0;
        t.rows = t.kind ? p.T : p.indptr[lo + 1] - p.indptr[lo];
        t.row0 = t.kind ? 0 : p.indptr[lo];
        tile -= p.tiles[lo];
    }
    const int mt = (t.rows + TM - 1) / TM;
    // bands of band_m M blocks, each over all N blocks, M fastest inside a band
    int h = mt, m0 = 0;
    const int bm = p.band_m[t.kind];
    if (bm > 0 && bm < mt) {
        const int per_band = bm * p.nt_blk[t.kind];
        const int band = tile / per_band;
        tile -= band * per_band;
        m0 = band * bm;
        h = min(bm, mt - m0);
    }
    t.n_blk = tile / h;
    t.m_blk = m0 + tile % h;
    t.num_kb = (p.K[t.kind] + BK - 1) / BK;
    return t;
}
__device__ __forceinline__ Tile decode_tile(const KParams& p, int tile) { return decode_tile_m<BM>(p, tile); }

// The units a CTA runs: first, first + step, ... below count. With the grid
// split, CTAs [0, S) run the small class (operand-swapped tiles of the
// groups of at most kSmallRows rows) and the others the large class.
struct Units {
    int first, step, count;
    bool small;
};
__device__ __forceinline__ Units cta_units(const KParams& p, int total, int nsplit) {
    Units r;
    if (p.split_grid && p.interleave) {
        const int G = p.E + p.has_shared;
        r.first = blockIdx.x; r.step = gridDim.x; r.count = total + p.tiles[2 * G + 3]; r.small = false;
        return r;
    }
    if (p.split_grid) {
        const int G = p.E + p.has_shared;
        const int S = p.tiles[G + 2];
        if (static_cast<int>(blockIdx.x) < S) {
            r.first = blockIdx.x; r.step = S; r.count = p.tiles[2 * G + 3]; r.small = true;
        } else {
            r.first = blockIdx.x - S; r.step = gridDim.x - S; r.count = total; r.small = false;
        }
        return r;
    }
    r.first = blockIdx.x; r.step = gridDim.x; r.count = total * nsplit; r.small = false;
    return r;
}
// Tile u of the small class: one M block of a routed group of 1..128 rows.
__device__ __forceinline__ Tile decode_small_tile(const KParams& p, int u) {
    const int G = p.E + p.has_shared;
    const int32_t* cum = p.tiles + G + 3;
    int lo = 0, hi = G;   // cum[lo] <= u < cum[hi]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cum[mid] <= u) lo = mid; else hi = mid;
    }
    Tile t;
    t.g = lo;
    t.kind = 0;
    t.row0 = p.indptr[lo];
    t.rows = p.indptr[lo + 1] - t.row0;
    t.m_blk = 0;
    t.n_blk = u - cum[lo];
    t.num_kb = (p.K[0] + BK - 1) / BK;
    return t;
}
__device__ __forceinline__ int small_boxes(const Tile& t) { return (t.rows + 31) / 32; }   // 32-row A boxes

// Unit u of the interleaved two-class order: the S tiles of the small class
// (groups of at most 128 rows, run as ordinary tiles) are spread evenly
// through the L tiles of the large class. Position u holds small tile
// floor(u S / (L + S)) when floor((u + 1) S / (L + S)) exceeds it, else large
// tile u - floor(u S / (L + S)) (the large tiles keep their order, so the
// CTAs that share a weight tile still run together).
__device__ __forceinline__ Tile decode_mixed(const KParams& p, int u, bool& small_class) {
    const int G = p.E + p.has_shared;
    const long long L = p.tiles[G], S = p.tiles[2 * G + 3], N = L + S;
    const long long a = (long long)u * S / N, b = (long long)(u + 1) * S / N;
    small_class = b > a;
    return small_class ? decode_small_tile(p, static_cast<int>(a)) : decode_tile(p, u - static_cast<int>(a));
}

struct SharedCtl {
    uint64_t full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
    uint32_t tmem_base;
    int abort_flag;
};

// Wait for phase `parity` of `bar`; false if the CTA aborted or the limit ran out.
__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, SharedCtl* ctl,
                                             const KParams& p) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*reinterpret_cast<volatile int*>(&ctl->abort_flag)) return false;
        if (global_timer_ns() - t0 > static_cast<uint64_t>(p.timeout_ns)) {
            *reinterpret_cast<volatile int*>(&ctl->abort_flag) = 1;
            atomicExch(p.status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
}
// Drain wait used on the abort path: ignores the abort flag and has a limit
// of its own, long, so that a short wait limit never cuts a drain short.
__device__ __forceinline__ void wait_drain(uint64_t* bar, uint32_t parity, const KParams& p) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > static_cast<uint64_t>(p.drain_ns)) {
            atomicExch(p.status, MOE_ERR_TIMEOUT);
            return;
        }
    }
}

__device__ __forceinline__ float silu(float a) { return a / (1.f + __expf(-a)); }

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// TMA coordinates of one unit's tiles: A rows of the group, and the two
// 128-row halves of the B tile (W1 and W3 rows of the same output columns in
// SWIGLU mode, 256 consecutive rows of one matrix otherwise).
struct TileLoads {
    const CUtensorMap *ma, *mlo, *mhi;
    int arow, brow0, brow1;
};
template <int MODE>
__device__ __forceinline__ TileLoads tile_loads(const KParams& p, const Tile& t, const CUtensorMap* tmA0,
                                                const CUtensorMap* tmA1, const CUtensorMap* tmB00,
                                                const CUtensorMap* tmB01, const CUtensorMap* tmB10,
                                                const CUtensorMap* tmB11) {
    TileLoads l;
    l.ma = t.kind ? tmA1 : tmA0;
    const CUtensorMap* mb0 = t.kind ? tmB10 : tmB00;
    const CUtensorMap* mb1 = t.kind ? tmB11 : tmB01;
    l.arow = t.row0 + t.m_blk * BM;
    const int eoff = t.kind ? 0 : t.g * p.b_rows[0];
    if (MODE == TC_SWIGLU) {
        l.brow0 = eoff + t.n_blk * 128; l.brow1 = l.brow0; l.mlo = mb0; l.mhi = mb1;
    } else {
        l.brow0 = eoff + t.n_blk * 256; l.brow1 = l.brow0 + 128; l.mlo = mb0; l.mhi = mb0;
    }
    return l;
}

// Split-K finish of the 32 rows of quarter q of a tile. Every split's warp
// writes its fp32 partial rows, then arrives on the (tile, quarter) counter;
// the warp that arrives last sums the splits in the fixed order 0, 1, ...,
// S-1 (so the result does not depend on which CTA came last) and writes the
// output rows: SiLU(gate) * up in SWIGLU mode, the plain sum otherwise.
// Lane l owns 4 (SWIGLU) or 8 (PLAIN) output columns of every row; two rows
// and four splits are loaded per step so the L2 round trips overlap.
template <int MODE>
__device__ __forceinline__ void splitk_sum_rows(const KParams& p, const Tile& t, int lane, int nsplit, int r0,
                                                int nrows) {
    const int N = p.N[t.kind];
    constexpr int CPL = MODE == TC_SWIGLU ? 4 : 8;   // output columns per lane
    const int c = lane * CPL;
    const int col = (MODE == TC_SWIGLU ? t.n_blk * 128 : t.n_blk * 256) + c;
    if (col >= N) return;
    // SWIGLU: gate sums at partial column c, up sums at c + 128;
    // PLAIN: the 8 sums at c .. c + 7
    const int off0 = c, off1 = MODE == TC_SWIGLU ? 128 + c : c + 4;
    __nv_bfloat16* outp = static_cast<__nv_bfloat16*>(p.out[t.kind]);
#pragma unroll 1
    for (int i = 0; i < nrows; i += 2) {
        const int ib = i + 1 < nrows ? i + 1 : i;   // second row (a repeat of the first on an odd tail)
        const size_t oa = static_cast<size_t>(t.row0) + static_cast<size_t>(r0 + i);
        const size_t ob = static_cast<size_t>(t.row0) + static_cast<size_t>(r0 + ib);
        const float* pa = p.partial + oa * p.partial_ld + static_cast<size_t>(t.n_blk) * 256;
        const float* pb = p.partial + ob * p.partial_ld + static_cast<size_t>(t.n_blk) * 256;
        float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0, b0 = a0, b1 = a0;
#pragma unroll 4
        for (int sp = 0; sp < nsplit; ++sp) {
            const size_t so = static_cast<size_t>(sp) * p.partial_stride;
            const float4 x0 = __ldcg(reinterpret_cast<const float4*>(pa + so + off0));
            const float4 x1 = __ldcg(reinterpret_cast<const float4*>(pa + so + off1));
            const float4 y0 = __ldcg(reinterpret_cast<const float4*>(pb + so + off0));
            const float4 y1 = __ldcg(reinterpret_cast<const float4*>(pb + so + off1));
            a0.x += x0.x; a0.y += x0.y; a0.z += x0.z; a0.w += x0.w;
            a1.x += x1.x; a1.y += x1.y; a1.z += x1.z; a1.w += x1.w;
            b0.x += y0.x; b0.y += y0.y; b0.z += y0.z; b0.w += y0.w;
            b1.x += y1.x; b1.y += y1.y; b1.z += y1.z; b1.w += y1.w;
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            if (r == 1 && ib == i) break;
            const float4 g = r ? b0 : a0, v = r ? b1 : a1;
            const size_t orow = r ? ob : oa;
            if (MODE == TC_SWIGLU) {
                uint2 packed;
                packed.x = pack_bf16(silu(g.x) * v.x, silu(g.y) * v.y);
                packed.y = pack_bf16(silu(g.z) * v.z, silu(g.w) * v.w);
                *reinterpret_cast<uint2*>(outp + orow * N + col) = packed;
            } else {
                *reinterpret_cast<uint4*>(outp + orow * N + col) =
                    make_uint4(pack_bf16(g.x, g.y), pack_bf16(g.z, g.w), pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
            }
        }
    }
}

template <int MODE>
__device__ __noinline__ void splitk_finish(const KParams& p, const Tile& t, int q, int lane, int nsplit, int tile) {
    int32_t* cnt = p.sem + static_cast<size_t>(tile) * kSemPerTile + q;
    __syncwarp();   // every lane's partial stores precede lane 0's release below
    int old = 0;
    if (lane == 0) {
        asm volatile("fence.acq_rel.gpu;" ::: "memory");   // release the warp's partial rows
        old = atomicAdd(cnt, 1);
        if (old == nsplit - 1) {
            *cnt = 0;   // ready for the next pass (the schedule writer zeroes it too)
            asm volatile("fence.acq_rel.gpu;" ::: "memory");   // acquire the other splits' rows
        }
    }
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old != nsplit - 1) return;
    const int r0 = t.m_blk * BM + q * 32;
    splitk_sum_rows<MODE>(p, t, lane, nsplit, r0, min(32, t.rows - r0));
}

template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
tc_grouped_gemm(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                const __grid_constant__ CUtensorMap tmB00, const __grid_constant__ CUtensorMap tmB01,
                const __grid_constant__ CUtensorMap tmB10, const __grid_constant__ CUtensorMap tmB11,
                const __grid_constant__ CUtensorMap tmA0s, const KParams p) {
    constexpr int COLS_PER_TILE = MODE == TC_SWIGLU ? 128 : 256;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SharedCtl* ctl = reinterpret_cast<SharedCtl*>(smem + STAGES * STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);
            mbar_init(&ctl->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&ctl->tfull[a], 1);
            mbar_init(&ctl->tempty[a], 4);
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort_flag = 0;
        fence_mbar_init();
        prefetch_map(&tmA0); prefetch_map(&tmA1);
        prefetch_map(&tmB00); prefetch_map(&tmB01);
        prefetch_map(&tmB10); prefetch_map(&tmB11);
        if (p.split_grid) prefetch_map(&tmA0s);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&ctl->tmem_base)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    // Everything above (barriers, TMEM, descriptor prefetch) overlapped the
    // previous kernel. The A rows are always an output of the previous
    // kernel; the schedule is one too unless b_before_wait says it was
    // written earlier, in which case the schedule is read and the first
    // stages' weight tiles are requested before the wait.
    const bool early = p.b_before_wait != 0;
    if (!early) {
        pdl_wait();
        pdl_launch();
    }
    const int total = total_tiles(p, COLS_PER_TILE);
    // split-K: the device-chosen factor is stored after the tile schedule;
    // unit u covers tile u / nsplit and the K-blocks of split u % nsplit, so
    // CTAs running at the same time read different K ranges of the weights
    // (spreading the traffic over all DRAM channels)
    const int nsplit = (p.partial != nullptr && p.tiles != nullptr) ? p.tiles[p.E + p.has_shared + 1] : 1;
    const Units un = cta_units(p, total, nsplit);

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t issued_mask = 0, issued_ph = 0;
            bool aborted = false;
            int pre = 0;   // stages of the first unit whose weight tiles were requested before the wait
            // the unit's tile and K-block range (a split of it with split-K)
            bool cls_small = false;   // interleaved order: the unit is a small-class tile
            const uint64_t evict_first = l2_evict_first_policy();
            auto unit_tile = [&](int u, int& kb0, int& kb1) {
                cls_small = false;
                if (un.small) {
                    const Tile t = decode_small_tile(p, u);
                    kb0 = 0; kb1 = t.num_kb;
                    return t;
                }
                if (p.split_grid && p.interleave) {
                    const Tile t = decode_mixed(p, u, cls_small);
                    kb0 = 0; kb1 = t.num_kb;
                    return t;
                }
                const int sp = u % nsplit;
                const Tile t = decode_tile(p, u / nsplit);
                kb0 = sp * t.num_kb / nsplit; kb1 = (sp + 1) * t.num_kb / nsplit;
                return t;
            };
            // bytes of one stage: small tiles load only the group's 32-row boxes of A
            auto stage_tx = [&](const Tile& t) {
                return un.small ? static_cast<uint32_t>(B_BYTES + small_boxes(t) * 4096) : static_cast<uint32_t>(STAGE_BYTES);
            };
            // the weight rows of a tile; a small-class tile's are read by that tile
            // alone, so they go to L2 as evict-first
            auto load_b = [&](uint32_t sa, const TileLoads& l, int kb, uint64_t* bar) {
                if (cls_small) {
                    tma_load_2d_hint(sa + A_BYTES, l.mlo, bar, kb * BK, l.brow0, evict_first);
                    tma_load_2d_hint(sa + A_BYTES + B_HALF_BYTES, l.mhi, bar, kb * BK, l.brow1, evict_first);
                } else {
                    tma_load_2d(sa + A_BYTES, l.mlo, bar, kb * BK, l.brow0);
                    tma_load_2d(sa + A_BYTES + B_HALF_BYTES, l.mhi, bar, kb * BK, l.brow1);
                }
            };
            auto load_a = [&](uint32_t sa, const Tile& t, const TileLoads& l, int kb, uint64_t* bar) {
                if (un.small) {
                    const int nb = small_boxes(t);
                    for (int j = 0; j < nb; ++j) tma_load_2d(sa + j * 4096, &tmA0s, bar, kb * BK, t.row0 + 32 * j);
                } else {
                    tma_load_2d(sa, l.ma, bar, kb * BK, l.arow);
                }
            };
            if (early) {
                if (un.first < un.count) {
                    int kb0, kb1;
                    const Tile t = unit_tile(un.first, kb0, kb1);
                    const TileLoads l = tile_loads<MODE>(p, t, &tmA0, &tmA1, &tmB00, &tmB01, &tmB10, &tmB11);
                    for (int kb = kb0; kb < kb1 && pre < STAGES; ++kb, ++pre) {
                        // every stage is free at the start: no empty-barrier wait
                        const uint32_t sa = smem_u32(smem + pre * STAGE_BYTES);
                        mbar_arrive_expect_tx(&ctl->full[pre], stage_tx(t));
                        load_b(sa, l, kb, &ctl->full[pre]);
                        issued_mask |= 1u << pre;
                    }
                }
                pdl_wait();
                pdl_launch();
            }
            for (int u = un.first; u < un.count && !aborted; u += un.step) {
                int kb0, kb1;
                const Tile t = unit_tile(u, kb0, kb1);
                const TileLoads l = tile_loads<MODE>(p, t, &tmA0, &tmA1, &tmB00, &tmB01, &tmB10, &tmB11);
                for (int kb = kb0; kb < kb1; ++kb) {
                    const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
                    if (u == un.first && kb - kb0 < pre) {
                        // weights already requested: the A rows complete the stage
                        load_a(sa, t, l, kb, &ctl->full[s]);
                    } else {
                        if (!wait_bounded(&ctl->empty[s], ph ^ 1u, ctl, p)) { aborted = true; break; }
                        mbar_arrive_expect_tx(&ctl->full[s], stage_tx(t));
                        load_a(sa, t, l, kb, &ctl->full[s]);
                        load_b(sa, l, kb, &ctl->full[s]);
                    }
                    issued_mask |= 1u << s;
                    issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
            }
            if (aborted) {
                // let every load this thread started land before the CTA exits
                // (the stages requested before the wait got their A rows before
                // any wait could give up, so their barriers complete too)
                for (int st = 0; st < STAGES; ++st)
                    if ((issued_mask >> st) & 1u) wait_drain(&ctl->full[st], (issued_ph >> st) & 1u, p);
            }
        } else if (early) {
            pdl_wait();
            pdl_launch();
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (early) {
            pdl_wait();
            pdl_launch();
        }
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc(BM, 256);
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t aph = 0;
            bool aborted = false, issued_any = false;
            for (int u = un.first; u < un.count && !aborted; u += un.step) {
                int kb0 = 0, kb1;
                Tile t;
                if (un.small) {
                    t = decode_small_tile(p, u);
                    kb1 = t.num_kb;
                } else if (p.split_grid && p.interleave) {
                    bool cs;
                    t = decode_mixed(p, u, cs);
                    kb1 = t.num_kb;
                } else {
                    const int sp = u % nsplit;
                    t = decode_tile(p, u / nsplit);
                    kb0 = sp * t.num_kb / nsplit; kb1 = (sp + 1) * t.num_kb / nsplit;
                }
                // operand-swapped small tile: the two 128-row halves of the
                // weight tile are the M operands, the group's rows (N = 32 per
                // A box) the N operand; D columns [0, N) and [128, 128 + N)
                const uint32_t idesc_s = un.small ? make_idesc(BM, 32 * small_boxes(t)) : 0u;
                if (!wait_bounded(&ctl->tempty[acc], aph ^ 1u, ctl, p)) { aborted = true; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * ACC_COLS);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!wait_bounded(&ctl->full[s], ph, ctl, p)) { aborted = true; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
                    const uint64_t adesc = sw128_desc(sa);
                    const uint64_t bdesc = sw128_desc(sa + A_BYTES);
                    if (un.small) {
                        const uint64_t wlo = bdesc, whi = sw128_desc(sa + A_BYTES + B_HALF_BYTES);
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint32_t accum = (kb != kb0 || kk != 0) ? 1u : 0u;
                            tc_mma(d_tmem, wlo + 2u * kk, adesc + 2u * kk, idesc_s, accum);
                            tc_mma(d_tmem + 128u, whi + 2u * kk, adesc + 2u * kk, idesc_s, accum);
                        }
                    } else {
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            tc_mma(d_tmem, adesc + 2u * kk, bdesc + 2u * kk, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
                    }
                    issued_any = true;
                    tc_commit(&ctl->empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (aborted) break;
                tc_commit(&ctl->tfull[acc]);
                acc ^= 1;
                if (acc == 0) aph ^= 1u;
            }
            if (aborted && issued_any) {
                // all MMAs of this thread must finish before TMEM is freed
                tc_commit(&ctl->drain);
                wait_drain(&ctl->drain, 0, p);
            }
        }
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        if (early) {
            pdl_wait();
            pdl_launch();
        }
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int r = q * 32 + lane;            // accumulator row of this thread
        int acc = 0;
        uint32_t aph = 0;
        for (int u = un.first; u < un.count; u += un.step) {
            const int sp = un.small ? 0 : u % nsplit;
            bool cs;
            const Tile t = un.small ? decode_small_tile(p, u)
                         : (p.split_grid && p.interleave) ? decode_mixed(p, u, cs) : decode_tile(p, u / nsplit);
            if (!wait_bounded(&ctl->tfull[acc], aph, ctl, p)) break;
            tc_fence_after();
            const int grow = t.m_blk * BM + r;
            bool valid = grow < t.rows;
            const size_t orow = static_cast<size_t>(t.row0) + static_cast<size_t>(grow);
            if (kDebugChecks && valid && orow >= static_cast<size_t>(p.out_rows[t.kind])) {
                debug_record_bounds(p.status);   // an output row past its buffer: not stored
                valid = false;
            }
            const int N = p.N[t.kind];
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                static_cast<uint32_t>(acc * ACC_COLS);
            bool released = false;
            if (MODE != TC_F32OUT && un.small) {
                // operand-swapped tile: this thread's TMEM lane is output
                // column m of the tile, its columns are the group's rows
                __nv_bfloat16* outp = static_cast<__nv_bfloat16*>(p.out[0]);
                const int ncol = 32 * small_boxes(t);
                const int col0 = MODE == TC_SWIGLU ? t.n_blk * 128 + r : t.n_blk * 256 + r;
#pragma unroll 1
                for (int c = 0; c < ncol; c += 32) {
                    uint32_t v0[32], v1[32];
                    tmem_ld32(tb + c, v0);
                    tmem_ld32(tb + 128 + c, v1);
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int n = c + i;
                        if (n < t.rows && (!kDebugChecks || t.row0 + n < p.out_rows[0])) {
                            __nv_bfloat16* orow_p = outp + (static_cast<size_t>(t.row0) + n) * N;
                            const float a = __uint_as_float(v0[i]), b = __uint_as_float(v1[i]);
                            if (MODE == TC_SWIGLU) {
                                if (col0 < N) orow_p[col0] = __float2bfloat16_rn(silu(a) * b);
                            } else {
                                if (col0 < N) orow_p[col0] = __float2bfloat16_rn(a);
                                if (col0 + 128 < N) orow_p[col0 + 128] = __float2bfloat16_rn(b);
                            }
                        }
                    }
                }
            } else if (MODE != TC_F32OUT && nsplit > 1) {
                // fp32 partial of this split: the raw 256 accumulator columns
                float* out = p.partial + static_cast<size_t>(sp) * p.partial_stride + orow * p.partial_ld;
#pragma unroll 1
                for (int c = 0; c < 256; c += 32) {
                    uint32_t v[32];
                    tmem_ld32(tb + c, v);
                    const int col = t.n_blk * 256 + c;
                    if (valid && col < p.partial_ld) {
                        uint4* dst = reinterpret_cast<uint4*>(out + col);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                    }
                }
                // the accumulator is free as soon as it is read
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->tempty[acc]);
                released = true;
                if (t.m_blk * BM + q * 32 < t.rows) splitk_finish<MODE>(p, t, q, lane, nsplit, u / nsplit);
            } else if (MODE == TC_SWIGLU) {
                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out[t.kind]) + orow * N;
                // training: the gate and up pre-activations of the tile, in the
                // accumulator's own column order ([128 gate | 128 up] per tile)
                __nv_bfloat16* abbase = t.kind == 0 ? p.ab_out : p.ab_out_s;
                __nv_bfloat16* abrow = abbase != nullptr
                                           ? abbase + orow * (2 * static_cast<size_t>(N)) + t.n_blk * 256
                                           : nullptr;
#pragma unroll 1
                for (int c = 0; c < 128; c += 32) {
                    uint32_t gv[32], uv[32];
                    tmem_ld32(tb + c, gv);
                    tmem_ld32(tb + 128 + c, uv);
                    const int col = t.n_blk * 128 + c;
                    if (valid && col < N && abrow != nullptr) {
                        uint32_t pg[16], pu[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            pg[i] = pack_bf16(__uint_as_float(gv[2 * i]), __uint_as_float(gv[2 * i + 1]));
                            pu[i] = pack_bf16(__uint_as_float(uv[2 * i]), __uint_as_float(uv[2 * i + 1]));
                        }
                        uint4* dg = reinterpret_cast<uint4*>(abrow + c);
                        uint4* du = reinterpret_cast<uint4*>(abrow + 128 + c);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            dg[i] = make_uint4(pg[4 * i], pg[4 * i + 1], pg[4 * i + 2], pg[4 * i + 3]);
                            du[i] = make_uint4(pu[4 * i], pu[4 * i + 1], pu[4 * i + 2], pu[4 * i + 3]);
                        }
                    }
                    if (valid && col < N) {
                        uint32_t packed[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            float g0 = __uint_as_float(gv[2 * i]), g1 = __uint_as_float(gv[2 * i + 1]);
                            float u0 = __uint_as_float(uv[2 * i]), u1 = __uint_as_float(uv[2 * i + 1]);
                            packed[i] = pack_bf16(silu(g0) * u0, silu(g1) * u1);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(out + col);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
                    }
                }
            } else if (MODE == TC_PLAIN) {
                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out[t.kind]) + orow * N;
#pragma unroll 1
                for (int c = 0; c < 256; c += 32) {
                    uint32_t v[32];
                    tmem_ld32(tb + c, v);
                    const int col = t.n_blk * 256 + c;
                    if (valid && col < N) {
                        uint32_t packed[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i)
                            packed[i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                        uint4* dst = reinterpret_cast<uint4*>(out + col);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
                    }
                }
            } else {
                float* out = static_cast<float*>(p.out[t.kind]) + orow * N;
#pragma unroll 1
                for (int c = 0; c < 256; c += 32) {
                    uint32_t v[32];
                    tmem_ld32(tb + c, v);
                    const int col = t.n_blk * 256 + c;
                    if (valid && col < N) {
                        uint4* dst = reinterpret_cast<uint4*>(out + col);
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            dst[i] = make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                    }
                }
            }
            if (!released) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&ctl->tempty[acc]);
            }
            acc ^= 1;
            if (acc == 0) aph ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---- CTA-pair kernel (cta_group::2, M = 256) ---------------------------------
//
// The same grouped GEMM for groups large enough to fill 256-row tiles. The
// grid is clusters of two CTAs on neighbouring SMs; a cluster takes one
// 256 x 256 accumulator tile at a time: rank r loads the A rows [128 r,
// 128 r + 128) of the tile and one 128-row half of the B tile (SWIGLU: the
// W1 rows in rank 0 and the W3 rows of the same output columns in rank 1;
// PLAIN: rows [128 r, 128 r + 128) of the 256), and the leader (rank 0)
// issues M = 256 MMAs that read both CTAs' shared memory and write each
// CTA's accumulator rows into that CTA's tensor memory, [gate | up] or the
// 256 output columns, exactly as in the single-CTA kernel, so the epilogue
// is the same. Per SM, a K step moves a third less data through shared
// memory than the single-CTA tile of the same FLOPs (the B tile is read once
// for both SMs), which is what lets the tensor pipe run without waiting on
// shared-memory fill; 32 KB stages leave room for six of them.
// Protocol: the leader's full barrier of a stage counts both CTAs' bytes
// (each CTA's loads complete on it; only the leader arms it); MMA completion
// is committed to both CTAs' empty and accumulator-full barriers (one
// multicast commit); each CTA's four epilogue warps arrive on the leader's
// accumulator-empty barrier. Waits are bounded as in the single-CTA kernel;
// a wait that gives up also raises the other CTA's abort flag. No TMA
// multicast: every CTA loads its own tiles.
constexpr int PBM = 256;                               // rows of a pair tile
constexpr int P_STAGES = 6;
constexpr int P_STAGE_BYTES = A_BYTES + B_HALF_BYTES;  // 32 KB per CTA
constexpr int P_SMEM_BYTES = P_STAGES * P_STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;

struct PairCtl {
    uint64_t full[P_STAGES], empty[P_STAGES], tfull[2], tempty[2], drain;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ bool pair_wait(uint64_t* bar, uint32_t parity, PairCtl* ctl, uint32_t peer_abort,
                                          const KParams& p) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*reinterpret_cast<volatile int*>(&ctl->abort_flag)) return false;
        if (global_timer_ns() - t0 > static_cast<uint64_t>(p.timeout_ns)) {
            *reinterpret_cast<volatile int*>(&ctl->abort_flag) = 1;
            st_shared_remote_u32(peer_abort, 1u);
            atomicExch(p.status, MOE_ERR_TIMEOUT);
            return false;
        }
    }
}

// Epilogue of one accumulator tile for this thread's row (shared by nothing
// else: the single-CTA kernel keeps its own, with the split-K and training
// variants).
template <int MODE>
__device__ __forceinline__ void pair_store_row(const KParams& p, const Tile& t, uint32_t tb, bool valid,
                                               size_t orow) {
    const int N = p.N[t.kind];
    if (MODE == TC_SWIGLU) {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out[t.kind]) + orow * N;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
            uint32_t gv[32], uv[32];
            tmem_ld32(tb + c, gv);
            tmem_ld32(tb + 128 + c, uv);
            const int col = t.n_blk * 128 + c;
            if (valid && col < N) {
                uint32_t packed[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float g0 = __uint_as_float(gv[2 * i]), g1 = __uint_as_float(gv[2 * i + 1]);
                    const float u0 = __uint_as_float(uv[2 * i]), u1 = __uint_as_float(uv[2 * i + 1]);
                    packed[i] = pack_bf16(silu(g0) * u0, silu(g1) * u1);
                }
                uint4* dst = reinterpret_cast<uint4*>(out + col);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
            }
        }
    } else {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out[t.kind]) + orow * N;
#pragma unroll 1
        for (int c = 0; c < 256; c += 32) {
            uint32_t v[32];
            tmem_ld32(tb + c, v);
            const int col = t.n_blk * 256 + c;
            if (valid && col < N) {
                uint32_t packed[16];
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    packed[i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
                uint4* dst = reinterpret_cast<uint4*>(out + col);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
            }
        }
    }
}

// Epilogue of a half-width tail tile (N = 128 pair MMA over half of each
// CTA's B rows): accumulator columns [0, 64) come from rank 0's B rows
// [64 h, 64 h + 64), columns [64, 128) from rank 1's. SWIGLU: gate and up of
// the 64 output columns [n_blk 128 + 64 h, + 64); PLAIN: output columns
// n_blk 256 + 64 h + [0, 64) and n_blk 256 + 128 + 64 h + [0, 64).
template <int MODE>
__device__ __forceinline__ void pair_store_half_row(const KParams& p, const Tile& t, uint32_t tb, bool valid,
                                                    size_t orow, int half) {
    const int N = p.N[t.kind];
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out[t.kind]) + orow * N;
#pragma unroll 1
    for (int c = 0; c < 64; c += 32) {
        uint32_t lo[32], hi[32];
        tmem_ld32(tb + c, lo);
        tmem_ld32(tb + 64 + c, hi);
        if (!valid) continue;
        uint32_t pk_lo[16], pk_hi[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float a0 = __uint_as_float(lo[2 * i]), a1 = __uint_as_float(lo[2 * i + 1]);
            const float b0 = __uint_as_float(hi[2 * i]), b1 = __uint_as_float(hi[2 * i + 1]);
            if (MODE == TC_SWIGLU) {
                pk_lo[i] = pack_bf16(silu(a0) * b0, silu(a1) * b1);
            } else {
                pk_lo[i] = pack_bf16(a0, a1);
                pk_hi[i] = pack_bf16(b0, b1);
            }
        }
        if (MODE == TC_SWIGLU) {
            const int col = t.n_blk * 128 + 64 * half + c;
            if (col < N) {
                uint4* dst = reinterpret_cast<uint4*>(out + col);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk_lo[4 * i], pk_lo[4 * i + 1], pk_lo[4 * i + 2], pk_lo[4 * i + 3]);
            }
        } else {
            const int col0 = t.n_blk * 256 + 64 * half + c, col1 = col0 + 128;
            if (col0 < N) {
                uint4* dst = reinterpret_cast<uint4*>(out + col0);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk_lo[4 * i], pk_lo[4 * i + 1], pk_lo[4 * i + 2], pk_lo[4 * i + 3]);
            }
            if (col1 < N) {
                uint4* dst = reinterpret_cast<uint4*>(out + col1);
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk_hi[4 * i], pk_hi[4 * i + 1], pk_hi[4 * i + 2], pk_hi[4 * i + 3]);
            }
        }
    }
}

// Work items of the pair kernel: the tiles that fill whole waves of the
// grid, then the remaining (tail) tiles as two half-width items each, so the
// last wave is as short as a half tile. Item v -> tile, and half (-1: whole).
struct PairWork {
    int full, items;
};
__device__ __forceinline__ PairWork pair_work(int units, int nclusters) {
    PairWork w;
    w.full = (units / nclusters) * nclusters;
    const int tail = units - w.full;
    w.items = (tail > 0 && 2 * tail <= nclusters) ? w.full + 2 * tail : units;
    if (w.items == units) w.full = units;
    return w;
}
__device__ __forceinline__ int pair_item_tile(const PairWork& w, int v, int& half) {
    if (v < w.full) { half = -1; return v; }
    half = (v - w.full) & 1;
    return w.full + ((v - w.full) >> 1);
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
tc_pair_gemm(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
             const __grid_constant__ CUtensorMap tmB00, const __grid_constant__ CUtensorMap tmB01,
             const __grid_constant__ CUtensorMap tmB10, const __grid_constant__ CUtensorMap tmB11,
             const KParams p) {
    static_assert(MODE == TC_SWIGLU || MODE == TC_PLAIN, "pair tiles: SWIGLU or PLAIN");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    PairCtl* ctl = reinterpret_cast<PairCtl*>(smem + P_STAGES * P_STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const uint32_t peer_abort = mapa_shared(smem_u32(&ctl->abort_flag), rank ^ 1u);
    const int cluster = static_cast<int>(blockIdx.x >> 1), nclusters = static_cast<int>(gridDim.x >> 1);

    if (threadIdx.x == 0) {
        for (int s = 0; s < P_STAGES; ++s) {
            mbar_init(&ctl->full[s], 1);    // the leader's arming arrive (+ both CTAs' bytes)
            mbar_init(&ctl->empty[s], 1);   // one multicast MMA commit
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&ctl->tfull[a], 1);   // one multicast MMA commit
            mbar_init(&ctl->tempty[a], 8);  // four epilogue warps of each CTA (used in the leader)
        }
        mbar_init(&ctl->drain, 1);
        ctl->abort_flag = 0;
        fence_mbar_init();
        prefetch_map(&tmA0); prefetch_map(&tmA1);
        prefetch_map(&tmB00); prefetch_map(&tmB01);
        prefetch_map(&tmB10); prefetch_map(&tmB11);
    }
    if (warp == 1) {
        // one warp of each CTA, the same warp in both, allocates the pair's tensor memory
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(&ctl->tmem_base)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();   // both CTAs' barriers initialised and tensor memory allocated
    tc_fence_after();
    const uint32_t tmem_base = ctl->tmem_base;
    const bool early = p.b_before_wait != 0;
    if (!early) {
        pdl_wait();
        pdl_launch();
    }
    const int units = p.tiles[p.E + p.has_shared];
    const PairWork work = pair_work(units, nclusters);

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t armed_mask = 0, armed_ph = 0;   // leader: stages whose full barrier it armed
            bool aborted = false;
            int pre = 0;
            const CUtensorMap* mbh[2] = {MODE == TC_SWIGLU && rank ? &tmB01 : &tmB00,
                                         MODE == TC_SWIGLU && rank ? &tmB11 : &tmB10};
            auto b_row = [&](const Tile& t) {
                const int eoff = t.kind ? 0 : t.g * p.b_rows[0];
                return MODE == TC_SWIGLU ? eoff + t.n_blk * 128 : eoff + t.n_blk * 256 + static_cast<int>(rank) * 128;
            };
            auto full_of = [&](int st) { return mapa_shared(smem_u32(&ctl->full[st]), 0u); };
            if (early) {
                if (cluster < work.items) {
                    int hf;
                    const Tile t = decode_tile_m<PBM>(p, pair_item_tile(work, cluster, hf));
                    const int brow = b_row(t);
                    for (int kb = 0; kb < t.num_kb && pre < P_STAGES; ++kb, ++pre) {
                        const uint32_t sa = smem_u32(smem + pre * P_STAGE_BYTES);
                        if (leader) {
                            mbar_arrive_expect_tx(&ctl->full[pre], 2 * P_STAGE_BYTES);
                            armed_mask |= 1u << pre;
                        }
                        tma_load_2d_pair(sa + A_BYTES, mbh[t.kind], full_of(pre), kb * BK, brow);
                    }
                }
                pdl_wait();
                pdl_launch();
            }
            for (int u = cluster; u < work.items && !aborted; u += nclusters) {
                int hf;
                const Tile t = decode_tile_m<PBM>(p, pair_item_tile(work, u, hf));
                const CUtensorMap* ma = t.kind ? &tmA1 : &tmA0;
                const int arow = t.row0 + t.m_blk * PBM + static_cast<int>(rank) * BM;
                const int brow = b_row(t);
                for (int kb = 0; kb < t.num_kb; ++kb) {
                    const uint32_t sa = smem_u32(smem + s * P_STAGE_BYTES);
                    if (u == cluster && kb < pre) {
                        tma_load_2d_pair(sa, ma, full_of(s), kb * BK, arow);
                    } else {
                        if (!pair_wait(&ctl->empty[s], ph ^ 1u, ctl, peer_abort, p)) { aborted = true; break; }
                        if (leader) {
                            mbar_arrive_expect_tx(&ctl->full[s], 2 * P_STAGE_BYTES);
                            armed_mask |= 1u << s;
                            armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
                        }
                        tma_load_2d_pair(sa, ma, full_of(s), kb * BK, arow);
                        tma_load_2d_pair(sa + A_BYTES, mbh[t.kind], full_of(s), kb * BK, brow);
                    }
                    if (++s == P_STAGES) { s = 0; ph ^= 1u; }
                }
            }
            if (aborted) {
                // the leader's armed stages complete when both CTAs' bytes have
                // landed; a load of the other CTA's that no armed phase counts
                // is given a fixed time to land (it cannot be observed here)
                if (leader) {
                    for (int st = 0; st < P_STAGES; ++st)
                        if ((armed_mask >> st) & 1u) wait_drain(&ctl->full[st], (armed_ph >> st) & 1u, p);
                } else {
                    const uint64_t t0 = global_timer_ns();
                    while (global_timer_ns() - t0 < 50000ull) {}
                }
            }
        } else if (early) {
            pdl_wait();
            pdl_launch();
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (the leader's) ----------------
        if (early) {
            pdl_wait();
            pdl_launch();
        }
        if (lane == 0 && leader) {
            constexpr uint32_t idesc = make_idesc(PBM, 256);
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t aph = 0;
            bool aborted = false, issued_any = false;
            constexpr uint32_t idesc_half = make_idesc(PBM, 128);
            for (int u = cluster; u < work.items && !aborted; u += nclusters) {
                int hf;
                const Tile t = decode_tile_m<PBM>(p, pair_item_tile(work, u, hf));
                // a half-width item multiplies half of each CTA's B rows (N = 128)
                const uint32_t id = hf < 0 ? idesc : idesc_half;
                const uint32_t boff = hf > 0 ? 64u * 128u : 0u;
                if (!pair_wait(&ctl->tempty[acc], aph ^ 1u, ctl, peer_abort, p)) { aborted = true; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * ACC_COLS);
                for (int kb = 0; kb < t.num_kb; ++kb) {
                    if (!pair_wait(&ctl->full[s], ph, ctl, peer_abort, p)) { aborted = true; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * P_STAGE_BYTES);
                    const uint64_t adesc = sw128_desc(sa);
                    const uint64_t bdesc = sw128_desc(sa + A_BYTES + boff);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        tc_mma_pair(d_tmem, adesc + 2u * kk, bdesc + 2u * kk, id, (kb | kk) != 0 ? 1u : 0u);
                    issued_any = true;
                    tc_commit_pair_mc(&ctl->empty[s], 0x3);
                    if (++s == P_STAGES) { s = 0; ph ^= 1u; }
                }
                if (aborted) break;
                tc_commit_pair_mc(&ctl->tfull[acc], 0x3);
                acc ^= 1;
                if (acc == 0) aph ^= 1u;
            }
            if (aborted && issued_any) {
                // every MMA of this thread (both CTAs' memories) must finish
                // before either CTA frees its tensor memory
                tc_commit_pair(&ctl->drain);
                wait_drain(&ctl->drain, 0, p);
            }
        }
    } else {
        // ---------------- epilogue (warps 2..5 of both CTAs) ----------------
        if (early) {
            pdl_wait();
            pdl_launch();
        }
        const int q = warp & 3;
        const int r = static_cast<int>(rank) * BM + q * 32 + lane;   // row of this thread in the 256-row tile
        const uint32_t tempty_leader[2] = {mapa_shared(smem_u32(&ctl->tempty[0]), 0u),
                                           mapa_shared(smem_u32(&ctl->tempty[1]), 0u)};
        int acc = 0;
        uint32_t aph = 0;
        for (int u = cluster; u < work.items; u += nclusters) {
            int hf;
            const Tile t = decode_tile_m<PBM>(p, pair_item_tile(work, u, hf));
            if (!pair_wait(&ctl->tfull[acc], aph, ctl, peer_abort, p)) break;
            tc_fence_after();
            const int grow = t.m_blk * PBM + r;
            const size_t orow = static_cast<size_t>(t.row0) + static_cast<size_t>(grow);
            const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * ACC_COLS);
            bool valid = grow < t.rows;
            if (kDebugChecks && valid && orow >= static_cast<size_t>(p.out_rows[t.kind])) {
                debug_record_bounds(p.status);   // an output row past its buffer: not stored
                valid = false;
            }
            if (hf < 0) pair_store_row<MODE>(p, t, tb, valid, orow);
            else pair_store_half_row<MODE>(p, t, tb, valid, orow, hf);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (leader) mbar_arrive(&ctl->tempty[acc]);
                else mbar_arrive_remote(tempty_leader[acc]);
            }
            acc ^= 1;
            if (acc == 0) aph ^= 1u;
        }
    }

    // neither CTA leaves (or frees tensor memory) while the other may still
    // use its shared memory, barriers or tensor memory
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

// ---- host side --------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool get_encode() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

// 2-D bf16 map over a [rows, cols] row-major matrix, box 64 columns x
// box_rows rows, 128-byte swizzle; reads outside the matrix return zeros.
bool encode_map(CUtensorMap* m, const void* base, int rows, int cols, int box_rows);

// Encoded maps keyed by (base, rows, cols): the same key always encodes to the
// same map, so a hit is exactly a fresh encode, without the driver call.
struct MapCacheEntry {
    const void* base;
    int rows, cols, box_rows;
    CUtensorMap map;
};
constexpr int kMapCacheSize = 64;
MapCacheEntry g_map_cache[kMapCacheSize];
int g_map_cache_n = 0, g_map_cache_next = 0;
std::mutex g_map_cache_mu;

bool make_map(CUtensorMap* m, const void* base, int rows, int cols, int box_rows = 128) {
    {
        std::lock_guard<std::mutex> lk(g_map_cache_mu);
        for (int i = 0; i < g_map_cache_n; ++i) {
            const MapCacheEntry& c = g_map_cache[i];
            if (c.base == base && c.rows == rows && c.cols == cols && c.box_rows == box_rows) {
                *m = c.map;
                return true;
            }
        }
    }
    if (!encode_map(m, base, rows, cols, box_rows)) return false;
    std::lock_guard<std::mutex> lk(g_map_cache_mu);
    MapCacheEntry& c = g_map_cache[g_map_cache_next];
    c.base = base;
    c.rows = rows;
    c.cols = cols;
    c.box_rows = box_rows;
    c.map = *m;
    g_map_cache_next = (g_map_cache_next + 1) % kMapCacheSize;
    if (g_map_cache_n < kMapCacheSize) ++g_map_cache_n;
    return true;
}

// box_rows == kF32StoreBox: an fp32 matrix with 32 x 32 boxes (128-byte rows),
// the layout of the weight-gradient stores
constexpr int kF32StoreBox = -32;

bool encode_map(CUtensorMap* m, const void* base, int rows, int cols, int box_rows) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows > 0 ? rows : 1)};
    cuuint32_t estr[2] = {1, 1};
    if (box_rows == kF32StoreBox) {
        cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 4};
        cuuint32_t box[2] = {32, 32};
        return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {BK, static_cast<cuuint32_t>(box_rows)};
    CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int MODE>
cudaError_t launch_pair_mode(const KParams& kp, const CUtensorMap (&maps)[7], cudaStream_t st) {
    static bool attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(tc_pair_gemm<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             P_SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const int sms = device_sm_count();
    if (sms < 2) return cudaErrorInvalidDevice;
    return launch_k(tc_pair_gemm<MODE>, dim3(sms & ~1), dim3(NUM_THREADS), (size_t)P_SMEM_BYTES, st, maps[0],
                    maps[1], maps[2], maps[3], maps[4], maps[5], kp);
}

template <int MODE>
cudaError_t launch_mode(const TcArgs& a, const KParams& kp, const CUtensorMap (&maps)[7], cudaStream_t st) {
    static bool attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(tc_grouped_gemm<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    int grid = device_sm_count();
    if (grid <= 0) return cudaErrorInvalidDevice;
    return launch_k(tc_grouped_gemm<MODE>, dim3(grid), dim3(NUM_THREADS), (size_t)SMEM_BYTES, st, maps[0], maps[1],
                    maps[2], maps[3], maps[4], maps[5], maps[6], kp);
}

}  // namespace

int tc_out_cols_per_tile(int mode) { return mode == TC_SWIGLU ? 128 : 256; }

bool make_tmap(void* m, const void* base, int rows, int cols, int box_rows) {
    return get_encode() && make_map(static_cast<CUtensorMap*>(m), base, rows, cols, box_rows);
}

bool make_tmap_f32_store(void* m, const float* base, int rows, int cols) {
    return get_encode() && make_map(static_cast<CUtensorMap*>(m), base, rows, cols, kF32StoreBox);
}

cudaError_t launch_tc_gemm(const TcArgs& a, cudaStream_t st) {
    if (!get_encode()) return cudaErrorNotSupported;
    CUtensorMap maps[7];
    // A maps: [rows, K]; B maps: [total rows, K]; slot 6: the routed A rows
    // in 32-row boxes (operand-swapped small tiles). Unused slots reuse slot 0.
    const int has1 = a.has_shared && a.A[1] != nullptr;
    if (!make_map(&maps[0], a.A[0], a.a_rows[0], a.K[0])) return cudaErrorInvalidValue;
    if (!make_map(&maps[1], has1 ? a.A[1] : a.A[0], has1 ? a.a_rows[1] : a.a_rows[0], has1 ? a.K[1] : a.K[0]))
        return cudaErrorInvalidValue;
    if (!make_map(&maps[2], a.B[0][0], a.b_total_rows[0], a.K[0])) return cudaErrorInvalidValue;
    const void* b01 = a.mode == TC_SWIGLU ? a.B[0][1] : a.B[0][0];
    if (!make_map(&maps[3], b01, a.b_total_rows[0], a.K[0])) return cudaErrorInvalidValue;
    if (has1) {
        if (!make_map(&maps[4], a.B[1][0], a.b_total_rows[1], a.K[1])) return cudaErrorInvalidValue;
        const void* b11 = a.mode == TC_SWIGLU ? a.B[1][1] : a.B[1][0];
        if (!make_map(&maps[5], b11, a.b_total_rows[1], a.K[1])) return cudaErrorInvalidValue;
    } else {
        maps[4] = maps[2];
        maps[5] = maps[3];
    }
    if (a.split_grid && !a.interleave) {
        if (!make_map(&maps[6], a.A[0], a.a_rows[0], a.K[0], 32)) return cudaErrorInvalidValue;
    } else {
        maps[6] = maps[0];
    }
    KParams kp;
    kp.split_grid = a.split_grid;
    kp.interleave = a.interleave;
    kp.out_rows[0] = a.a_rows[0];
    kp.out_rows[1] = a.T;
    kp.indptr = a.indptr;
    kp.tiles = a.tiles;
    kp.static_rows = a.static_rows;
    kp.E = a.E;
    kp.has_shared = has1;
    kp.T = a.T;
    kp.b_rows[0] = a.b_rows[0]; kp.b_rows[1] = a.b_rows[1];
    kp.N[0] = a.N[0]; kp.N[1] = a.N[1];
    kp.K[0] = a.K[0]; kp.K[1] = a.K[1];
    kp.out[0] = a.out[0]; kp.out[1] = a.out[1];
    kp.status = a.status;
    kp.timeout_ns = a.timeout_ns > 0 ? a.timeout_ns : wait_limit_ns();
    kp.drain_ns = kDrainLimitNs;
    kp.partial = a.partial;
    kp.partial_stride = a.partial_stride;
    kp.partial_ld = a.partial_ld;
    kp.sem = a.sem;
    kp.ab_out = static_cast<__nv_bfloat16*>(a.ab_out);
    kp.ab_out_s = static_cast<__nv_bfloat16*>(a.ab_out_s);
    kp.b_before_wait = a.b_before_wait;
    const int cols = tc_out_cols_per_tile(a.mode);
    const bool pair = a.pair != 0;
    if ((pair || a.split_grid) && (a.mode == TC_F32OUT || a.partial != nullptr || a.ab_out != nullptr ||
                                   a.ab_out_s != nullptr || a.tiles == nullptr || a.indptr == nullptr))
        return cudaErrorInvalidValue;
    if (pair && a.split_grid) return cudaErrorInvalidValue;
    for (int kd = 0; kd < 2; ++kd) {
        kp.nt_blk[kd] = ceil_div(a.N[kd] > 0 ? a.N[kd] : 1, cols);
        const long long row_bytes = static_cast<long long>(pair ? PBM : BM) * (a.K[kd] > 0 ? a.K[kd] : 1) * 2;
        kp.band_m[kd] = MOE_RASTER_BYTES > 0 ? static_cast<int>(std::max(8ll, MOE_RASTER_BYTES / row_bytes)) : 0;
    }
    if (kp.partial != nullptr && kp.sem == nullptr) return cudaErrorInvalidValue;
    if (pair) return a.mode == TC_SWIGLU ? launch_pair_mode<TC_SWIGLU>(kp, maps, st)
                                         : launch_pair_mode<TC_PLAIN>(kp, maps, st);
    switch (a.mode) {
        case TC_SWIGLU: return launch_mode<TC_SWIGLU>(a, kp, maps, st);
        case TC_PLAIN: return launch_mode<TC_PLAIN>(a, kp, maps, st);
        default: return launch_mode<TC_F32OUT>(a, kp, maps, st);
    }
}

}  // namespace moe
