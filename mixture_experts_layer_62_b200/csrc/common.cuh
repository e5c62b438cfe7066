// Internal declarations shared by the kernels of the MoE-layer library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "moe.h"

namespace moe {

// Tokens per permutation chunk: the histogram, the rank computation and the
// gather all work on chunks of this many consecutive tokens.
constexpr int kChunk = 32;

// Debug build (compiled with MOE_DEBUG): device-side bounds checks record
// MOE_ERR_BOUNDS in a status word and skip the access.
#ifdef MOE_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
__device__ __forceinline__ void debug_record_bounds(int32_t* status) {
    if (status != nullptr) atomicCAS(status, MOE_OK, MOE_ERR_BOUNDS);
}

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Programmatic dependent launch. moe_forward launches every kernel after its
// first one with the programmatic-serialization attribute, so a kernel's
// launch and prologue overlap the tail of the kernel before it. Every kernel
// calls pdl_wait() before it touches anything an earlier kernel of the pass
// wrote (the wait returns once the preceding grid has completed and its
// writes are visible; without the attribute it returns at once), then
// pdl_launch() to let the next kernel start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Set by moe_forward (per host thread) while it enqueues the launches that
// may overlap their predecessor: g_pdl_pass marks the pass, g_pdl turns the
// attribute on once the pass's first kernel is enqueued.
extern thread_local bool g_pdl;
extern thread_local bool g_pdl_pass;
inline void g_pdl_after_first() {
    if (g_pdl_pass) g_pdl = true;
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                            Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = g_pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

inline size_t elem_bytes(int dtype) { return dtype == MOE_DTYPE_BF16 ? 2 : 4; }

// Byte offsets of everything the library keeps in the caller's workspace.
struct Layout {
    size_t idx, gate, pos, indptr, row_token, logits, wrt;
    size_t blockcnt, blockoff, blockpsum, blockextra, tiles13, tiles2;
    size_t xp, h, o, hs, s;
    size_t ab;              // gate/up pre-activations kept for the backward (train)
    size_t abs;             // the shared expert's, [T][2 d_ff_shared] (train)
    size_t part13, part2;   // fp32 split-K partials (small-T forward only)
    size_t sem;             // split-K arrival counters: [sem13_n] then [sem2_n]
    int sem13_n, sem2_n;
    size_t total;
};

// Split-K of the grouped GEMMs is used by moe_forward when the whole batch
// fits one M-block per expert (T*k <= kSplitMaxRows) and there is no shared
// expert; the split factor (<= kSplitMax) is chosen on the device from the
// real tile counts.
constexpr int kSplitMaxRows = 128;
constexpr int kSplitMax = 16;
bool split_allowed(const moe_problem& p);
Layout make_layout(const moe_problem& p);
// Rows a permuted buffer holds: T*k, plus E*(pad_rows-1) when rows are padded.
long long permuted_rows(const moe_problem& p);
// Byte offsets of the backward pass's own workspace.
struct BwdLayout {
    size_t dO, dAB, dXp, dz, dgate, tiles_dh, tiles_dx, dwr_part;
    size_t dz16, dxr;   // wide routers (E % 64 == 0): bf16 dz and the router term of dx
    size_t dABs, dXs, indptr_s, tiles_s_dh, tiles_s_dx;   // shared expert
    size_t total;
};
BwdLayout make_bwd_layout(const moe_problem& p);

// Split factors by the number of active experts (0 .. kSplitMaxRows): with at
// most kSplitMaxRows rows every active expert is one M-block, so a GEMM has
// n_active x (N-blocks) tiles and its factor is a function of n_active alone.
// Filled on the host (pick_split), read by the kernel that writes the tile
// schedule.
struct SplitTable {
    uint8_t s13[kSplitMaxRows + 1];
    uint8_t s2[kSplitMaxRows + 1];
};
// Split factor of a GEMM with `tiles` output tiles of `nkb` K-blocks on `sm`
// persistent CTAs: the s in [1, smax] that minimises rounds x unit cost,
// ceil(tiles * s / sm) * u(s), u(s) = ceil(nkb / s) + 1 K-blocks (the + 1 is
// each unit's pipeline start/finish), and for s > 1 at least the split
// epilogue's cost, which grows with the rows of the busiest expert (rows_q).
// The smaller s wins ties.
int pick_split(int tiles, int nkb, int sm, int smax, int rows_q);
// rows: T*k, the permuted rows of the pass
void fill_split_table(SplitTable& t, int nt13, int nt2, int nkb13, int nkb2, int sm, int smax, int rows);
// Arrival counters of the split-K GEMMs: one per (tile, quarter of the
// 128-row M-block), zeroed by the kernel that writes the tile schedule.
constexpr int kSemPerTile = 4;

// Kernel launchers (each returns cudaGetLastError() of its launches).
// status (may be null): the statistics' status word, reset to MOE_OK by the
// first kernel of a pass.
cudaError_t launch_transpose_wr(int dtype, const void* W_r, void* wrt, int d, int E, cudaStream_t st,
                                int32_t* status = nullptr);
cudaError_t launch_logits_simt(int dtype, const void* x, const void* wrt, float* logits,
                               int T, int d, int E, cudaStream_t st);
// Per-chunk expert counts are laid out [E][kk][NB] (expert, slot, chunk) with
// kk = k under the slot-priority drop order and kk = 1 otherwise.
constexpr int kMaxSlotCounts = 4096;   // E * k limit of the slot-priority order
inline int count_slots(const moe_problem& p) { return p.drop_order == MOE_DROP_SLOT ? p.k : 1; }
// Logits and selection in one kernel (E <= 64, d % 8 == 0): the outputs of
// launch_logits_simt followed by launch_select, from x and W_r [d, E] as
// given; resets *status (if not null) to MOE_OK.
bool route_fused_ok(int dtype, int d, int E);
bool route_fused_mma_ok(int d, int E);   // the bf16 fused router runs its MMA form
cudaError_t launch_route_fused(int dtype, const void* x, const void* W_r, const float* bias, int bias_mode,
                               int gate_mode, int kk, int T, int d, int E, int k, float* logits, int32_t* idx,
                               float* gate, int32_t* blockcnt, float* blockpsum, float* blockextra, int32_t* status,
                               cudaStream_t st);
cudaError_t launch_select(const float* logits, const float* bias, int bias_mode, int gate_mode, int kk, int T,
                          int E, int k, int32_t* idx, float* gate, int32_t* blockcnt, float* blockpsum,
                          float* blockextra, cudaStream_t st);
cudaError_t launch_hist(const int32_t* idx, int T, int k, int kk, int E, int32_t* blockcnt, cudaStream_t st);

// Scan over per-chunk expert counts: per-expert totals, capacity, indptr,
// chunk rank bases, statistics and (optionally) the tile schedules of the
// two grouped GEMMs.
// Grid split of the single-CTA grouped GEMMs for fine-grained experts: the
// groups of at most kSmallRows rows run as operand-swapped tiles (the
// weights as the 128-row MMA operand, the group's rows as N = 32..128, so a
// 7-row group costs little tensor work and its time is its weight stream) on
// the first S CTAs, while the other CTAs run the larger groups' ordinary
// tiles; the schedule writer picks S so that both classes end together.
// Schedule array of one GEMM with the split: [0..G] cumulative tiles of the
// large class, [G+1] split-K factor (1), [G+2] S, [G+3 .. 2G+3] cumulative
// tiles of the small class (one M block per group); without the split only
// [0..G+1] are used and [G+2] is 0.
constexpr int kSmallRows = 128;
struct GridSplit {
    int on;
    int interleave;           // 1: no CTA split; the small groups' tiles are spread through the large
                              // groups' in the order all CTAs take them (S written as 0)
    int k13, k2, k13s, k2s;   // K of the routed and shared GEMM 1/3 and GEMM 2
    int grid;                 // CTAs of the GEMM launches
    int force_ctas;           // > 0: S from the environment (tuning), else the cost model
};
inline int schedule_ints(int E) { return 2 * (E + 1) + 6; }

struct ScanArgs {
    int T, k, E, capacity;       // capacity < 0: unlimited
    int kk;                      // count slots per expert (k for slot priority, else 1)
    const int32_t* blockcnt;     // [E][kk][NB]
    int32_t* blockoff;           // [E][kk][NB]
    const float* blockpsum;      // [NB][E] or null (then P, f, l_aux untouched)
    const float* blockextra;     // [NB][3] z-loss, entropy, gap sums, or null
    int32_t* indptr;             // [E+1]
    void* stats;                 // moe_stats block
    // tile schedules (null pointers: skipped)
    int32_t* tiles13; int32_t* tiles2;   // [G+2]: cumulative tiles, then the split factor
    int tile_m, ntiles13, ntiles2, ntiles13_shared, ntiles2_shared, has_shared;
    int split_on;                // 0: no split (factors 1)
    int32_t* sem; int sem_n;     // split-K counters to zero (sem_n ints), or null
    SplitTable split;
    int pad;                     // > 0: indptr over kept rows rounded up to a multiple of pad
    GridSplit gsplit;            // small/large tile classes of the single-CTA GEMMs
};
cudaError_t launch_scan(const ScanArgs& a, cudaStream_t st);
// Padding rows of a padded permutation: rows [indptr[e] + kept[e], indptr[e+1])
// of xp become zeros and their row_token -1 (kept[] from the stats block).
cudaError_t launch_pad_fill(int dtype, const int32_t* indptr, const void* stats, int E, int d, void* xp,
                            int32_t* row_token, int pad, cudaStream_t st);
// Split-K setup of a tile schedule: factors by active-expert count and the
// counters to zero.
struct ScheduleSplit {
    int split_on;
    int32_t* sem; int sem_n;
    SplitTable split;
    GridSplit gsplit;
    // debug build: the given group offsets are checked against rows_max and
    // a violation is recorded in *status (when not null)
    int rows_max;
    int32_t* status;
};
cudaError_t launch_schedule(const int32_t* indptr, int E, int T, int has_shared, int tile_m,
                            int ntiles13, int ntiles2, int ntiles13_shared, int ntiles2_shared,
                            int32_t* tiles13, int32_t* tiles2, const ScheduleSplit& sp, cudaStream_t st);
cudaError_t launch_permute_gather(int dtype, const void* x, const int32_t* idx,
                                  const int32_t* blockoff, const int32_t* indptr,
                                  int T, int d, int E, int k, int kk, int capacity,
                                  int32_t* pos, int32_t* row_token, void* xp, cudaStream_t st);
// rows: rows of o (permuted rows); status: where a debug build records an
// out-of-range position (may be null)
cudaError_t launch_combine(int dtype, const void* o, const int32_t* pos, const float* gate,
                           const void* s, void* out, int T, int d, int k, int rows, int32_t* status,
                           cudaStream_t st);
cudaError_t launch_zero_stats(void* stats, int E, int capacity, cudaStream_t st);

// Small-batch router (T*k <= kSmallMaxPairs, E <= kSmallMaxE, E % 8 == 0,
// bf16, no shared expert): logits, selection, statistics, capacity, indptr,
// tile schedules with split factors, destinations and the row gather in two
// launches (one block per token, then one finishing kernel).
constexpr int kSmallMaxPairs = 64;
constexpr int kSmallMaxE = 64;
constexpr int kSmallMaxParts = 16;   // partial-logit blocks per token
struct SmallRouteArgs {
    const void* x; const void* W_r; const float* bias;
    int bias_mode, gate_mode, drop_slot, T, d, E, k, capacity;
    float* logits; float* probs /* partial logits [T][parts][E] */; int32_t* idx; float* gate; int32_t* pos; int32_t* indptr; int32_t* row_token;
    int32_t* status_reset;
    void* xp; void* stats;
    int32_t* tiles13; int32_t* tiles2;
    int nt13, nt2, split_on;
    int32_t* sem; int sem_n;     // split-K counters to zero, or null
    SplitTable split;
};
bool small_route_ok(const moe_problem& p);
cudaError_t launch_route_small(const SmallRouteArgs& a, cudaStream_t st);
int small_route_parts(int d);   // partial-logit blocks per token for row width d

// fp32 grouped GEMM on CUDA cores (the fp32 path). Tile 64 x 64.
constexpr int kSimtTileM = 64;
constexpr int kSimtTileN = 64;
struct GroupedArgs {
    const int32_t* indptr;   // routed row offsets [E+1] (device)
    const int32_t* tiles;    // cumulative tile counts [G+1] (device)
    int E, has_shared, T;    // group E (if present) covers rows [0, T)
    const void* A[2];        // routed A rows [*, K0], shared A rows [T, K1]
    int a_rows[2];           // allocated rows of each A buffer
    const void* B[2][2];     // [kind][0/1]: SWIGLU uses W1/W3, PLAIN uses [kind][0]
    int N[2], K[2];          // output columns and reduction length per kind
    void* out[2];            // [*, N0] and [T, N1]
    int32_t* status;
};
cudaError_t launch_simt_gemm(bool swiglu, const GroupedArgs& a, cudaStream_t st);

// Decode-sized bf16 grouped GEMM 1/3 + SwiGLU as weight-streaming GEMVs
// (groups of at most kGemvMaxRows rows, no shared expert): one contiguous
// range of 8-column output groups per CTA, K split over the CTA's warps.
constexpr int kGemvMaxRows = 8;
struct GemvLaunch {
    const int32_t* indptr;   // [E+1] (device)
    int E;
    const void* A;           // [rows_max, K] bf16: the permuted rows
    const void* B0;          // [E, N, K] bf16: W1
    const void* B1;          // [E, N, K] bf16: W3
    void* out;               // [rows_max, N] bf16: H
    int N, K, rows_max;
    int max_group_rows;      // largest group the offsets can hold (<= kGemvMaxRows)
    int grid;                // CTAs (the SM count)
    int32_t* status;
};
cudaError_t launch_gemv_swiglu(const GemvLaunch& a, cudaStream_t st);

// bf16 grouped GEMM on tcgen05 tensor cores (sm_100a). Tile 128 x 256.
constexpr int kTcTileM = 128;
constexpr int kTcPairTileM = 256;   // rows of a CTA-pair tile
// CTA-pair tiles for the prefill-sized grouped GEMMs of p (bf16, no split-K,
// not the training forward, unpadded, at least 512 rows per expert on
// average); the environment variable MOE_CTA_PAIR=0 turns them off.
bool use_pair_tiles(const moe_problem& p);
// The two-class schedule for p (bf16 inference, no split-K, no pairs, at
// least 32 experts), opt-in: MOE_INTERLEAVE=1 interleaves the classes,
// MOE_SMALL_CTAS=n > 0 splits the grid, n CTAs for the small class.
GridSplit grid_split_of(const moe_problem& p);
int tc_out_cols_per_tile(int mode);   // 128 for SWIGLU, 256 otherwise
enum TcMode { TC_SWIGLU = 0, TC_PLAIN = 1, TC_F32OUT = 2 };
struct TcArgs {
    int mode;
    const int32_t* indptr;   // null: one static group of `static_rows` rows
    const int32_t* tiles;    // null with indptr == null
    int static_rows;
    int E, has_shared, T;
    const void* A[2]; int a_rows[2];
    const void* B[2][2]; int b_rows[2];   // rows of one expert's matrix in B
    int b_total_rows[2];                  // rows of the whole B buffer
    int N[2], K[2];
    void* out[2];
    int32_t* status;
    long long timeout_ns;
    float* partial;            // split-K partials [split][rows][partial_ld] or null
    long long partial_stride;  // elements between splits
    int partial_ld;            // elements per row
    int32_t* sem;              // split-K arrival counters [tiles][kSemPerTile] (with partial)
    void* ab_out;              // SWIGLU, routed groups: also store the raw gate/up
                               // accumulators as bf16 [rows][2 N] (null: not kept)
    void* ab_out_s;            // SWIGLU, the shared expert's rows: the same [T][2 N1]
    // the tile schedule (indptr, tiles) was written two or more launches
    // back, so the weight loads of the first stages may start before the
    // dependency wait
    int b_before_wait;
    // 1: CTA pairs with 256-row tiles (the schedule counts 256-row M blocks);
    // SWIGLU or PLAIN, no split-K, no pre-activation output
    int pair;
    // 1: the schedule carries the small/large grid split (GridSplit); SWIGLU
    // or PLAIN, no split-K, no pre-activation output
    int split_grid;
    // with split_grid: the two classes are interleaved in one order over all
    // CTAs, the small groups as ordinary tiles whose weights are loaded with
    // an evict-first L2 policy
    int interleave;
};
cudaError_t launch_tc_gemm(const TcArgs& a, cudaStream_t st);
// Backward grouped GEMMs (tcgen05): see gemm_bwd_sm100.cu.
enum BwMode { BW_DH = 0, BW_DX = 1, BW_DW2 = 2, BW_DW13 = 3 };
struct BwdGemmArgs {
    int mode;
    const int32_t* indptr;   // padded group row offsets [E+1]
    const int32_t* tiles;    // BW_DH / BW_DX tile schedule [E+1] (null for the weight gradients)
    int E, M, N, K, d, d_ff;
    const void* A; int a_rows, a_cols;         // A operand matrix (row-major)
    const void* B0; const void* B1; int b_rows, b_cols;   // B operand matrices (B1: W3 for BW_DX)
    const void* ab;          // BW_DH: forward gate/up pre-activations
    void* out_bf16;          // BW_DH: dAB; BW_DX: dXp
    float* out0; float* out1;   // weight gradients
    int32_t* status;
};
cudaError_t launch_bwd_gemm(const BwdGemmArgs& a, cudaStream_t st);

// Backward elementwise and reduction kernels: see bwd.cu.
cudaError_t launch_bwd_gather(const void* dy, const void* o, const int32_t* pos, const float* gate, int T, int d,
                              int k, void* dO, float* dgate, cudaStream_t st);
// dz16 (may be null): a bf16 copy of dz for the tensor-core router GEMMs
cudaError_t launch_router_bwd(const float* logits, const int32_t* idx, const float* gate, const float* dgate,
                              const void* stats, int T, int E, int k, int gate_mode, float alpha, float beta,
                              float* dz, void* dz16, cudaStream_t st);
// dW_r = x^T dz via fp32 partials over 128-token chunks (part: ceil(T/128) * d * E floats)
cudaError_t launch_dwr(const void* x, const float* dz, int T, int d, int E, float* part, float* dW_r,
                       cudaStream_t st);
// dx = sum_j dXp[pos] + W_r dz (+ dXs, the shared expert's input gradient, when not null);
// dxr (may be null): the router term W_r dz already computed, fp32 [T][d]
cudaError_t launch_bwd_dx(const void* dXp, const int32_t* pos, const void* W_r, const float* dz, const void* dXs,
                          const float* dxr, int T, int d, int E, int k, void* dx, cudaStream_t st);
// indptr = {0, T}: the shared expert as one group over all tokens
cudaError_t launch_single_group(int32_t* indptr, int T, cudaStream_t st);
cudaError_t launch_bias_update(const void* stats, int T, int E, int k, float gamma, float* bias, cudaStream_t st);

// A cached 2-D bf16 tensor map over a row-major [rows, cols] matrix: box 64
// columns x box_rows rows, 128-byte swizzle, zeros outside (CUtensorMap is
// the driver type; passed as void* so this header needs no driver header).
bool make_tmap(void* map, const void* base, int rows, int cols, int box_rows);
// A cached 2-D fp32 tensor map for bulk stores: box 32 x 32, 128-byte swizzle.
bool make_tmap_f32_store(void* map, const float* base, int rows, int cols);

int device_sm_count();

// The problem checks every entry point shares (MOE_OK or an error code), and
// the capacity C = ceil(cf T k / E) (-1 = no limit).
int check_problem(const moe_problem* p);
// Wall-clock limit of every bounded mbarrier wait in the tensor-core kernels
// (nanoseconds; moe_set_wait_limit sets it, 2 s by default), and the limit of
// the drain that lets in-flight copies and MMAs land after a wait gave up
// (fixed, long: a drain cut short would let a CTA exit with a copy still
// landing in its shared memory).
long long wait_limit_ns();
constexpr long long kDrainLimitNs = 2000000000LL;
int capacity_of(const moe_problem* p);

}  // namespace moe
