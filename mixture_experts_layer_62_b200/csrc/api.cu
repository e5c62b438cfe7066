// C ABI of the MoE-layer library: argument checks, workspace layout and the
// launch sequence of the forward pass (route -> scan -> permute/gather ->
// grouped GEMM 1/3 + SwiGLU -> grouped GEMM 2 -> combine). Every launch is
// asynchronous on the caller's stream; the host never waits on the device.
#include <atomic>
#include <cmath>
#include <cstdlib>

#include "common.cuh"

namespace moe {

long long permuted_rows(const moe_problem& p) {
    const long long T = p.T > 0 ? p.T : 0;
    return T * p.k + (p.pad_rows > 0 ? (long long)p.E * (p.pad_rows - 1) : 0);
}

Layout make_layout(const moe_problem& p) {
    const size_t T = p.T > 0 ? (size_t)p.T : 0, k = (size_t)p.k, E = (size_t)p.E;
    const size_t Rmax = (size_t)permuted_rows(p);
    const size_t d = (size_t)p.d, dff = (size_t)p.d_ff, dfs = (size_t)(p.d_ff_shared > 0 ? p.d_ff_shared : 0);
    const size_t eb = elem_bytes(p.dtype);
    const size_t NB = (T + kChunk - 1) / kChunk;
    Layout L;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + (bytes > 0 ? bytes : 1), 256);
        return o;
    };
    L.idx = take(T * k * 4);
    L.gate = take(T * k * 4);
    L.pos = take(T * k * 4);
    L.indptr = take((E + 1) * 4);
    L.row_token = take(Rmax * 4);
    L.logits = take(T * E * 4);
    L.wrt = take(E * d * eb);
    const size_t kk = (size_t)count_slots(p);
    L.blockcnt = take(E * kk * NB * 4);
    L.blockoff = take(E * kk * NB * 4);
    // per-chunk probability sums; the small-batch router keeps its partial
    // logits [T][parts][E] here
    L.blockpsum = take((small_route_ok(p) ? T * kSmallMaxParts : NB) * E * 4);
    L.blockextra = take(NB * 3 * 4);
    L.tiles13 = take((size_t)schedule_ints(p.E) * 4);
    L.tiles2 = take((size_t)schedule_ints(p.E) * 4);
    L.xp = take(Rmax * d * eb);
    L.h = take(Rmax * dff * eb);
    L.o = take(Rmax * d * eb);
    L.hs = take(T * dfs * eb);
    L.s = take(dfs ? T * d * eb : 0);
    L.ab = take(p.train ? Rmax * 2 * dff * eb : 0);
    L.abs = take(p.train ? T * 2 * dfs * eb : 0);
    const bool split = split_allowed(p);
    L.part13 = take(split ? (size_t)kSplitMax * T * k * (size_t)ceil_div(p.d_ff, 128) * 256 * 4 : 0);
    L.part2 = take(split ? (size_t)kSplitMax * T * k * d * 4 : 0);
    // at most min(E, T*k) experts are active, each with one M-block of tiles
    const size_t active = split ? (T * k < E ? T * k : E) : 0;
    L.sem13_n = (int)(active * (size_t)ceil_div(p.d_ff, 128) * kSemPerTile);
    L.sem2_n = (int)(active * (size_t)ceil_div(p.d, 256) * kSemPerTile);
    L.sem = take(((size_t)L.sem13_n + (size_t)L.sem2_n) * 4);
    L.total = off;
    return L;
}

BwdLayout make_bwd_layout(const moe_problem& p) {
    const size_t T = p.T > 0 ? (size_t)p.T : 0, k = (size_t)p.k, E = (size_t)p.E;
    const size_t d = (size_t)p.d, dff = (size_t)p.d_ff, eb = elem_bytes(p.dtype);
    const size_t Rmax = (size_t)permuted_rows(p);
    BwdLayout B;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off = align_up(off + (bytes > 0 ? bytes : 1), 256);
        return o;
    };
    B.dO = take(Rmax * d * eb);
    B.dAB = take(Rmax * 2 * dff * eb);
    B.dXp = take(Rmax * d * eb);
    B.dz = take(T * E * 4);
    B.dgate = take(T * k * 4);
    B.tiles_dh = take((size_t)schedule_ints(p.E) * 4);
    B.tiles_dx = take((size_t)schedule_ints(p.E) * 4);
    const bool tc_router = E % 64 == 0;
    B.dwr_part = take(tc_router ? 0 : (size_t)ceil_div((int)T, 128) * d * E * 4);
    B.dz16 = take(tc_router ? T * E * 2 : 0);
    B.dxr = take(tc_router ? T * d * 4 : 0);
    const size_t dfs = (size_t)(p.d_ff_shared > 0 ? p.d_ff_shared : 0);
    B.dABs = take(T * 2 * dfs * eb);
    B.dXs = take(dfs ? T * d * eb : 0);
    B.indptr_s = take(2 * 4);
    B.tiles_s_dh = take(4 * 4);
    B.tiles_s_dx = take(4 * 4);
    B.total = off;
    return B;
}

int pick_split(int tiles, int nkb, int sm, int smax, int rows_q) {
    if (smax <= 1 || tiles <= 0 || sm <= 0) return 1;
    // a split unit costs at least the split epilogue (partial rows out, the
    // arrival, and for the last split the sum over all splits), charged in
    // K-blocks: 12 plus 2.5 per row of the busiest 32-row quarter
    const int epi = 12 + (5 * (rows_q < 32 ? rows_q : 32) + 1) / 2;
    long long best = -1;
    int bs = 1;
    for (int s = 1; s <= smax && s <= nkb; ++s) {
        int unit = (nkb + s - 1) / s + 1;
        if (s > 1 && unit < epi) unit = epi;
        const long long c = ((long long)tiles * s + sm - 1) / sm * unit;
        if (best < 0 || c < best) {
            best = c;
            bs = s;
        }
    }
    return bs;
}

void fill_split_table(SplitTable& t, int nt13, int nt2, int nkb13, int nkb2, int sm, int smax, int rows) {
    // the table depends on seven integers; reuse the last one this thread built
    static thread_local int key[7] = {-1, -1, -1, -1, -1, -1, -1};
    static thread_local SplitTable last;
    const int k7[7] = {nt13, nt2, nkb13, nkb2, sm, smax, rows};
    bool hit = true;
    for (int i = 0; i < 7; ++i) hit = hit && key[i] == k7[i];
    if (!hit) {
        for (int n = 0; n <= kSplitMaxRows; ++n) {
            // rows of the busiest expert, estimated as 1.5 x the mean
            const int rq = n > 0 ? (3 * rows + 2 * n - 1) / (2 * n) : 0;
            last.s13[n] = (uint8_t)pick_split(n * nt13, nkb13, sm, smax, rq);
            last.s2[n] = (uint8_t)pick_split(n * nt2, nkb2, sm, smax, rq);
        }
        for (int i = 0; i < 7; ++i) key[i] = k7[i];
    }
    t = last;
}

bool split_allowed(const moe_problem& p) {
    return p.dtype == MOE_DTYPE_BF16 && p.d_ff_shared == 0 && p.T > 0 && p.pad_rows == 0 && !p.train &&
           (long long)p.T * p.k <= kSplitMaxRows;
}

// Decode-sized batches (at most 8 permuted rows by default, bf16, no shared
// expert) run GEMM 1/3 as weight-streaming GEMVs; GEMM 2 keeps the split-K
// tensor-core tiles. Measured against split-K tiles for both (decode at
// d = 4096, d_ff = 14336, top-2 of 8): 3 % faster per step at one token,
// 1.4 % at two, 0.5 % at four, 2.7 % slower at eight. MOE_GEMV=0 keeps the
// split-K tiles; MOE_GEMV_ROWS=n lowers the row limit (measurement; n <= 8).
bool gemv_on(const moe_problem& p) {
    static const bool enabled = [] {
        const char* v = std::getenv("MOE_GEMV");
        return !(v != nullptr && v[0] == '0');
    }();
    static const int rows = [] {
        const char* v = std::getenv("MOE_GEMV_ROWS");
        const int n = v != nullptr ? std::atoi(v) : 8;
        return n < 0 ? 0 : (n > kGemvMaxRows ? kGemvMaxRows : n);
    }();
    return enabled && split_allowed(p) && (long long)p.T * p.k <= rows;
}

// Split-K tensor-core tiles (GEMM 2 of every small batch; GEMM 1/3 where the
// GEMVs do not take it).
bool split_k_on(const moe_problem& p) { return split_allowed(p); }

bool use_pair_tiles(const moe_problem& p) {
    static const bool enabled = [] {
        const char* v = std::getenv("MOE_CTA_PAIR");
        return !(v != nullptr && v[0] == '0');
    }();
    return enabled && p.dtype == MOE_DTYPE_BF16 && p.T > 0 && p.pad_rows == 0 && !p.train && !split_allowed(p) &&
           (long long)p.T * p.k >= 512LL * p.E;
}

GridSplit grid_split_of(const moe_problem& p) {
    static const int forced = [] {
        const char* v = std::getenv("MOE_SMALL_CTAS");
        return v != nullptr ? std::atoi(v) : -1;
    }();
    // Both two-class schedules are opt-in: on the DeepSeek-shaped layer
    // (alternating runs on one box) the grid split (MOE_SMALL_CTAS=n > 0)
    // measured 7.43-7.49 ms per step against 7.39-7.44 ms without, the
    // interleaved order (MOE_INTERLEAVE=1) 7.86-7.89 ms against 7.75-7.82 ms.
    static const bool interleave = [] {
        const char* v = std::getenv("MOE_INTERLEAVE");
        return v != nullptr && v[0] == '1';
    }();
    GridSplit g = {};
    g.interleave = forced > 0 ? 0 : 1;
    g.on = (forced > 0 || (forced != 0 && interleave)) && p.dtype == MOE_DTYPE_BF16 && p.T > 0 && p.pad_rows == 0 &&
           !p.train && !split_allowed(p) && !use_pair_tiles(p) && p.E >= 32 && p.d % 64 == 0;
    g.k13 = p.d; g.k2 = p.d_ff; g.k13s = p.d; g.k2s = p.d_ff_shared;
    g.grid = device_sm_count();
    g.force_ctas = forced > 0 ? forced : 0;
    if (g.grid <= 1 && !g.interleave) g.on = 0;
    return g;
}

thread_local bool g_pdl = false;
thread_local bool g_pdl_pass = false;

constexpr long long kDefaultWaitLimitNs = 2000000000LL;
std::atomic<long long> g_wait_limit_ns{kDefaultWaitLimitNs};

long long wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

int device_sm_count() {
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return -1;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
        cache[dev] = n;
    }
    return cache[dev];
}

int check_problem(const moe_problem* p) {
    if (p == nullptr) return MOE_ERR_INVALID_ARG;
    if (p->T < 0 || p->d <= 0 || p->d_ff <= 0 || p->E < 1 || p->E > MOE_MAX_E || p->k < 1 ||
        p->k > p->E || p->k > MOE_MAX_K || p->d_ff_shared < 0)
        return MOE_ERR_INVALID_ARG;
    if (p->dtype != MOE_DTYPE_F32 && p->dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (p->bias_mode < MOE_BIAS_NONE || p->bias_mode > MOE_BIAS_PROB) return MOE_ERR_INVALID_ARG;
    if (p->gate_mode != MOE_GATE_SELECTED && p->gate_mode != MOE_GATE_FULL) return MOE_ERR_INVALID_ARG;
    if (p->drop_order != MOE_DROP_TOKEN && p->drop_order != MOE_DROP_SLOT) return MOE_ERR_INVALID_ARG;
    if (p->drop_order == MOE_DROP_SLOT && p->E * p->k > kMaxSlotCounts) return MOE_ERR_UNSUPPORTED;
    if (!std::isfinite(p->capacity_factor)) return MOE_ERR_INVALID_ARG;
    if (p->pad_rows != 0 && p->pad_rows != 64 && p->pad_rows != 128) return MOE_ERR_INVALID_ARG;
    if (p->train != 0 && p->train != 1) return MOE_ERR_INVALID_ARG;
    if (p->train && (p->dtype != MOE_DTYPE_BF16 || p->d_ff % 128 || p->d_ff_shared % 128)) return MOE_ERR_UNSUPPORTED;
    const long long rows = permuted_rows(*p);
    if (rows * (long long)(p->d > p->d_ff ? p->d : p->d_ff) >= (1LL << 40) || rows >= (1LL << 30))
        return MOE_ERR_UNSUPPORTED;
    if (p->dtype == MOE_DTYPE_BF16) {
        if (p->d % 64 || p->d_ff % 64 || p->d_ff_shared % 64) return MOE_ERR_UNSUPPORTED;
    } else {
        if (p->d % 8 || p->d_ff % 4 || p->d_ff_shared % 4) return MOE_ERR_UNSUPPORTED;
    }
    return MOE_OK;
}

// C = ceil(cf * T * k / E), computed in double from the float factor; -1 = none.
int capacity_of(const moe_problem* p) {
    double cf = (double)p->capacity_factor;
    if (!(cf > 0.0)) return -1;
    double c = std::ceil(cf * (double)p->T * (double)p->k / (double)p->E);
    if (c > 2147483647.0) return -1;
    return (int)c;
}

}  // namespace moe

using namespace moe;

namespace {

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

#define CK(expr)                                   \
    do {                                           \
        if ((expr) != cudaSuccess) return MOE_ERR_CUDA; \
    } while (0)

char* wsp(void* ws, size_t off) { return static_cast<char*>(ws) + off; }

// The general-path router: tensor cores for wide bf16 routers (a real GEMM),
// otherwise one fused kernel (logits and selection) where it applies.
bool router_on_tensor_cores(const moe_problem* p) {
    return p->dtype == MOE_DTYPE_BF16 && p->E >= 64 && p->E % 32 == 0;
}
bool router_fused(const moe_problem* p) {
    return !router_on_tensor_cores(p) && route_fused_ok(p->dtype, p->d, p->E);
}

// Router: logits (fp32) for all tokens into `logits`.
int run_logits(const moe_problem* p, const void* x, const void* W_r, float* logits, const Layout& L,
               void* ws, int32_t* status, cudaStream_t st, bool reset_status = false) {
    void* wrt = wsp(ws, L.wrt);
    CK(launch_transpose_wr(p->dtype, W_r, wrt, p->d, p->E, st, reset_status ? status : nullptr));
    g_pdl_after_first();
    if (router_on_tensor_cores(p)) {
        // wide routers (e.g. 256 experts) are a real GEMM: tensor cores, fp32 out
        TcArgs a = {};
        a.mode = TC_F32OUT;
        a.indptr = nullptr;
        a.tiles = nullptr;
        a.static_rows = p->T;
        a.E = 1;
        a.has_shared = 0;
        a.T = p->T;
        a.A[0] = x; a.a_rows[0] = p->T;
        a.B[0][0] = wrt; a.B[0][1] = wrt; a.b_rows[0] = p->E; a.b_total_rows[0] = p->E;
        a.N[0] = p->E; a.K[0] = p->d;
        a.out[0] = logits;
        a.status = status;
        CK(launch_tc_gemm(a, st));
    } else {
        CK(launch_logits_simt(p->dtype, x, wrt, logits, p->T, p->d, p->E, st));
    }
    return MOE_OK;
}

// Arguments of a GEMV launch. group_rows: the most rows one expert can
// hold (T when the offsets come from the router, which picks distinct experts
// per token; 0: any split of the T*k rows).
GemvLaunch gemv_launch(const moe_problem* p, const int32_t* indptr, const void* A, const void* B0, const void* B1,
                       void* out, int N, int K, int group_rows, int32_t* status) {
    GemvLaunch g = {};
    g.indptr = indptr;
    g.E = p->E;
    g.A = A;
    g.B0 = B0;
    g.B1 = B1;
    g.out = out;
    g.N = N;
    g.K = K;
    g.rows_max = (int)permuted_rows(*p);
    g.max_group_rows = group_rows > 0 && group_rows < g.rows_max ? group_rows : g.rows_max;
    g.grid = device_sm_count();
    g.status = status;
    return g;
}

// Grouped GEMM 1/3 with the SwiGLU epilogue (and the shared expert's).
int run_up(const moe_problem* p, const void* xp, const int32_t* indptr, const int32_t* tiles13, const void* W1,
           const void* W3, const void* x, const void* Ws1, const void* Ws3, void* h, void* hs, int32_t* status,
           cudaStream_t st, float* part13 = nullptr, int32_t* sem13 = nullptr, bool sched_early = true,
           void* ab = nullptr, void* ab_s = nullptr, int group_rows = 0) {
    const int has_shared = p->d_ff_shared > 0 ? 1 : 0;
    const int rows = p->T * p->k;
    const int arows = (int)permuted_rows(*p);   // rows of the permuted buffers
    if (gemv_on(*p)) {
        CK(launch_gemv_swiglu(gemv_launch(p, indptr, xp, W1, W3, h, p->d_ff, p->d, group_rows, status), st));
        return MOE_OK;
    }
    if (p->dtype == MOE_DTYPE_BF16) {
        TcArgs a = {};
        a.mode = TC_SWIGLU;
        a.pair = use_pair_tiles(*p) ? 1 : 0;
        {
            const GridSplit gs = grid_split_of(*p);
            a.split_grid = gs.on;
            a.interleave = gs.on && gs.interleave;
        }
        a.b_before_wait = sched_early ? 1 : 0;
        a.indptr = indptr; a.tiles = tiles13;
        a.E = p->E; a.has_shared = has_shared; a.T = p->T;
        a.A[0] = xp; a.a_rows[0] = arows; a.A[1] = has_shared ? x : nullptr; a.a_rows[1] = p->T;
        a.B[0][0] = W1; a.B[0][1] = W3; a.b_rows[0] = p->d_ff; a.b_total_rows[0] = p->E * p->d_ff;
        a.B[1][0] = Ws1; a.B[1][1] = Ws3; a.b_rows[1] = p->d_ff_shared; a.b_total_rows[1] = p->d_ff_shared;
        a.N[0] = p->d_ff; a.N[1] = p->d_ff_shared;
        a.K[0] = p->d; a.K[1] = p->d;
        a.out[0] = h; a.out[1] = hs;
        a.ab_out = ab;
        a.ab_out_s = ab_s;
        a.status = status;
        if (part13 != nullptr) {
            a.partial = part13;
            a.partial_ld = ceil_div(p->d_ff, 128) * 256;
            a.partial_stride = (long long)rows * a.partial_ld;
            a.sem = sem13;
        }
        CK(launch_tc_gemm(a, st));
    } else {
        GroupedArgs a = {};
        a.indptr = indptr; a.tiles = tiles13;
        a.E = p->E; a.has_shared = has_shared; a.T = p->T;
        a.A[0] = xp; a.a_rows[0] = arows; a.A[1] = x; a.a_rows[1] = p->T;
        a.B[0][0] = W1; a.B[0][1] = W3; a.B[1][0] = Ws1; a.B[1][1] = Ws3;
        a.N[0] = p->d_ff; a.N[1] = p->d_ff_shared;
        a.K[0] = p->d; a.K[1] = p->d;
        a.out[0] = h; a.out[1] = hs;
        a.status = status;
        CK(launch_simt_gemm(true, a, st));
    }
    return MOE_OK;
}

// Grouped GEMM 2 (down projection, and the shared expert's).
int run_down(const moe_problem* p, const void* h, const int32_t* indptr, const int32_t* tiles2, const void* W2,
             const void* hs, const void* Ws2, void* o, void* s, int32_t* status, cudaStream_t st,
             float* part2 = nullptr, int32_t* sem2 = nullptr) {
    const int has_shared = p->d_ff_shared > 0 ? 1 : 0;
    const int rows = p->T * p->k;
    const int arows = (int)permuted_rows(*p);   // rows of the permuted buffers
    if (p->dtype == MOE_DTYPE_BF16) {
        TcArgs b = {};
        b.mode = TC_PLAIN;
        b.pair = use_pair_tiles(*p) ? 1 : 0;
        {
            const GridSplit gs = grid_split_of(*p);
            b.split_grid = gs.on;
            b.interleave = gs.on && gs.interleave;
        }
        b.b_before_wait = 1;   // the schedule comes from the router, two or more launches back
        b.indptr = indptr; b.tiles = tiles2;
        b.E = p->E; b.has_shared = has_shared; b.T = p->T;
        b.A[0] = h; b.a_rows[0] = arows; b.A[1] = has_shared ? hs : nullptr; b.a_rows[1] = p->T;
        b.B[0][0] = W2; b.B[0][1] = W2; b.b_rows[0] = p->d; b.b_total_rows[0] = p->E * p->d;
        b.B[1][0] = Ws2; b.B[1][1] = Ws2; b.b_rows[1] = p->d; b.b_total_rows[1] = p->d;
        b.N[0] = p->d; b.N[1] = p->d;
        b.K[0] = p->d_ff; b.K[1] = p->d_ff_shared;
        b.out[0] = o; b.out[1] = s;
        b.status = status;
        if (part2 != nullptr) {
            b.partial = part2;
            b.partial_ld = p->d;
            b.partial_stride = (long long)rows * p->d;
            b.sem = sem2;
        }
        CK(launch_tc_gemm(b, st));
    } else {
        GroupedArgs b = {};
        b.indptr = indptr; b.tiles = tiles2;
        b.E = p->E; b.has_shared = has_shared; b.T = p->T;
        b.A[0] = h; b.a_rows[0] = arows; b.A[1] = hs; b.a_rows[1] = p->T;
        b.B[0][0] = W2; b.B[0][1] = nullptr; b.B[1][0] = Ws2; b.B[1][1] = nullptr;
        b.N[0] = p->d; b.N[1] = p->d;
        b.K[0] = p->d_ff; b.K[1] = p->d_ff_shared;
        b.out[0] = o; b.out[1] = s;
        b.status = status;
        CK(launch_simt_gemm(false, b, st));
    }
    return MOE_OK;
}

int run_experts(const moe_problem* p, const void* xp, const int32_t* indptr, const int32_t* tiles13,
                const int32_t* tiles2, const void* W1, const void* W3, const void* W2, const void* x,
                const void* Ws1, const void* Ws3, const void* Ws2, void* h, void* hs, void* o, void* s,
                int32_t* status, cudaStream_t st, float* part13 = nullptr, float* part2 = nullptr,
                int32_t* sem13 = nullptr, int32_t* sem2 = nullptr, bool sched_early = true, void* ab = nullptr,
                void* ab_s = nullptr, int group_rows = 0) {
    int rc = run_up(p, xp, indptr, tiles13, W1, W3, x, Ws1, Ws3, h, hs, status, st, part13, sem13, sched_early, ab,
                    ab_s, group_rows);
    if (rc != MOE_OK) return rc;
    return run_down(p, h, indptr, tiles2, W2, hs, Ws2, o, s, status, st, part2, sem2);
}

void schedule_sizes(const moe_problem* p, int& tile_m, int& nt13, int& nt2, int& nt13s, int& nt2s) {
    if (p->dtype == MOE_DTYPE_BF16) {
        tile_m = use_pair_tiles(*p) ? kTcPairTileM : kTcTileM;
        int c13 = tc_out_cols_per_tile(TC_SWIGLU), c2 = tc_out_cols_per_tile(TC_PLAIN);
        nt13 = ceil_div(p->d_ff, c13);
        nt2 = ceil_div(p->d, c2);
        nt13s = ceil_div(p->d_ff_shared, c13);
        nt2s = nt2;
    } else {
        tile_m = kSimtTileM;
        nt13 = ceil_div(p->d_ff, kSimtTileN);
        nt2 = ceil_div(p->d, kSimtTileN);
        nt13s = ceil_div(p->d_ff_shared, kSimtTileN);
        nt2s = nt2;
    }
}

// Split-K state of the expert stages: factors, partial buffers, counters.
struct StageSplit {
    ScheduleSplit sched = {};
    float* part13 = nullptr;
    float* part2 = nullptr;
    int32_t* sem13 = nullptr;
    int32_t* sem2 = nullptr;
};
StageSplit stage_split(const moe_problem* p, const Layout& L, void* ws, int32_t* status) {
    StageSplit s;
    s.sched.gsplit = grid_split_of(*p);
    s.sched.rows_max = (int)permuted_rows(*p);
    s.sched.status = status;
    if (!split_k_on(*p)) return s;
    int tile_m, nt13, nt2, nt13s, nt2s;
    schedule_sizes(p, tile_m, nt13, nt2, nt13s, nt2s);
    s.sched.split_on = 1;
    s.sem13 = reinterpret_cast<int32_t*>(wsp(ws, L.sem));
    s.sem2 = s.sem13 + L.sem13_n;
    s.sched.sem = s.sem13;
    s.sched.sem_n = L.sem13_n + L.sem2_n;
    fill_split_table(s.sched.split, nt13, nt2, ceil_div(p->d, 64), ceil_div(p->d_ff, 64), device_sm_count(),
                     kSplitMax, p->T * p->k);
    s.part13 = reinterpret_cast<float*>(wsp(ws, L.part13));
    s.part2 = reinterpret_cast<float*>(wsp(ws, L.part2));
    return s;
}

}  // namespace

extern "C" {

size_t moe_stats_size(int32_t E) { return sizeof(moe_stats) + 16u * (size_t)(E > 0 ? E : 0); }

size_t moe_workspace_size(const moe_problem* p) {
    if (check_problem(p) != MOE_OK) return 0;
    return make_layout(*p).total;
}

int moe_workspace_layout(const moe_problem* p, moe_workspace_layout_t* out) {
    int rc = check_problem(p);
    if (rc != MOE_OK) return rc;
    if (out == nullptr) return MOE_ERR_INVALID_ARG;
    Layout L = make_layout(*p);
    out->idx = L.idx; out->gate = L.gate; out->pos = L.pos; out->indptr = L.indptr;
    out->row_token = L.row_token; out->logits = L.logits; out->xp = L.xp; out->h = L.h;
    out->o = L.o; out->hs = L.hs; out->s = L.s; out->ab = L.ab; out->total = L.total;
    return MOE_OK;
}

int moe_device_sm_count(void) { return device_sm_count(); }

int moe_gemm_variant(const moe_problem* p) {
    const int rc = check_problem(p);
    if (rc != MOE_OK) return -rc;
    if (p->dtype != MOE_DTYPE_BF16) return MOE_GEMM_SIMT;
    if (gemv_on(*p)) return MOE_GEMM_GEMV;
    if (split_allowed(*p)) return MOE_GEMM_SPLIT_K;
    if (use_pair_tiles(*p)) return MOE_GEMM_PAIR;
    {
        const GridSplit gs = grid_split_of(*p);
        if (gs.on) return gs.interleave ? MOE_GEMM_INTERLEAVED : MOE_GEMM_GRID_SPLIT;
    }
    return MOE_GEMM_SINGLE;
}

int moe_router_variant(const moe_problem* p, int forward) {
    const int rc = check_problem(p);
    if (rc != MOE_OK) return -rc;
    if (forward && small_route_ok(*p)) return MOE_ROUTER_SMALL;
    if (router_fused(p))
        return p->dtype == MOE_DTYPE_BF16 && route_fused_mma_ok(p->d, p->E) ? MOE_ROUTER_FUSED_MMA
                                                                            : MOE_ROUTER_FUSED_FMA;
    return router_on_tensor_cores(p) ? MOE_ROUTER_TENSOR : MOE_ROUTER_SIMT;
}

long long moe_set_wait_limit(long long ns) {
    return g_wait_limit_ns.exchange(ns > 0 ? ns : kDefaultWaitLimitNs);
}

// ---- backward ----------------------------------------------------------------

size_t moe_backward_workspace_size(const moe_problem* p) {
    if (check_problem(p) != MOE_OK) return 0;
    return make_bwd_layout(*p).total;
}

int moe_backward(const moe_problem* p, const void* x, const void* W_r, const void* W1, const void* W3,
                 const void* W2, const void* Ws1, const void* Ws3, const void* Ws2, const void* dy, float alpha,
                 float beta, void* dx, float* dW_r, float* dW1, float* dW3, float* dW2, float* dWs1, float* dWs3,
                 float* dWs2, void* stats, const void* workspace, size_t workspace_bytes, void* bwd_workspace,
                 size_t bwd_workspace_bytes, void* stream) {
    int rc = check_problem(p);
    if (rc != MOE_OK) return rc;
    if (!p->train || (p->pad_rows != 64 && p->pad_rows != 128) || p->E % 8) return MOE_ERR_UNSUPPORTED;
    const bool shared = p->d_ff_shared > 0;
    if (!x || !W_r || !W1 || !W3 || !W2 || !dy || !dx || !dW_r || !dW1 || !dW3 || !dW2 || !stats)
        return MOE_ERR_INVALID_ARG;
    if (shared && (!Ws1 || !Ws3 || !Ws2 || !dWs1 || !dWs3 || !dWs2)) return MOE_ERR_INVALID_ARG;
    for (const void* q : {x, W_r, W1, W3, W2, dy, (const void*)dx, (const void*)dW_r, (const void*)dW1,
                          (const void*)dW3, (const void*)dW2, (const void*)stats})
        if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (shared)
        for (const void* q : {Ws1, Ws3, Ws2, (const void*)dWs1, (const void*)dWs3, (const void*)dWs2})
            if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (!std::isfinite(alpha) || !std::isfinite(beta)) return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(*p);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_WORKSPACE;
    const BwdLayout B = make_bwd_layout(*p);
    if (!bwd_workspace || bwd_workspace_bytes < B.total || (reinterpret_cast<uintptr_t>(bwd_workspace) & 255u))
        return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (p->T == 0) {
        CK(cudaMemsetAsync(dW_r, 0, sizeof(float) * (size_t)p->d * p->E, st));
        const size_t nw = (size_t)p->E * p->d_ff * p->d * sizeof(float);
        CK(cudaMemsetAsync(dW1, 0, nw, st));
        CK(cudaMemsetAsync(dW3, 0, nw, st));
        CK(cudaMemsetAsync(dW2, 0, nw, st));
        if (shared) {
            const size_t ns = (size_t)p->d_ff_shared * p->d * sizeof(float);
            CK(cudaMemsetAsync(dWs1, 0, ns, st));
            CK(cudaMemsetAsync(dWs3, 0, ns, st));
            CK(cudaMemsetAsync(dWs2, 0, ns, st));
        }
        return MOE_OK;
    }
    struct PdlPass {
        PdlPass() { g_pdl_pass = true; g_pdl = false; }
        ~PdlPass() { g_pdl_pass = false; g_pdl = false; }
    } pdl_pass;
    char* ws = static_cast<char*>(const_cast<void*>(workspace));
    char* bw = static_cast<char*>(bwd_workspace);
    const int32_t* pos = reinterpret_cast<const int32_t*>(ws + L.pos);
    const int32_t* idx = reinterpret_cast<const int32_t*>(ws + L.idx);
    const float* gate = reinterpret_cast<const float*>(ws + L.gate);
    const int32_t* indptr = reinterpret_cast<const int32_t*>(ws + L.indptr);
    const float* logits = reinterpret_cast<const float*>(ws + L.logits);
    void* dO = bw + B.dO;
    void* dAB = bw + B.dAB;
    void* dXp = bw + B.dXp;
    float* dz = reinterpret_cast<float*>(bw + B.dz);
    float* dgate = reinterpret_cast<float*>(bw + B.dgate);
    int32_t* tiles_dh = reinterpret_cast<int32_t*>(bw + B.tiles_dh);
    int32_t* tiles_dx = reinterpret_cast<int32_t*>(bw + B.tiles_dx);
    int32_t* status = static_cast<int32_t*>(stats);
    const int Rmax = (int)permuted_rows(*p);

    CK(launch_bwd_gather(dy, ws + L.o, pos, gate, p->T, p->d, p->k, dO, dgate, st));
    g_pdl_after_first();
    CK(launch_pad_fill(p->dtype, indptr, stats, p->E, p->d, dO, nullptr, p->pad_rows, st));
    // wide routers (E % 64 == 0) run both router GEMMs on the tensor cores
    // with dz rounded to bf16: dW_r = x^T dz (one group of T rows, both
    // operands MN-major) and the router term of dx, dz W_r^T (fp32 out)
    const bool tc_router = p->E % 64 == 0;
    void* dz16 = tc_router ? bw + B.dz16 : nullptr;
    float* dxr = tc_router ? reinterpret_cast<float*>(bw + B.dxr) : nullptr;
    int32_t* indptr_s = reinterpret_cast<int32_t*>(bw + B.indptr_s);
    CK(launch_router_bwd(logits, idx, gate, dgate, stats, p->T, p->E, p->k, p->gate_mode, alpha, beta, dz, dz16,
                         st));
    if (tc_router) {
        CK(launch_single_group(indptr_s, p->T, st));
        BwdGemmArgs r = {};
        r.mode = BW_DW2; r.indptr = indptr_s; r.tiles = nullptr; r.E = 1;
        r.M = p->d; r.N = p->E; r.K = 0; r.d = p->d; r.d_ff = p->E;
        r.A = x; r.a_rows = p->T; r.a_cols = p->d;
        r.B0 = dz16; r.b_rows = p->T; r.b_cols = p->E;
        r.out0 = dW_r; r.status = status;
        CK(launch_bwd_gemm(r, st));
        TcArgs a = {};
        a.mode = TC_F32OUT; a.indptr = nullptr; a.tiles = nullptr; a.static_rows = p->T;
        a.E = 1; a.has_shared = 0; a.T = p->T;
        a.A[0] = dz16; a.a_rows[0] = p->T;
        a.B[0][0] = W_r; a.B[0][1] = W_r; a.b_rows[0] = p->d; a.b_total_rows[0] = p->d;
        a.N[0] = p->d; a.K[0] = p->E;
        a.out[0] = dxr; a.status = status;
        CK(launch_tc_gemm(a, st));
    } else {
        CK(launch_dwr(x, dz, p->T, p->d, p->E, reinterpret_cast<float*>(bw + B.dwr_part), dW_r, st));
    }
    ScheduleSplit nosplit = {};
    CK(launch_schedule(indptr, p->E, p->T, 0, kTcTileM, ceil_div(p->d_ff, 256), ceil_div(p->d, 256), 0, 0,
                       tiles_dh, tiles_dx, nosplit, st));
    BwdGemmArgs g = {};
    g.indptr = indptr;
    g.E = p->E;
    g.d = p->d;
    g.d_ff = p->d_ff;
    g.status = status;
    // dH = dO W2_e, with the SwiGLU derivative in the epilogue -> dAB
    g.mode = BW_DH; g.tiles = tiles_dh; g.N = p->d_ff; g.K = p->d;
    g.A = dO; g.a_rows = Rmax; g.a_cols = p->d;
    g.B0 = W2; g.B1 = nullptr; g.b_rows = p->E * p->d; g.b_cols = p->d_ff;
    g.ab = ws + L.ab; g.out_bf16 = dAB;
    CK(launch_bwd_gemm(g, st));
    // dXp = dA W1_e + dB W3_e
    g.mode = BW_DX; g.tiles = tiles_dx; g.N = p->d; g.K = 2 * p->d_ff;
    g.A = dAB; g.a_rows = Rmax; g.a_cols = 2 * p->d_ff;
    g.B0 = W1; g.B1 = W3; g.b_rows = p->E * p->d_ff; g.b_cols = p->d;
    g.ab = nullptr; g.out_bf16 = dXp;
    CK(launch_bwd_gemm(g, st));
    // dW2_e = dO_e^T H_e
    g.mode = BW_DW2; g.tiles = nullptr; g.M = p->d; g.N = p->d_ff; g.K = 0;
    g.A = dO; g.a_rows = Rmax; g.a_cols = p->d;
    g.B0 = ws + L.h; g.B1 = nullptr; g.b_rows = Rmax; g.b_cols = p->d_ff;
    g.out_bf16 = nullptr; g.out0 = dW2; g.out1 = nullptr;
    CK(launch_bwd_gemm(g, st));
    // [dW1_e; dW3_e] = dAB_e^T Xp_e
    g.mode = BW_DW13; g.M = 2 * p->d_ff; g.N = p->d;
    g.A = dAB; g.a_rows = Rmax; g.a_cols = 2 * p->d_ff;
    g.B0 = ws + L.xp; g.b_rows = Rmax; g.b_cols = p->d;
    g.out0 = dW1; g.out1 = dW3;
    CK(launch_bwd_gemm(g, st));
    void* dXs = nullptr;
    if (shared) {
        // the always-on expert: one group of all T rows, gate 1, so its output
        // gradient is dy itself; rows are not padded (the tensor maps end at
        // row T, so the last K-block of its weight gradients reads zeros)
        const int dfs = p->d_ff_shared;
        int32_t* ts_dh = reinterpret_cast<int32_t*>(bw + B.tiles_s_dh);
        int32_t* ts_dx = reinterpret_cast<int32_t*>(bw + B.tiles_s_dx);
        void* dABs = bw + B.dABs;
        dXs = bw + B.dXs;
        if (!tc_router) CK(launch_single_group(indptr_s, p->T, st));
        CK(launch_schedule(indptr_s, 1, p->T, 0, kTcTileM, ceil_div(dfs, 256), ceil_div(p->d, 256), 0, 0, ts_dh,
                           ts_dx, nosplit, st));
        BwdGemmArgs s1 = {};
        s1.indptr = indptr_s;
        s1.E = 1;
        s1.d = p->d;
        s1.d_ff = dfs;
        s1.status = status;
        s1.mode = BW_DH; s1.tiles = ts_dh; s1.N = dfs; s1.K = p->d;
        s1.A = dy; s1.a_rows = p->T; s1.a_cols = p->d;
        s1.B0 = Ws2; s1.b_rows = p->d; s1.b_cols = dfs;
        s1.ab = ws + L.abs; s1.out_bf16 = dABs;
        CK(launch_bwd_gemm(s1, st));
        s1.mode = BW_DX; s1.tiles = ts_dx; s1.N = p->d; s1.K = 2 * dfs;
        s1.A = dABs; s1.a_rows = p->T; s1.a_cols = 2 * dfs;
        s1.B0 = Ws1; s1.B1 = Ws3; s1.b_rows = dfs; s1.b_cols = p->d;
        s1.ab = nullptr; s1.out_bf16 = dXs;
        CK(launch_bwd_gemm(s1, st));
        s1.mode = BW_DW2; s1.tiles = nullptr; s1.M = p->d; s1.N = dfs; s1.K = 0;
        s1.A = dy; s1.a_rows = p->T; s1.a_cols = p->d;
        s1.B0 = ws + L.hs; s1.B1 = nullptr; s1.b_rows = p->T; s1.b_cols = dfs;
        s1.out_bf16 = nullptr; s1.out0 = dWs2; s1.out1 = nullptr;
        CK(launch_bwd_gemm(s1, st));
        s1.mode = BW_DW13; s1.M = 2 * dfs; s1.N = p->d;
        s1.A = dABs; s1.a_rows = p->T; s1.a_cols = 2 * dfs;
        s1.B0 = x; s1.b_rows = p->T; s1.b_cols = p->d;
        s1.out0 = dWs1; s1.out1 = dWs3;
        CK(launch_bwd_gemm(s1, st));
    }
    CK(launch_bwd_dx(dXp, pos, W_r, dz, dXs, dxr, p->T, p->d, p->E, p->k, dx, st));
    return MOE_OK;
}

int moe_bias_update(const moe_problem* p, const void* stats, float gamma, float* bias, void* stream) {
    int rc = check_problem(p);
    if (rc != MOE_OK) return rc;
    if (!stats || !bias || !aligned16(stats) || !std::isfinite(gamma)) return MOE_ERR_INVALID_ARG;
    CK(launch_bias_update(stats, p->T, p->E, p->k, gamma, bias, static_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

int32_t moe_permuted_rows(const moe_problem* p) {
    if (check_problem(p) != MOE_OK) return 0;
    return (int32_t)permuted_rows(*p);
}

const char* moe_error_string(int code) {
    switch (code) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_CUDA: return "CUDA launch or driver error";
        case MOE_ERR_TIMEOUT: return "device-side bounded wait timed out";
        case MOE_ERR_BOUNDS: return "device-side bounds check failed (debug build)";
        default: return "unknown error";
    }
}

int moe_forward(const moe_problem* p, const void* x, const void* W_r, const float* bias, const void* W1,
                const void* W3, const void* W2, const void* Ws1, const void* Ws3, const void* Ws2, void* out,
                void* stats, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_problem(p);
    if (rc != MOE_OK) return rc;
    const bool shared = p->d_ff_shared > 0;
    if (!x || !W_r || !W1 || !W3 || !W2 || !out || !stats) return MOE_ERR_INVALID_ARG;
    if (p->bias_mode != MOE_BIAS_NONE && !bias) return MOE_ERR_INVALID_ARG;
    if (shared && (!Ws1 || !Ws3 || !Ws2)) return MOE_ERR_INVALID_ARG;
    for (const void* q : {x, W_r, W1, W3, W2, (const void*)out, (const void*)stats})
        if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (shared)
        for (const void* q : {Ws1, Ws3, Ws2})
            if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(*p);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int C = capacity_of(p);
    int32_t* status = static_cast<int32_t*>(stats);
    if (p->T == 0) {
        CK(launch_zero_stats(stats, p->E, C, st));
        return MOE_OK;
    }
    // launches after the first overlap their predecessor (programmatic
    // dependent launch); the first kernel resets the status word
    struct PdlPass {
        PdlPass() { g_pdl_pass = true; g_pdl = false; }
        ~PdlPass() { g_pdl_pass = false; g_pdl = false; }
    } pdl_pass;
    float* logits = reinterpret_cast<float*>(wsp(workspace, L.logits));
    int32_t* idx = reinterpret_cast<int32_t*>(wsp(workspace, L.idx));
    float* gate = reinterpret_cast<float*>(wsp(workspace, L.gate));
    int32_t* pos = reinterpret_cast<int32_t*>(wsp(workspace, L.pos));
    int32_t* indptr = reinterpret_cast<int32_t*>(wsp(workspace, L.indptr));
    int32_t* row_token = reinterpret_cast<int32_t*>(wsp(workspace, L.row_token));
    int32_t* blockcnt = reinterpret_cast<int32_t*>(wsp(workspace, L.blockcnt));
    int32_t* blockoff = reinterpret_cast<int32_t*>(wsp(workspace, L.blockoff));
    float* blockpsum = reinterpret_cast<float*>(wsp(workspace, L.blockpsum));
    int32_t* tiles13 = reinterpret_cast<int32_t*>(wsp(workspace, L.tiles13));
    int32_t* tiles2 = reinterpret_cast<int32_t*>(wsp(workspace, L.tiles2));

    const bool split = split_k_on(*p);
    int32_t* sem = split ? reinterpret_cast<int32_t*>(wsp(workspace, L.sem)) : nullptr;
    void* xp = wsp(workspace, L.xp);
    const bool small = small_route_ok(*p);
    if (small) {
        // decode-sized batch: routing, statistics, schedules and the gather in one block
        SmallRouteArgs sr = {};
        sr.x = x; sr.W_r = W_r; sr.bias = bias;
        sr.bias_mode = p->bias_mode; sr.gate_mode = p->gate_mode; sr.drop_slot = p->drop_order == MOE_DROP_SLOT;
        sr.T = p->T; sr.d = p->d; sr.E = p->E; sr.k = p->k; sr.capacity = C;
        sr.logits = logits; sr.probs = blockpsum; sr.idx = idx; sr.gate = gate; sr.pos = pos; sr.indptr = indptr; sr.row_token = row_token;
        sr.xp = xp; sr.stats = stats; sr.tiles13 = tiles13; sr.tiles2 = tiles2; sr.status_reset = status;
        int tile_m, nt13s, nt2s;
        schedule_sizes(p, tile_m, sr.nt13, sr.nt2, nt13s, nt2s);
        sr.split_on = split ? 1 : 0;
        if (split) {
            sr.sem = sem;
            sr.sem_n = L.sem13_n + L.sem2_n;
            fill_split_table(sr.split, sr.nt13, sr.nt2, ceil_div(p->d, 64), ceil_div(p->d_ff, 64),
                             device_sm_count(), kSplitMax, p->T * p->k);
        }
        CK(launch_route_small(sr, st));
    } else {
    float* blockextra = reinterpret_cast<float*>(wsp(workspace, L.blockextra));
    const int kk = count_slots(*p);
    if (router_fused(p)) {
        CK(launch_route_fused(p->dtype, x, W_r, bias, p->bias_mode, p->gate_mode, kk, p->T, p->d, p->E, p->k,
                              logits, idx, gate, blockcnt, blockpsum, blockextra, status, st));
        g_pdl_after_first();
    } else {
        rc = run_logits(p, x, W_r, logits, L, workspace, status, st, /*reset_status=*/true);
        if (rc != MOE_OK) return rc;
        CK(launch_select(logits, bias, p->bias_mode, p->gate_mode, kk, p->T, p->E, p->k, idx, gate, blockcnt,
                         blockpsum, blockextra, st));
    }
    ScanArgs sa = {};
    sa.T = p->T; sa.k = p->k; sa.E = p->E; sa.capacity = C; sa.kk = kk;
    sa.blockcnt = blockcnt; sa.blockoff = blockoff; sa.blockpsum = blockpsum; sa.blockextra = blockextra;
    sa.indptr = indptr; sa.stats = stats;
    sa.tiles13 = tiles13; sa.tiles2 = tiles2; sa.has_shared = shared ? 1 : 0;
    schedule_sizes(p, sa.tile_m, sa.ntiles13, sa.ntiles2, sa.ntiles13_shared, sa.ntiles2_shared);
    sa.gsplit = grid_split_of(*p);
    sa.split_on = split ? 1 : 0;
    if (split) {
        sa.sem = sem;
        sa.sem_n = L.sem13_n + L.sem2_n;
        fill_split_table(sa.split, sa.ntiles13, sa.ntiles2, ceil_div(p->d, 64), ceil_div(p->d_ff, 64),
                         device_sm_count(), kSplitMax, p->T * p->k);
    }
    sa.pad = p->pad_rows;
    CK(launch_scan(sa, st));
    CK(launch_permute_gather(p->dtype, x, idx, blockoff, indptr, p->T, p->d, p->E, p->k, kk, C, pos, row_token, xp,
                             st));
    if (p->pad_rows > 0)
        CK(launch_pad_fill(p->dtype, indptr, stats, p->E, p->d, xp, row_token, p->pad_rows, st));
    }
    void* h = wsp(workspace, L.h);
    void* o = wsp(workspace, L.o);
    void* hs = shared ? wsp(workspace, L.hs) : nullptr;
    void* s = shared ? wsp(workspace, L.s) : nullptr;
    float* part13 = split ? reinterpret_cast<float*>(wsp(workspace, L.part13)) : nullptr;
    float* part2 = split ? reinterpret_cast<float*>(wsp(workspace, L.part2)) : nullptr;
    // the small router writes the schedule right before GEMM 1/3; the general
    // path writes it in the scan, two launches before
    rc = run_experts(p, xp, indptr, tiles13, tiles2, W1, W3, W2, x, Ws1, Ws3, Ws2, h, hs, o, s, status, st, part13,
                     part2, sem, sem ? sem + L.sem13_n : nullptr, /*sched_early=*/!small,
                     p->train ? wsp(workspace, L.ab) : nullptr,
                     (p->train && shared) ? wsp(workspace, L.abs) : nullptr, /*group_rows=*/p->T);
    if (rc != MOE_OK) return rc;
    CK(launch_combine(p->dtype, o, pos, gate, s, out, p->T, p->d, p->k, (int)permuted_rows(*p), status, st));
    return MOE_OK;
}

int moe_route(const moe_problem* p, const void* x, const void* W_r, const float* bias, int32_t* idx, float* gate,
              float* logits, void* stats, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_problem(p);
    if (rc != MOE_OK) return rc;
    if (!x || !W_r || !idx || !gate || !stats) return MOE_ERR_INVALID_ARG;
    if (p->bias_mode != MOE_BIAS_NONE && !bias) return MOE_ERR_INVALID_ARG;
    for (const void* q : {x, W_r, (const void*)stats})
        if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (logits && !aligned16(logits)) return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(*p);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int C = capacity_of(p);
    if (p->T == 0) {
        CK(launch_zero_stats(stats, p->E, C, st));
        return MOE_OK;
    }
    int32_t* status = static_cast<int32_t*>(stats);
    CK(cudaMemsetAsync(status, 0, sizeof(int32_t), st));
    float* lg = logits ? logits : reinterpret_cast<float*>(wsp(workspace, L.logits));
    int32_t* blockcnt = reinterpret_cast<int32_t*>(wsp(workspace, L.blockcnt));
    float* blockpsum = reinterpret_cast<float*>(wsp(workspace, L.blockpsum));
    float* blockextra = reinterpret_cast<float*>(wsp(workspace, L.blockextra));
    const int kk = count_slots(*p);
    if (router_fused(p)) {
        CK(launch_route_fused(p->dtype, x, W_r, bias, p->bias_mode, p->gate_mode, kk, p->T, p->d, p->E, p->k, lg,
                              idx, gate, blockcnt, blockpsum, blockextra, nullptr, st));
    } else {
        rc = run_logits(p, x, W_r, lg, L, workspace, status, st);
        if (rc != MOE_OK) return rc;
        CK(launch_select(lg, bias, p->bias_mode, p->gate_mode, kk, p->T, p->E, p->k, idx, gate, blockcnt,
                         blockpsum, blockextra, st));
    }
    ScanArgs sa = {};
    sa.T = p->T; sa.k = p->k; sa.E = p->E; sa.capacity = C; sa.kk = kk;
    sa.blockcnt = blockcnt; sa.blockoff = reinterpret_cast<int32_t*>(wsp(workspace, L.blockoff));
    sa.blockpsum = blockpsum; sa.blockextra = blockextra;
    sa.indptr = reinterpret_cast<int32_t*>(wsp(workspace, L.indptr));
    sa.stats = stats;
    sa.pad = p->pad_rows;
    CK(launch_scan(sa, st));
    return MOE_OK;
}

int moe_route_from_logits(const moe_problem* p, const float* logits, const float* bias, int32_t* idx, float* gate,
                          void* stats, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_problem(p);
    if (rc != MOE_OK) return rc;
    if (!logits || !idx || !gate || !stats) return MOE_ERR_INVALID_ARG;
    if (p->bias_mode != MOE_BIAS_NONE && !bias) return MOE_ERR_INVALID_ARG;
    if (!aligned16(stats)) return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(*p);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int C = capacity_of(p);
    if (p->T == 0) {
        CK(launch_zero_stats(stats, p->E, C, st));
        return MOE_OK;
    }
    CK(cudaMemsetAsync(stats, 0, sizeof(int32_t), st));
    int32_t* blockcnt = reinterpret_cast<int32_t*>(wsp(workspace, L.blockcnt));
    float* blockpsum = reinterpret_cast<float*>(wsp(workspace, L.blockpsum));
    float* blockextra = reinterpret_cast<float*>(wsp(workspace, L.blockextra));
    const int kk = count_slots(*p);
    CK(launch_select(logits, bias, p->bias_mode, p->gate_mode, kk, p->T, p->E, p->k, idx, gate, blockcnt, blockpsum,
                     blockextra, st));
    ScanArgs sa = {};
    sa.T = p->T; sa.k = p->k; sa.E = p->E; sa.capacity = C; sa.kk = kk;
    sa.blockcnt = blockcnt; sa.blockoff = reinterpret_cast<int32_t*>(wsp(workspace, L.blockoff));
    sa.blockpsum = blockpsum; sa.blockextra = blockextra;
    sa.indptr = reinterpret_cast<int32_t*>(wsp(workspace, L.indptr));
    sa.stats = stats;
    sa.pad = p->pad_rows;
    CK(launch_scan(sa, st));
    return MOE_OK;
}

int moe_permute(const moe_problem* p, const void* x, const int32_t* idx, int32_t* pos, int32_t* indptr,
                int32_t* row_token, void* xp, void* stats, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_problem(p);
    if (rc != MOE_OK) return rc;
    if (!idx || !pos || !indptr || !stats) return MOE_ERR_INVALID_ARG;
    if (xp && (!x || !aligned16(x) || !aligned16(xp))) return MOE_ERR_INVALID_ARG;
    if (!aligned16(stats)) return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(*p);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_WORKSPACE;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int C = capacity_of(p);
    if (p->T == 0) {
        CK(launch_zero_stats(stats, p->E, C, st));
        CK(cudaMemsetAsync(indptr, 0, sizeof(int32_t) * (size_t)(p->E + 1), st));
        return MOE_OK;
    }
    CK(cudaMemsetAsync(stats, 0, sizeof(int32_t), st));
    int32_t* blockcnt = reinterpret_cast<int32_t*>(wsp(workspace, L.blockcnt));
    int32_t* blockoff = reinterpret_cast<int32_t*>(wsp(workspace, L.blockoff));
    const int kk = count_slots(*p);
    CK(launch_hist(idx, p->T, p->k, kk, p->E, blockcnt, st));
    ScanArgs sa = {};
    sa.T = p->T; sa.k = p->k; sa.E = p->E; sa.capacity = C; sa.kk = kk;
    sa.blockcnt = blockcnt; sa.blockoff = blockoff; sa.blockpsum = nullptr;
    sa.indptr = indptr; sa.stats = stats;
    sa.pad = p->pad_rows;
    CK(launch_scan(sa, st));
    CK(launch_permute_gather(p->dtype, x, idx, blockoff, indptr, p->T, p->d, p->E, p->k, kk, C, pos, row_token, xp,
                             st));
    if (p->pad_rows > 0)
        CK(launch_pad_fill(p->dtype, indptr, stats, p->E, p->d, xp, row_token, p->pad_rows, st));
    return MOE_OK;
}

int moe_experts(const moe_problem* p, const void* xp, const int32_t* indptr, const void* W1, const void* W3,
                const void* W2, const void* x, const void* Ws1, const void* Ws3, const void* Ws2, void* o, void* s,
                void* stats, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = check_problem(p);
    if (rc != MOE_OK) return rc;
    const bool shared = p->d_ff_shared > 0;
    if (!xp || !indptr || !W1 || !W3 || !W2 || !o) return MOE_ERR_INVALID_ARG;
    if (shared && (!x || !Ws1 || !Ws3 || !Ws2 || !s)) return MOE_ERR_INVALID_ARG;
    for (const void* q : {xp, W1, W3, W2, (const void*)o})
        if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (shared)
        for (const void* q : {x, Ws1, Ws3, Ws2, (const void*)s})
            if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    const Layout L = make_layout(*p);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_WORKSPACE;
    if (p->T == 0) return MOE_OK;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* status = stats ? static_cast<int32_t*>(stats)
                            : reinterpret_cast<int32_t*>(wsp(workspace, L.blockcnt));
    CK(cudaMemsetAsync(status, 0, sizeof(int32_t), st));
    int32_t* tiles13 = reinterpret_cast<int32_t*>(wsp(workspace, L.tiles13));
    int32_t* tiles2 = reinterpret_cast<int32_t*>(wsp(workspace, L.tiles2));
    int tile_m, nt13, nt2, nt13s, nt2s;
    schedule_sizes(p, tile_m, nt13, nt2, nt13s, nt2s);
    const StageSplit sp = stage_split(p, L, workspace, status);
    CK(launch_schedule(indptr, p->E, p->T, shared ? 1 : 0, tile_m, nt13, nt2, nt13s, nt2s, tiles13, tiles2,
                       sp.sched, st));
    void* h = wsp(workspace, L.h);
    void* hs = shared ? wsp(workspace, L.hs) : nullptr;
    return run_experts(p, xp, indptr, tiles13, tiles2, W1, W3, W2, x, Ws1, Ws3, Ws2, h, hs, o, s, status, st,
                       sp.part13, sp.part2, sp.sem13, sp.sem2);
}

// Shared prologue of the expert-stage entry points: the workspace check and
// the status word and tile schedule buffers.
static int expert_stage_setup(const moe_problem* p, void* stats, void* workspace, size_t workspace_bytes,
                              int32_t** status, int32_t** tiles13, int32_t** tiles2) {
    const Layout L = make_layout(*p);
    if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return MOE_ERR_WORKSPACE;
    *status = stats ? static_cast<int32_t*>(stats) : reinterpret_cast<int32_t*>(wsp(workspace, L.blockcnt));
    *tiles13 = reinterpret_cast<int32_t*>(wsp(workspace, L.tiles13));
    *tiles2 = reinterpret_cast<int32_t*>(wsp(workspace, L.tiles2));
    return MOE_OK;
}

int moe_expert_up(const moe_problem* p, const void* xp, const int32_t* indptr, const void* W1, const void* W3,
                  const void* x, const void* Ws1, const void* Ws3, void* h, void* hs, void* stats, void* workspace,
                  size_t workspace_bytes, void* stream) {
    int rc = check_problem(p);
    if (rc != MOE_OK) return rc;
    const bool shared = p->d_ff_shared > 0;
    if (!xp || !indptr || !W1 || !W3 || !h) return MOE_ERR_INVALID_ARG;
    if (shared && (!x || !Ws1 || !Ws3 || !hs)) return MOE_ERR_INVALID_ARG;
    for (const void* q : {xp, W1, W3, (const void*)h})
        if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (shared)
        for (const void* q : {x, Ws1, Ws3, (const void*)hs})
            if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t *status, *tiles13, *tiles2;
    rc = expert_stage_setup(p, stats, workspace, workspace_bytes, &status, &tiles13, &tiles2);
    if (rc != MOE_OK) return rc;
    if (p->T == 0) return MOE_OK;
    CK(cudaMemsetAsync(status, 0, sizeof(int32_t), st));
    int tile_m, nt13, nt2, nt13s, nt2s;
    schedule_sizes(p, tile_m, nt13, nt2, nt13s, nt2s);
    const StageSplit sp = stage_split(p, make_layout(*p), workspace, status);
    CK(launch_schedule(indptr, p->E, p->T, shared ? 1 : 0, tile_m, nt13, nt2, nt13s, nt2s, tiles13, tiles2,
                       sp.sched, st));
    return run_up(p, xp, indptr, tiles13, W1, W3, x, Ws1, Ws3, h, shared ? hs : nullptr, status, st, sp.part13,
                  sp.sem13);
}

int moe_expert_down(const moe_problem* p, const void* h, const int32_t* indptr, const void* W2, const void* hs,
                    const void* Ws2, void* o, void* s, void* stats, void* workspace, size_t workspace_bytes,
                    void* stream) {
    int rc = check_problem(p);
    if (rc != MOE_OK) return rc;
    const bool shared = p->d_ff_shared > 0;
    if (!h || !indptr || !W2 || !o) return MOE_ERR_INVALID_ARG;
    if (shared && (!hs || !Ws2 || !s)) return MOE_ERR_INVALID_ARG;
    for (const void* q : {h, W2, (const void*)o})
        if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (shared)
        for (const void* q : {hs, Ws2, (const void*)s})
            if (!aligned16(q)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t *status, *tiles13, *tiles2;
    rc = expert_stage_setup(p, stats, workspace, workspace_bytes, &status, &tiles13, &tiles2);
    if (rc != MOE_OK) return rc;
    if (p->T == 0) return MOE_OK;
    CK(cudaMemsetAsync(status, 0, sizeof(int32_t), st));
    int tile_m, nt13, nt2, nt13s, nt2s;
    schedule_sizes(p, tile_m, nt13, nt2, nt13s, nt2s);
    const StageSplit sp = stage_split(p, make_layout(*p), workspace, status);
    CK(launch_schedule(indptr, p->E, p->T, shared ? 1 : 0, tile_m, nt13, nt2, nt13s, nt2s, tiles13, tiles2,
                       sp.sched, st));
    return run_down(p, h, indptr, tiles2, W2, shared ? hs : nullptr, Ws2, o, shared ? s : nullptr, status, st,
                    sp.part2, sp.sem2);
}

int moe_combine(const moe_problem* p, const void* o, const int32_t* pos, const float* gate, const void* s, void* out,
                void* stream) {
    int rc = check_problem(p);
    if (rc != MOE_OK) return rc;
    if (!o || !pos || !gate || !out) return MOE_ERR_INVALID_ARG;
    if (!aligned16(o) || !aligned16(out) || (s && !aligned16(s))) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    CK(launch_combine(p->dtype, o, pos, gate, s, out, p->T, p->d, p->k, (int)permuted_rows(*p), nullptr, st));
    return MOE_OK;
}

}  // extern "C"
