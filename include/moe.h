/*
 * moe.h - C ABI of the B200 (sm_100a) forward pass of one sparse
 * Mixture-of-Experts layer.
 *
 * The pass (citations name the source page and its section):
 *   1. router logits z = W_r^T x            ("Week 2 Day 2: Mixture of Experts", §1.3)
 *   2. top-k of a selection key, optionally z + b or softmax(z) + b; gates are
 *      the softmax over the k selected raw logits   (same page §1.3, §4.2;
 *      "Stanford CS336 Lecture 04", §2.3.3c)
 *   3. expert histogram, expert-major prefix sum, capacity truncation and
 *      permutation of token rows       ("Lecture 21 · LLM: Mixture-of-Experts", §3.3, §3.5)
 *   4. grouped GEMM over E SwiGLU experts, Z = GroupGemm(data, indptr, weights)
 *                                       (Lecture 21, §3.3; Week 2 Day 2, §2.1)
 *   5. un-permute and gate-weighted sum (Lecture 21, §3.2 step 4), plus an
 *      always-on shared expert           (Week 2 Day 2, §4.1)
 *   6. load statistics f, P, L_aux = E sum f P (Week 2 Day 2, §3.2)
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major,
 *    16-byte aligned. The library allocates no device memory and keeps no
 *    per-call state; scratch lives in a caller-provided workspace.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*, NULL
 *    = legacy default stream). Results, including the status word of the
 *    statistics block, are valid after the stream is synchronised.
 *  - Return value: MOE_OK, or an MOE_ERR_* code for a host-side rejection
 *    (nothing was launched) or a launch failure. Device-side failures (a
 *    bounded wait that ran out) are reported in moe_stats.status.
 *  - Element type of activations and expert weights: MOE_DTYPE_BF16 (bf16
 *    storage, fp32 accumulation, tcgen05 tensor cores) or MOE_DTYPE_F32
 *    (fp32 storage and arithmetic on CUDA cores). Router math is fp32 for
 *    both; gates and the bias are fp32.
 *  - Inputs are assumed finite; NaN handling is unspecified.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- error codes ------------------------------------------------------- */
#define MOE_OK              0
#define MOE_ERR_INVALID_ARG 1  /* null pointer, bad size, k<1, k>E, misaligned pointer */
#define MOE_ERR_UNSUPPORTED 2  /* shape/dtype combination this build does not run */
#define MOE_ERR_WORKSPACE   3  /* workspace missing or smaller than moe_workspace_size() */
#define MOE_ERR_CUDA        4  /* a CUDA launch or driver call failed */
#define MOE_ERR_TIMEOUT     5  /* device status only: a bounded wait gave up */
#define MOE_ERR_BOUNDS      6  /* device status only, debug build (libmoe_debug.so): an index
                                  out of its buffer was found and the access skipped */

/* ---- enums -------------------------------------------------------------- */
#define MOE_DTYPE_F32  0
#define MOE_DTYPE_BF16 1

/* Selection key of the top-k (gates always use the raw logits z):
 * NONE : key = z                       (Week 2 Day 2, §1.3)
 * LOGIT: key = z + b                   (Week 2 Day 2, §4.2; tutorial route())
 * PROB : key = softmax(z) + b          (CS336 Lecture 04, §2.3.3c)          */
#define MOE_BIAS_NONE  0
#define MOE_BIAS_LOGIT 1
#define MOE_BIAS_PROB  2

/* Gate of a selected expert:
 * SELECTED: softmax over the k selected raw logits (Week 2 Day 2, §1.3)
 * FULL    : full-softmax probability of the expert, not renormalised
 *           (the Switch top-1 gate; Lecture 21, §2.5)                     */
#define MOE_GATE_SELECTED 0
#define MOE_GATE_FULL     1

/* Order in which pairs claim an expert's capacity (and rows):
 * TOKEN: token order inside each expert (Lecture 21, §3.3 prefix sum)
 * SLOT : every token's first choice before any second choice, then token
 *        order (GShard's Algorithm 1; Lecture 21, §3.5). Requires E*k <= 4096. */
#define MOE_DROP_TOKEN 0
#define MOE_DROP_SLOT  1

/* Limits of this build. */
#define MOE_MAX_E 512
#define MOE_MAX_K 16

/* ---- problem description ----------------------------------------------- */
typedef struct moe_problem {
    int32_t T;                /* tokens (rows of x), >= 0                                 */
    int32_t d;                /* model width                                              */
    int32_t d_ff;             /* hidden width of a routed expert                          */
    int32_t E;                /* routed experts, 1..MOE_MAX_E                             */
    int32_t k;                /* experts per token, 1..min(E, MOE_MAX_K)                  */
    float   capacity_factor;  /* C = ceil(cf*T*k/E) pairs per expert; <= 0: no limit     */
    int32_t dtype;            /* MOE_DTYPE_*                                              */
    int32_t bias_mode;        /* MOE_BIAS_*                                               */
    int32_t d_ff_shared;      /* hidden width of the always-on shared expert, 0 = none    */
    int32_t gate_mode;        /* MOE_GATE_*  (0 = selected softmax)                       */
    int32_t drop_order;       /* MOE_DROP_*  (0 = token order)                            */
    int32_t pad_rows;         /* 0, 64 or 128: pad every expert's kept rows to a multiple
                                 of this inside the permutation (the MegaBlocks layout,
                                 "Lecture 21 · LLM: Mixture-of-Experts" §3.6); padding rows
                                 are zero in Xp and belong to no token. 0 = dense rows.  */
    int32_t train;            /* 1: moe_forward also keeps the experts' gate and up
                                 pre-activations (W1 x, W3 x) in the workspace for
                                 moe_backward (bf16 only); 0: inference               */
} moe_problem;

/* ---- statistics block (device memory, moe_stats_size(E) bytes) ----------
 * A fixed header followed by four per-expert arrays:
 *     int32_t counts[E]  pairs routed to e before capacity (c_e)
 *     int32_t kept[E]    pairs kept after capacity
 *     float   P[E]       mean full-softmax router probability of e
 *     float   f[E]       c_e / (T k)
 * L_aux = E * sum_e f_e P_e (the coefficient alpha is left to the caller;
 * uniform routing gives 1). Reductions run in a fixed order, so repeated
 * calls on the same inputs give bit-identical statistics.               */
typedef struct moe_stats {
    int32_t status;        /* MOE_OK, or MOE_ERR_TIMEOUT from a device-side bounded wait */
    int32_t capacity;      /* C, or -1 when unlimited                                     */
    int32_t rows;          /* R = sum_e kept_e (kept pairs; with pad_rows the permuted
                              buffer holds indptr[E] >= R rows, the rest zero padding)   */
    int32_t dropped;       /* sum_e (c_e - kept_e)                                        */
    int32_t max_count;     /* max_e c_e                                                   */
    float   l_aux;         /* E * sum_e f_e P_e                                           */
    float   max_over_mean; /* max_e c_e / (T k / E)                                       */
    float   z_loss;        /* (1/T) sum_t (log sum_e exp z_{t,e})^2 (Week 2 Day 2, §3.4)  */
    float   entropy;       /* mean over tokens of -sum_e p log p    (W11 routing, §5)     */
    float   top_gap;       /* mean over tokens of p_(1) - p_(2)     (W11 routing, §5)     */
    int32_t reserved[2];
} moe_stats;

#define MOE_STATS_COUNTS(base, E) ((int32_t*)((char*)(base) + sizeof(moe_stats)))
#define MOE_STATS_KEPT(base, E)   ((int32_t*)((char*)(base) + sizeof(moe_stats)) + (E))
#define MOE_STATS_P(base, E)      ((float*)((int32_t*)((char*)(base) + sizeof(moe_stats)) + 2 * (E)))
#define MOE_STATS_F(base, E)      ((float*)((int32_t*)((char*)(base) + sizeof(moe_stats)) + 3 * (E)))

/* Bytes of the statistics block for E experts (48-byte header + 16 E). */
size_t moe_stats_size(int32_t E);

/* ---- workspace ---------------------------------------------------------
 * Scratch of moe_forward and of the stage entry points. The caller allocates
 * moe_workspace_size(p) bytes of device memory (256-byte aligned) and keeps
 * it alive until the stream has finished the call. Its contents need no
 * initialisation. moe_workspace_layout() gives byte offsets of the
 * intermediates that moe_forward leaves in it, for inspection:           */
typedef struct moe_workspace_layout_t {
    size_t idx;        /* int32 [T, k]  selected experts, descending key            */
    size_t gate;       /* fp32  [T, k]  gates                                         */
    size_t pos;        /* int32 [T, k]  permuted row of (t, j), -1 = dropped          */
    size_t indptr;     /* int32 [E+1]   CSR row offsets over kept rows                */
    size_t row_token;  /* int32 [Rmax]  token of each permuted row, -1 on padding     */
    size_t logits;     /* fp32  [T, E]  router logits                                 */
    size_t xp;         /* dtype [Rmax, d]     permuted activations (first indptr[E])  */
    size_t h;          /* dtype [Rmax, d_ff]  SwiGLU hidden rows                      */
    size_t o;          /* dtype [Rmax, d]     expert outputs, permuted order          */
    size_t hs;         /* dtype [T, d_ff_shared]  shared-expert hidden rows           */
    size_t s;          /* dtype [T, d]        shared-expert output                    */
    size_t ab;         /* dtype [Rmax, 2*d_ff] with train: per 128 hidden units, 128
                          gate pre-activations then the 128 up pre-activations   */
    size_t total;      /* = moe_workspace_size(p)                                    */
} moe_workspace_layout_t;

size_t moe_workspace_size(const moe_problem* p);
int    moe_workspace_layout(const moe_problem* p, moe_workspace_layout_t* out);

/* Rmax: rows a permuted buffer (xp, h, o, row_token) must hold for p:
 * T*k, plus E*(pad_rows-1) when pad_rows > 0; 0 when p is invalid. */
int32_t moe_permuted_rows(const moe_problem* p);

/* ---- the whole layer ----------------------------------------------------
 * moe_forward: out[t] = sum_{j<k, kept} gate[t,j] * FFN_{idx[t,j]}(x[t]) + FFN_shared(x[t]).
 *   x     [T, d]          dtype
 *   W_r   [d, E]          dtype (z = W_r^T x, Week 2 Day 2 §1.3)
 *   bias  [E]             fp32, required unless bias_mode == MOE_BIAS_NONE
 *   W1,W3 [E, d_ff, d]    dtype (nn.Linear layout: out x in)
 *   W2    [E, d, d_ff]    dtype
 *   Ws1,Ws3 [d_ff_shared, d], Ws2 [d, d_ff_shared]  dtype; NULL when d_ff_shared == 0
 *   out   [T, d]          dtype, written fully (a fully dropped token gets 0)
 *   stats moe_stats_size(E) bytes of device memory, written fully
 * bf16 also requires d % 64 == 0, d_ff % 64 == 0, d_ff_shared % 64 == 0;
 * f32 requires d % 4 == 0 and d_ff % 4 == 0. Otherwise MOE_ERR_UNSUPPORTED. */
int moe_forward(const moe_problem* p,
                const void* x, const void* W_r, const float* bias,
                const void* W1, const void* W3, const void* W2,
                const void* Ws1, const void* Ws3, const void* Ws2,
                void* out, void* stats,
                void* workspace, size_t workspace_bytes, void* stream);

/* ---- stage entry points (the same kernels moe_forward launches) --------- */

/* Router: logits (fp32, accumulated in fp32), selection key, top-k with the
 * lowest index winning ties, gates, and the statistics counts/P/f/L_aux
 * (kept/rows/dropped assume the capacity of p).
 * logits [T, E] fp32 may be NULL. idx [T, k] int32, gate [T, k] fp32. */
int moe_route(const moe_problem* p, const void* x, const void* W_r, const float* bias,
              int32_t* idx, float* gate, float* logits, void* stats,
              void* workspace, size_t workspace_bytes, void* stream);

/* Routing from given fp32 logits [T, E] (selection, gates, statistics). */
int moe_route_from_logits(const moe_problem* p, const float* logits, const float* bias,
                          int32_t* idx, float* gate, void* stats,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Permutation (Lecture 21 §3.3 and §3.5): per-expert histogram, expert-major
 * exclusive scan, rank of each pair in token order, capacity truncation,
 * and gather of token rows: xp[pos[t,j]] = x[t] for kept pairs.
 *   idx [T, k] int32 in; pos [T, k], indptr [E+1], row_token [Rmax] int32 out;
 *   xp [Rmax, d] dtype out (rows >= indptr[E] untouched).
 * With pad_rows > 0 (§3.6) indptr counts every expert's kept rows rounded up
 * to a multiple of pad_rows; the padding rows after an expert's kept rows
 * are written as zeros in xp and -1 in row_token.
 * stats receives counts/kept/capacity/rows/dropped/max_count; P, f and
 * l_aux are left as they are. */
int moe_permute(const moe_problem* p, const void* x, const int32_t* idx,
                int32_t* pos, int32_t* indptr, int32_t* row_token, void* xp, void* stats,
                void* workspace, size_t workspace_bytes, void* stream);

/* Expert FFNs over the permuted rows (Lecture 21 §3.3, Z = GroupGemm(data,
 * indptr, weights)): for every expert e and row r in [indptr[e], indptr[e+1]):
 *   o[r] = W2_e (SiLU(W1_e xp[r]) * (W3_e xp[r]))
 * and, when d_ff_shared > 0, s[t] = Ws2 (SiLU(Ws1 x[t]) * (Ws3 x[t])).
 *   xp [Rmax, d], o [Rmax, d] (rows >= indptr[E] untouched), x [T, d], s [T, d].
 * indptr is read on the device; the host never waits for it; its entries must
 * be non-decreasing with indptr[0] = 0 and indptr[E] <= Rmax.
 * stats (may be NULL): only the status word is written (MOE_OK, or
 * MOE_ERR_TIMEOUT if a bounded wait of the tensor-core kernel gave up). */
int moe_experts(const moe_problem* p, const void* xp, const int32_t* indptr,
                const void* W1, const void* W3, const void* W2,
                const void* x, const void* Ws1, const void* Ws3, const void* Ws2,
                void* o, void* s, void* stats,
                void* workspace, size_t workspace_bytes, void* stream);

/* The two halves of moe_experts, for per-stage timing and inspection:
 *   moe_expert_up:   h[r] = SiLU(W1_e xp[r]) * (W3_e xp[r])      h  [Rmax, d_ff]
 *                    hs[t] = SiLU(Ws1 x[t]) * (Ws3 x[t])          hs [T, d_ff_shared]
 *   moe_expert_down: o[r] = W2_e h[r];  s[t] = Ws2 hs[t]          o [Rmax, d], s [T, d]
 * Same indptr rules and workspace as moe_experts (the tile schedule is
 * rebuilt from indptr by each call). */
int moe_expert_up(const moe_problem* p, const void* xp, const int32_t* indptr,
                  const void* W1, const void* W3, const void* x, const void* Ws1, const void* Ws3,
                  void* h, void* hs, void* stats,
                  void* workspace, size_t workspace_bytes, void* stream);
int moe_expert_down(const moe_problem* p, const void* h, const int32_t* indptr, const void* W2,
                    const void* hs, const void* Ws2, void* o, void* s, void* stats,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Un-permute and mix (Lecture 21 §3.2 step 4): for every token, in slot order
 *   out[t] = sum_{j<k, pos[t,j] >= 0} gate[t,j] * o[pos[t,j]]  (+ s[t] if s != NULL)
 * accumulated in fp32 and rounded once; no atomics. */
int moe_combine(const moe_problem* p, const void* o, const int32_t* pos, const float* gate,
                const void* s, void* out, void* stream);

/* ---- allocation-free permutation ----------------------------------------
 * Not a step of the notes (they have no counterpart): a variant of
 * moe_permute for callers that cannot allocate device memory where they run
 * the layer, e.g. a plugin of an inference runtime that owns all device
 * memory and passes in only the input and output buffers, or a
 * latency-critical loop in which cudaMalloc could block or synchronise the
 * device. It takes no workspace: the scratch of the permutation (per-chunk
 * expert counts and their scan) lives in a fixed 1 MiB array inside the
 * library, which every GPU that loads the library holds until the process
 * exits. Arguments, outputs and results are those of moe_permute.
 *  - Limit: E * kk * ceil(T / 32) <= 131072, with kk = k under
 *    MOE_DROP_SLOT and 1 otherwise (e.g. T <= 16384 at E = 256 with the
 *    token drop order); larger problems return MOE_ERR_UNSUPPORTED before
 *    anything is launched. The problem checks and error codes are otherwise
 *    those of moe_permute.
 *  - The first call on a device looks up the array's device address on that
 *    device (the device must be current); make that first call before any
 *    stream capture. If the lookup fails the call returns MOE_ERR_CUDA and
 *    the next call on that device tries again.
 *  - All calls share the one array and it keeps the last call's contents
 *    (every entry a call reads is written earlier in the same call). Calls
 *    that overlap on the GPU (different streams, or different host threads,
 *    on the same device) race on it: serialise them.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
/* (pad_rows must be 0 here: MOE_ERR_UNSUPPORTED otherwise.) */
int moe_permute_noalloc(const moe_problem* p, const void* x, const int32_t* idx,
                        int32_t* pos, int32_t* indptr, int32_t* row_token, void* xp, void* stats,
                        void* stream);

/* ---- backward pass ------------------------------------------------------
 * Gradients of L = sum_t <dy_t, y_t> + alpha * L_aux + beta * L_z, where y is
 * the output of the moe_forward call that filled `workspace` and `stats`
 * (same p, same inputs, nothing run on the workspace since), L_aux =
 * E sum_e f_e P_e with the counts f frozen (Week 2 Day 2 §3.2: its gradient
 * reaches the router through P only) and L_z the router z-loss (§3.4). The
 * expert selection and the capacity drops carry no gradient; the selection
 * bias gets none.
 * Requires p->train = 1 (the forward kept the gate/up pre-activations) and
 * p->pad_rows = 64 or 128 (the weight-gradient GEMMs contract over each
 * expert's rows, which padding keeps in whole 64-row blocks), bf16 and
 * E % 8 == 0; otherwise MOE_ERR_UNSUPPORTED.
 *   dy [T, d] bf16 in; dx [T, d] bf16 out;
 *   dW_r [d, E] fp32, dW1 and dW3 [E, d_ff, d] fp32, dW2 [E, d, d_ff] fp32
 *   out, each written fully (an expert without rows gets zeros);
 *   with d_ff_shared > 0: Ws1, Ws3, Ws2 as in moe_forward, and dWs1, dWs3
 *   [d_ff_shared, d], dWs2 [d, d_ff_shared] fp32 out (NULL otherwise);
 *   stats: the forward's block (f is read; the status word gets
 *   MOE_ERR_TIMEOUT if a bounded wait of a tensor-core kernel gave up);
 *   bwd_workspace: moe_backward_workspace_size(p) bytes, 256-byte aligned,
 *   no initialisation needed.
 * Reductions run in a fixed order: repeated calls give identical results. */
size_t moe_backward_workspace_size(const moe_problem* p);
int moe_backward(const moe_problem* p, const void* x, const void* W_r, const void* W1, const void* W3,
                 const void* W2, const void* Ws1, const void* Ws3, const void* Ws2,
                 const void* dy, float alpha, float beta,
                 void* dx, float* dW_r, float* dW1, float* dW3, float* dW2,
                 float* dWs1, float* dWs3, float* dWs2, void* stats,
                 const void* workspace, size_t workspace_bytes,
                 void* bwd_workspace, size_t bwd_workspace_bytes, void* stream);

/* Auxiliary-loss-free balancing step (Lecture 21 §2.4, DeepSeek-V3): for
 * every expert, bias[e] -= gamma if its count c_e in `stats` is above the
 * mean load T*k/E, bias[e] += gamma if below, unchanged if equal (decided
 * exactly, as the sign of c_e*E - T*k). bias [E] fp32 device memory, updated
 * in place on the stream. */
int moe_bias_update(const moe_problem* p, const void* stats, float gamma, float* bias, void* stream);

/* Human-readable text of an MOE_* code (static storage). */
const char* moe_error_string(int code);

/* Number of streaming multiprocessors the library sizes persistent grids for
 * on the current device, or -1 on error. */
int moe_device_sm_count(void);

/* Failure detection (no step of the notes): every mbarrier wait inside the
 * tensor-core kernels gives up after `ns` nanoseconds of wall-clock time,
 * records MOE_ERR_TIMEOUT in the status word of the call's statistics block,
 * lets the copies and MMAs it already started land (a separate, fixed 2 s
 * drain limit), frees its tensor memory and returns, so a stalled pipeline
 * surfaces as an error the host reads instead of a hung GPU. ns <= 0 restores
 * the default of 2 s. The setting is process-wide and applies to launches
 * made after the call; the previous value is returned. A limit far below a
 * kernel's normal run time makes its calls fail with MOE_ERR_TIMEOUT (their
 * outputs are then unspecified); the next call with a normal limit is
 * unaffected. */
long long moe_set_wait_limit(long long ns);

/* Which grouped-GEMM kernel moe_forward and the expert stages use for p:
 * MOE_GEMM_SINGLE (one CTA per 128-row tile), MOE_GEMM_PAIR (CTA pairs,
 * 256-row tiles), MOE_GEMM_GRID_SPLIT (single-CTA tiles, groups of at most
 * 128 rows as operand-swapped tiles on their own CTAs; MOE_SMALL_CTAS
 * below), MOE_GEMM_SPLIT_K
 * (decode-sized batches: K split over CTAs), MOE_GEMM_SIMT (fp32, CUDA
 * cores), MOE_GEMM_INTERLEAVED (single-CTA tiles; with 32 or more experts
 * averaging fewer than 512 rows, the tiles of the groups of at most 128
 * rows are spread evenly through the others' and load their weights with an
 * evict-first L2 policy), MOE_GEMM_GEMV (bf16 batches of at most 8
 * permuted rows and no shared expert: GEMM 1/3 + SwiGLU as weight-streaming
 * GEMVs, the weights copied through shared memory, the K range split over
 * the warps of each CTA, each CTA one equal, contiguous range of 8-column
 * output groups; GEMM 2 as split-K tiles); a negative MOE_ERR_* code if p is
 * invalid. Host only. */
#define MOE_GEMM_SINGLE      0
#define MOE_GEMM_PAIR        1
#define MOE_GEMM_GRID_SPLIT  2
#define MOE_GEMM_SPLIT_K     3
#define MOE_GEMM_SIMT        4
#define MOE_GEMM_INTERLEAVED 5
#define MOE_GEMM_GEMV        6
int moe_gemm_variant(const moe_problem* p);

/* Which router a call uses for p ("Week 2 Day 2: Mixture of Experts" §1.3:
 * z = W_r^T x, top-k, gates; the forms differ in kernels, not in results
 * beyond the order of the fp32 sums). forward != 0: the router moe_forward
 * uses; forward == 0: the one moe_route uses (never MOE_ROUTER_SMALL).
 *   MOE_ROUTER_SMALL      decode-sized batches in moe_forward: partial
 *                         logits, then one block that selects, counts,
 *                         ranks and gathers;
 *   MOE_ROUTER_FUSED_MMA  bf16, at most 63 experts, W_r^T of eight experts
 *                         within the kernel's shared memory (d <= 5344):
 *                         logits on the warp-level MMA (bf16 products, fp32
 *                         sums) and the selection in one kernel;
 *   MOE_ROUTER_FUSED_FMA  the same kernel layout with fp32 FMAs: fp32 up to
 *                         64 experts and d <= 5120, bf16 rows past the MMA
 *                         form's budget (d <= 10240), or MOE_ROUTER_MMA=0;
 *   MOE_ROUTER_TENSOR     wide bf16 routers (E >= 64, E % 32 == 0): W_r
 *                         transposed, logits as a tensor-core GEMM (fp32
 *                         out), then the selection kernel;
 *   MOE_ROUTER_SIMT       everything else: W_r transposed, logits on CUDA
 *                         cores, then the selection kernel.
 * A negative MOE_ERR_* code if p is invalid. Host only. */
#define MOE_ROUTER_SMALL     0
#define MOE_ROUTER_FUSED_MMA 1
#define MOE_ROUTER_FUSED_FMA 2
#define MOE_ROUTER_TENSOR    3
#define MOE_ROUTER_SIMT      4
int moe_router_variant(const moe_problem* p, int forward);

/* Debug build. The library also builds as libmoe_debug.so (compiled with
 * MOE_DEBUG), with the same entry points and results, plus device-side bounds
 * checks that record MOE_ERR_BOUNDS in the call's status word and skip the
 * access instead of faulting: the group offsets handed to the expert stages
 * (non-decreasing, within the permuted rows; a violation empties the tile
 * schedule, so no tile runs; the GEMV kernel skips the groups whose offsets
 * are out of range, and so does the release build), every output row a
 * grouped GEMM stores, and
 * every permuted row the combine reads (moe_forward's status word; the
 * standalone moe_combine has none, so it only skips). The Python binding
 * loads it when MOE_LIBRARY=debug. */

/* Kernel-selection overrides, read once per process from the environment
 * (for measurement and tests; results are the same either way, up to the
 * order of the fp32 sums):
 *   MOE_CTA_PAIR=0   the grouped GEMMs never use CTA pairs (256-row tiles on
 *                    two SMs); by default they do when the experts average
 *                    at least 512 rows (bf16 inference, no split-K).
 *   MOE_SMALL_CTAS=n with 32 or more experts and fewer than 512 rows per
 *                    expert on average, the first n > 0 CTAs run the groups
 *                    of at most 128 rows as operand-swapped tiles beside the
 *                    larger groups (a grid split; measured no faster on the
 *                    DeepSeek-shaped layer).
 *   MOE_INTERLEAVE=1 for the same shapes, the interleaved two-class order
 *                    (MOE_GEMM_INTERLEAVED above; also measured no faster
 *                    there). Without either, one order in expert order.
 *   MOE_GEMV=0       decode-sized batches use the split-K tensor-core tiles
 *                    (MOE_GEMM_SPLIT_K) for GEMM 1/3 too.
 *   MOE_GEMV_ROWS=n  the GEMV path takes batches of at most n permuted rows
 *                    (default and largest 8).
 *   MOE_ROUTER_MMA=0 the fused bf16 router (up to 63 experts) forms its
 *                    logits with fp32 FMAs instead of the warp-level MMA
 *                    (bf16 products, fp32 sums; the default where W_r^T of
 *                    eight experts fits its shared memory, d <= 5344). */

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
