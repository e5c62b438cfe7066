// Decode-sized grouped GEMM 1/3 + SwiGLU as weight-streaming GEMVs (bf16,
// sm_100a).
//
// With a few permuted rows in the pass ("W11 · MoE routing and parallel
// cost" §5 and "Lecture 21 · LLM: Mixture-of-Experts" §3.1: a decode step
// reads every active expert's weights once and does almost no math per
// byte), each active expert has a handful of rows, and GEMM 1/3 is bound by
// the stream of W1 and W3 alone. This kernel streams those weights with
// 16-byte asynchronous copies (cp.async) into shared memory, 256 contiguous
// bytes of a weight row per half-warp, and does the multiply on the
// warp-level MMA (m16n8k16, bf16 in, fp32 accumulate) as a dot-product
// engine, reading its operand fragments back from shared memory.
//
// Work split. An output group is 8 consecutive hidden units n of one active
// expert: rows n0..n0+7 of W1 and of W3 (the MMA's 16 A rows: W1 rows on
// top, W3 rows below). The groups of all active experts, in expert order,
// are split into one contiguous, equal range per CTA. A weight row's K range is cut into items of kGvItemK elements; the
// CTA's items (group-major) are dealt to its kGvWarps "K warps" in turn, so
// the warps get the same number of items to within one. Each K warp keeps
// its own ring of item buffers filled ahead of its MMAs, and leaves one
// partial tile per group; a reducer warp sums the K warps' partial tiles in
// a fixed order (the result does not depend on timing), applies SiLU(a)·b
// and stores bf16 hidden rows. K warps and reducer hand partial
// tiles over through a ring of shared-memory slots guarded by named barriers
// (hardware barriers: nothing spins).
//
// Operand mapping. For a 32-element chunk of K starting at kb, lane (g =
// lane/4, t = lane%4) takes the 8 values at kb + 8t of weight row g (and of
// row g + 8's source, W3) and of token row g of the expert's rows; values 0-3
// feed one MMA (its k-pairs t and t+4), values 4-7 a second. A and B use the
// same assignment, so every k of the chunk is multiplied exactly once; the
// order of k inside an MMA differs from memory order, which a dot product
// does not see. In shared memory, 16-byte piece p of buffer row r sits at
// position p ^ (r & 7) of the row, so the fragment reads (8 rows, the same
// pieces) fall in different banks.

#include "warp_mma.cuh"

namespace moe {
namespace {

constexpr int kGvWarps = 15;                       // K warps per CTA (16 warps in all: 4 per SM sub-partition)
constexpr int kGvThreads = (kGvWarps + 1) * 32;    // + the reducer warp
constexpr int kGvRing = 4;                         // partial-tile slots
constexpr int kGvRows = 8;                         // output columns per group
constexpr int kGvItemK = 128;                      // K elements of one item (256 bytes of a row)
constexpr int kGvChunks = kGvItemK / 32;           // 32-element MMA chunks per item
constexpr int kGvBufBytes = 16 * kGvItemK * 2;     // one item buffer: 16 rows

struct GemvParams {
    const int32_t* indptr;    // [E+1] row offsets of the experts' groups
    int E;
    const __nv_bfloat16* A;   // [rows_max, K] permuted rows
    const __nv_bfloat16* B0;  // [E, N, K]: W1
    const __nv_bfloat16* B1;  // [E, N, K]: W3
    __nv_bfloat16* out;       // [rows_max, N]
    int N, K;
    int rows_max;
    int32_t* status;          // debug build: where an invalid offset is recorded
};

__device__ __forceinline__ uint4 ld_cached(const __nv_bfloat16* p) {
    return __ldg(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ void bar_sync(int id) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "n"(kGvThreads) : "memory");
}
__device__ __forceinline__ void bar_arrive(int id) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "n"(kGvThreads) : "memory");
}
// named barrier ids: 0 is __syncthreads; slot s is full at 1 + s, free at
// 1 + kGvRing + s
__device__ __forceinline__ int bar_full(int s) { return 1 + s; }
__device__ __forceinline__ int bar_free(int s) { return 1 + kGvRing + s; }

__device__ __forceinline__ float silu(float a) { return a / (1.f + __expf(-a)); }

// Item buffers per K warp. Two keep the shared memory at 154 KB, which
// leaves L1 room for the token rows every item reads; a third buffer per
// warp (215 KB) made the token rows miss in L1 at four rows per expert and
// was slower from four tokens up.
constexpr int kGvStages = 2;
// Token rows per group: one 8-column MMA tile.
constexpr int NT = 1;
constexpr size_t kGvSmemBytes = (size_t)kGvWarps * kGvStages * kGvBufBytes + (size_t)kGvRing * kGvWarps * 32 * NT * 16;

__global__ void __launch_bounds__(kGvThreads, 1) gemv_swiglu_kernel(GemvParams p) {
    constexpr int NS = kGvStages;
    extern __shared__ __align__(128) uint8_t gv_smem[];
    // [kGvWarps][NS] item buffers, then [kGvRing][kGvWarps][32] partial tiles
    float4* part = reinterpret_cast<float4*>(gv_smem + (size_t)kGvWarps * NS * kGvBufBytes);
    __shared__ int s_e[MOE_MAX_E];                       // active experts, in order
    __shared__ int s_r0[MOE_MAX_E];                      // their first row
    __shared__ int s_nr[MOE_MAX_E];                      // and their row count
    __shared__ int s_nact;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    pdl_wait();
    pdl_launch();

    // active experts: rows > 0 and offsets inside [0, rows_max]; an expert
    // whose offsets are not is skipped (and recorded by the debug build)
    if (warp == 0) {
        int base = 0;
        bool bad = false;
        for (int e0 = 0; e0 < p.E; e0 += 32) {
            const int e = e0 + lane;
            int r0 = 0, nr = 0;
            if (e < p.E) {
                r0 = p.indptr[e];
                const int r1 = p.indptr[e + 1];
                nr = r1 - r0;
                if (r0 < 0 || nr < 0 || r1 > p.rows_max || nr > kGvRows * NT) {
                    bad = true;
                    nr = 0;
                }
            }
            const unsigned act = __ballot_sync(0xffffffffu, nr > 0);
            if (nr > 0) {
                const int at = base + __popc(act & ((1u << lane) - 1u));
                s_e[at] = e;
                s_r0[at] = r0;
                s_nr[at] = nr;
            }
            base += __popc(act);
        }
        if (lane == 0) s_nact = base;
        if constexpr (kDebugChecks) {
            if (__any_sync(0xffffffffu, bad) && lane == 0) debug_record_bounds(p.status);
        }
    }
    __syncthreads();

    const int gpe = p.N / kGvRows;                        // groups per expert
    const long long G = (long long)s_nact * gpe;
    const int g0 = (int)(G * blockIdx.x / gridDim.x);
    const int g1 = (int)(G * (blockIdx.x + 1) / gridDim.x);
    const int ng = g1 - g0;
    if (ng <= 0) return;

    const int gid = lane >> 2;
    const int tig = lane & 3;

    if (warp < kGvWarps) {
        // ---------------------------------------------------------- K warps
        // Item it of the CTA's i-th group is the CTA's item i*S + it; warp w
        // runs the items congruent to w modulo kGvWarps, in order.
        const int C = p.K / 32;                          // 32-element chunks per row
        const int S = (p.K + kGvItemK - 1) / kGvItemK;   // items per group
        const int S_mod = S % kGvWarps;
        const uint32_t buf0 = smem_addr(gv_smem + (size_t)warp * NS * kGvBufBytes);
        constexpr int kRowsPerItem = 16;

        // the prefetch cursor walks the same item sequence ahead of the MMAs
        int pf_i = 0, pf_first = warp, pf_it = warp;
        auto pf_settle = [&]() {   // move to the first group that has an item for this warp
            while (pf_i < ng && pf_it >= S) {
                ++pf_i;
                pf_first -= S_mod;
                if (pf_first < 0) pf_first += kGvWarps;
                pf_it = pf_first;
            }
        };
        pf_settle();
        auto issue = [&](int slot) {
            // copy the next item's weight rows into buffer `slot` (piece p of
            // row r at position p ^ (r & 7)); always one commit group, empty
            // past the end, so the wait counts below stay aligned
            if (pf_i < ng) {
                const int g = g0 + pf_i;
                const int a = g / gpe;
                const int n0 = (g - a * gpe) * kGvRows;
                const size_t wrow = ((size_t)s_e[a] * p.N + n0) * (size_t)p.K;
                const int k0 = pf_it * kGvItemK;
                const int npieces = min(kGvItemK, p.K - k0) / 8;   // 16-byte pieces per row
                const uint32_t dst = buf0 + (uint32_t)slot * kGvBufBytes;
                const int pc = lane & 15;
#pragma unroll
                for (int i = 0; i < kRowsPerItem / 2; ++i) {
                    const int r = 2 * i + (lane >> 4);
                    if (pc < npieces) {
                        const __nv_bfloat16* src =
                            (r < 8 ? p.B0 + wrow + (size_t)r * p.K : p.B1 + wrow + (size_t)(r - 8) * p.K) + k0 + pc * 8;
                        cp_async16(dst + (uint32_t)(r * (kGvItemK * 2) + ((pc ^ (r & 7)) << 4)), src);
                    }
                }
                pf_it += kGvWarps;
                pf_settle();
            }
            cp_async_commit();
        };
#pragma unroll
        for (int s = 0; s < NS - 1; ++s) issue(s);

        int cons = 0;         // items consumed
        int first = warp;     // (warp - i*S) mod kGvWarps
        for (int i = 0; i < ng; ++i) {
            const int g = g0 + i;
            const int a = g / gpe;
            const int r0 = s_r0[a];
            const int nr = s_nr[a];
            const __nv_bfloat16* xr[NT];
            bool xv[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                xv[nt] = nt * 8 + gid < nr;
                xr[nt] = p.A + (size_t)(r0 + (xv[nt] ? nt * 8 + gid : 0)) * p.K + tig * 8;
            }
            float acc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;

            for (int it = first; it < S; it += kGvWarps) {
                issue((cons + NS - 1) % NS);
                cp_async_wait<NS - 1>();
                __syncwarp();
                const uint32_t buf = buf0 + (uint32_t)(cons % NS) * kGvBufBytes;
                const int kc0 = it * kGvChunks;
                const int kc1 = min(kc0 + kGvChunks, C);
#pragma unroll
                for (int u = 0; u < kGvChunks; ++u) {
                    if (kc0 + u < kc1) {
                        const int pc = 4 * u + tig;
                        const uint32_t sw = (uint32_t)((pc ^ (gid & 7)) << 4);
                        const uint4 wa = lds128(buf + (uint32_t)(gid * (kGvItemK * 2)) + sw);
                        const uint4 wb = lds128(buf + (uint32_t)((gid + 8) * (kGvItemK * 2)) + sw);
                        const size_t off = (size_t)(kc0 + u) * 32;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const uint4 xb = xv[nt] ? ld_cached(xr[nt] + off) : make_uint4(0, 0, 0, 0);
                            mma_bf16(acc[nt], wa.x, wb.x, wa.y, wb.y, xb.x, xb.y);
                            mma_bf16(acc[nt], wa.z, wb.z, wa.w, wb.w, xb.z, xb.w);
                        }
                    }
                }
                __syncwarp();   // the buffer is refilled by a later issue()
                ++cons;
            }
            first -= S_mod;
            if (first < 0) first += kGvWarps;
            const int s = i % kGvRing;
            if (i >= kGvRing) bar_sync(bar_free(s));
            float4* dst = part + ((size_t)(s * kGvWarps + warp) * 32 + lane) * NT;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) dst[nt] = make_float4(acc[nt][0], acc[nt][1], acc[nt][2], acc[nt][3]);
            bar_arrive(bar_full(s));
        }
        cp_async_wait<0>();
    } else {
        // ---------------------------------------------------------- reducer
        for (int i = 0; i < ng; ++i) {
            const int g = g0 + i;
            const int a = g / gpe;
            const int n = (g - a * gpe) * kGvRows + gid;
            const int r0 = s_r0[a];
            const int nr = s_nr[a];
            const int s = i % kGvRing;
            bar_sync(bar_full(s));
            float4 sum[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) sum[nt] = make_float4(0.f, 0.f, 0.f, 0.f);
            const float4* src = part + ((size_t)s * kGvWarps * 32 + lane) * NT;
            for (int w = 0; w < kGvWarps; ++w) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const float4 v = src[(size_t)w * 32 * NT + nt];
                    sum[nt].x += v.x;
                    sum[nt].y += v.y;
                    sum[nt].z += v.z;
                    sum[nt].w += v.w;
                }
            }
            if (i + kGvRing < ng) bar_arrive(bar_free(s));
            // accumulator (row gid, token 2t), (gid, 2t+1), (gid+8, 2t), (gid+8, 2t+1)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int j0 = nt * 8 + 2 * tig;
                const float o0 = silu(sum[nt].x) * sum[nt].z;
                const float o1 = silu(sum[nt].y) * sum[nt].w;
                if (j0 < nr) p.out[(size_t)(r0 + j0) * p.N + n] = __float2bfloat16(o0);
                if (j0 + 1 < nr) p.out[(size_t)(r0 + j0 + 1) * p.N + n] = __float2bfloat16(o1);
            }
        }
    }
}

}  // namespace

cudaError_t launch_gemv_swiglu(const GemvLaunch& a, cudaStream_t st) {
    GemvParams p = {};
    p.indptr = a.indptr;
    p.E = a.E;
    p.A = static_cast<const __nv_bfloat16*>(a.A);
    p.B0 = static_cast<const __nv_bfloat16*>(a.B0);
    p.B1 = static_cast<const __nv_bfloat16*>(a.B1);
    p.out = static_cast<__nv_bfloat16*>(a.out);
    p.N = a.N;
    p.K = a.K;
    p.rows_max = a.rows_max;
    p.status = a.status;
    if (a.max_group_rows > kGvRows) return cudaErrorInvalidValue;   // one 8-row token tile per group
    static bool attr_set[64] = {};   // per device; the size never changes
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(gemv_swiglu_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)kGvSmemBytes);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    cudaError_t e = launch_k(gemv_swiglu_kernel, dim3(a.grid), dim3(kGvThreads), kGvSmemBytes, st, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace moe
