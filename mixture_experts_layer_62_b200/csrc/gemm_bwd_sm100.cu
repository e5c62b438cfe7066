// Backward grouped GEMMs of the SwiGLU experts on the sm_100a tensor cores
// (tcgen05 + TMEM + TMA), one kernel template, four modes. Rows are the
// padded permuted rows of the forward (every expert's rows a multiple of 64,
// padding rows zero), so every K-block of a weight-gradient GEMM lies inside
// one expert.
//
// With dO = g * dy gathered to permuted rows, and per expert e:
//   BW_DH   dH = dO W2_e            A = dO  [rows, d] (K-major),  B = W2_e [d, d_ff] (N-major)
//           epilogue: dA = dH * b * SiLU'(a), dB = dH * SiLU(a) from the
//           forward's gate/up pre-activations (a, b), written as dAB in the
//           same [128 gate | 128 up] column order
//   BW_DX   dXp = dA W1_e + dB W3_e A = dAB [rows, 2 d_ff] (K-major), B = W1_e / W3_e
//           [d_ff, d] (N-major), the K-block picks W1 or W3 by its half
//   BW_DW2  dW2_e = dO_e^T H_e      A = dO^T (M-major), B = H (N-major), K = the expert's rows
//   BW_DW13 [dW1_e; dW3_e] = dAB_e^T Xp_e   A = dAB^T (M-major), B = Xp (N-major)
// ("Week 2 Day 2: Mixture of Experts" §1.3 and §2.1 for the expert; the
// chain rule of the forward's GEMMs for the shapes.)
//
// Same pipeline as the forward kernel: persistent grid, warp 0 issues TMA
// into a 4-stage ring (A 16 KB + B 32 KB per stage), warp 1 issues
// tcgen05.mma M=128 N=256 K=16 into two TMEM accumulators, warps 2-5 drain.
// MN-major operands are loaded as 64-wide (128-byte) column chunks of 64 K
// rows, 128-byte swizzle, and described to the MMA with the MN-major
// descriptor (chunks 8 KB apart, 8-row swizzle atoms 1 KB apart). Every wait
// is bounded; no cluster multicast.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_common.cuh"

namespace moe {

namespace {

using namespace tc;

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_BYTES = BN * BK * 2;          // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int MN_CHUNK = 64 * BK * 2;         // one 64-wide chunk of an MN-major operand: 8 KB
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int NUM_THREADS = 192;
constexpr int OUT_BLOCK = 32 * 32 * 4;        // one 32 x 32 fp32 block, 128-byte swizzled rows
constexpr int OUT_WARP_BYTES = 2 * OUT_BLOCK;  // double-buffered per epilogue warp
constexpr int CTL_BYTES = 1024;                // barriers; keeps the output blocks 1024-byte aligned
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 /*align*/ + CTL_BYTES + 4 * OUT_WARP_BYTES;

struct BParams {
    const int32_t* indptr;    // padded row offsets of the groups [E+1]
    const int32_t* tiles;     // BW_DH / BW_DX: cumulative tiles [E+1]
    int E;
    int M, N, K;              // dgrad: output columns N, reduction K; wgrad: gradient rows M, columns N
    int mt, nt;               // wgrad: M- and N-blocks per expert
    int d, d_ff;
    const __nv_bfloat16* ab;  // BW_DH: forward gate/up pre-activations [rows][2 d_ff]
    __nv_bfloat16* out_bf16;  // BW_DH: dAB [rows][2 d_ff]; BW_DX: dXp [rows][d]
    float* out0;              // BW_DW2: dW2 [E][d][d_ff]; BW_DW13: dW1 [E][d_ff][d]
    float* out1;              // BW_DW13: dW3 [E][d_ff][d]
    int32_t* status;
    long long timeout_ns;      // limit of every wait of the work itself
    long long drain_ns;        // limit of the drain after a wait gave up
};

struct BTile {
    int g, row0, rows, m_blk, n_blk, num_kb;
};

template <int MODE>
__device__ __forceinline__ int total_units(const BParams& p) {
    if (MODE == BW_DH || MODE == BW_DX) return p.tiles[p.E];
    return p.E * p.mt * p.nt;
}

template <int MODE>
__device__ __forceinline__ BTile decode(const BParams& p, int tile) {
    BTile t;
    if (MODE == BW_DH || MODE == BW_DX) {
        int lo = 0, hi = p.E;   // tiles[lo] <= tile < tiles[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (p.tiles[mid] <= tile) lo = mid; else hi = mid;
        }
        t.g = lo;
        t.row0 = p.indptr[lo];
        t.rows = p.indptr[lo + 1] - t.row0;
        tile -= p.tiles[lo];
        const int mt = (t.rows + BM - 1) / BM;
        t.n_blk = tile / mt;
        t.m_blk = tile % mt;
        t.num_kb = p.K / BK;
    } else {
        const int per = p.mt * p.nt;
        t.g = tile / per;
        tile -= t.g * per;
        t.n_blk = tile / p.mt;
        t.m_blk = tile % p.mt;
        t.row0 = p.indptr[t.g];
        t.rows = p.indptr[t.g + 1] - t.row0;
        t.num_kb = (t.rows + BK - 1) / BK;
    }
    return t;
}

struct Ctl {
    uint64_t full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ bool wait_b(uint64_t* bar, uint32_t parity, Ctl* ctl, const BParams& p) {
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
// drain after a wait gave up: its own long limit
__device__ __forceinline__ void wait_d(uint64_t* bar, uint32_t parity, const BParams& p) {
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - t0 > static_cast<uint64_t>(p.drain_ns)) {
            atomicExch(p.status, MOE_ERR_TIMEOUT);
            return;
        }
    }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
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

// One stage of loads for (tile, K-block kb) into the stage at `sa`.
template <int MODE>
__device__ __forceinline__ void issue_stage(const BParams& p, const BTile& t, int kb, uint32_t sa, uint64_t* bar,
                                            const CUtensorMap* mA, const CUtensorMap* mB0, const CUtensorMap* mB1,
                                            bool with_a, bool with_b) {
    if (with_a) {
        if (MODE == BW_DH || MODE == BW_DX) {
            tma_load_2d(sa, mA, bar, kb * BK, t.row0 + t.m_blk * BM);   // 128 rows x 64 K
        } else {
#pragma unroll
            for (int i = 0; i < 2; ++i)                                  // 2 x (64 M x 64 K rows)
                tma_load_2d(sa + i * MN_CHUNK, mA, bar, t.m_blk * BM + 64 * i, t.row0 + kb * BK);
        }
    }
    if (with_b) {
        const CUtensorMap* mb = mB0;
        int krow;
        if (MODE == BW_DH) {
            krow = t.g * p.d + kb * BK;                    // rows of W2_e = K
        } else if (MODE == BW_DX) {
            const int nb = kb >> 2, half = (kb >> 1) & 1, sub = kb & 1;   // [128 gate | 128 up] per 128 units
            mb = half ? mB1 : mB0;
            krow = t.g * p.d_ff + nb * 128 + sub * 64;
        } else {
            krow = t.row0 + kb * BK;                       // permuted rows = K
        }
        const uint32_t sb = sa + A_BYTES;
#pragma unroll
        for (int i = 0; i < 4; ++i) tma_load_2d(sb + i * MN_CHUNK, mb, bar, t.n_blk * BN + 64 * i, krow);
    }
}

template <int MODE>
__global__ void __launch_bounds__(NUM_THREADS, 1)
tc_bwd_gemm(const __grid_constant__ CUtensorMap mA, const __grid_constant__ CUtensorMap mB0,
            const __grid_constant__ CUtensorMap mB1, const __grid_constant__ CUtensorMap mO0,
            const __grid_constant__ CUtensorMap mO1, const BParams p) {
    constexpr bool A_MN = (MODE == BW_DW2 || MODE == BW_DW13);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    Ctl* ctl = reinterpret_cast<Ctl*>(smem + STAGES * STAGE_BYTES);
    static_assert(sizeof(Ctl) <= CTL_BYTES, "barrier block");
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
        prefetch_map(&mA);
        prefetch_map(&mB0);
        prefetch_map(&mB1);
        prefetch_map(&mO0);
        prefetch_map(&mO1);
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
    pdl_wait();
    pdl_launch();
    const int units = total_units<MODE>(p);

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0, issued_mask = 0, issued_ph = 0;
            bool aborted = false;
            for (int u = blockIdx.x; u < units && !aborted; u += gridDim.x) {
                const BTile t = decode<MODE>(p, u);
                for (int kb = 0; kb < t.num_kb; ++kb) {
                    if (!wait_b(&ctl->empty[s], ph ^ 1u, ctl, p)) { aborted = true; break; }
                    mbar_arrive_expect_tx(&ctl->full[s], STAGE_BYTES);
                    issue_stage<MODE>(p, t, kb, smem_u32(smem + s * STAGE_BYTES), &ctl->full[s], &mA, &mB0, &mB1,
                                      true, true);
                    issued_mask |= 1u << s;
                    issued_ph = (issued_ph & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
            }
            if (aborted)
                for (int st = 0; st < STAGES; ++st)
                    if ((issued_mask >> st) & 1u) wait_d(&ctl->full[st], (issued_ph >> st) & 1u, p);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            constexpr uint32_t idesc = make_idesc_major(BM, BN, A_MN ? 1 : 0, 1);
            int s = 0, acc = 0;
            uint32_t ph = 0, aph = 0;
            bool aborted = false, issued_any = false;
            for (int u = blockIdx.x; u < units && !aborted; u += gridDim.x) {
                const BTile t = decode<MODE>(p, u);
                if (!wait_b(&ctl->tempty[acc], aph ^ 1u, ctl, p)) { aborted = true; break; }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * ACC_COLS);
                for (int kb = 0; kb < t.num_kb; ++kb) {
                    if (!wait_b(&ctl->full[s], ph, ctl, p)) { aborted = true; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * STAGE_BYTES);
                    const uint64_t a0 = A_MN ? sw128_mn_desc(sa, MN_CHUNK) : sw128_desc(sa);
                    const uint64_t b0 = sw128_mn_desc(sa + A_BYTES, MN_CHUNK);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        // K-major: the next 16 K are 32 bytes along the row; MN-major:
                        // two 8-row swizzle atoms (2048 bytes) further
                        const uint64_t ad = a0 + (A_MN ? static_cast<uint64_t>(kk) * (2048 >> 4) : 2u * kk);
                        const uint64_t bd = b0 + static_cast<uint64_t>(kk) * (2048 >> 4);
                        tc_mma(d_tmem, ad, bd, idesc, (kb != 0 || kk != 0) ? 1u : 0u);
                    }
                    issued_any = true;
                    tc_commit(&ctl->empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (aborted) break;
                tc_commit(&ctl->tfull[acc]);   // with no K-block this arrives at once
                acc ^= 1;
                if (acc == 0) aph ^= 1u;
            }
            if (aborted && issued_any) {
                tc_commit(&ctl->drain);
                wait_d(&ctl->drain, 0, p);
            }
        }
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        const int q = warp & 3;
        const int r = q * 32 + lane;
        int acc = 0;
        uint32_t aph = 0;
        uint8_t* outbuf = smem + STAGES * STAGE_BYTES + CTL_BYTES + q * OUT_WARP_BYTES;
        int nstore = 0;   // bulk stores this warp has issued (buffer = nstore & 1)
        for (int u = blockIdx.x; u < units; u += gridDim.x) {
            const BTile t = decode<MODE>(p, u);
            if (MODE == BW_DH) {
                // the forward's pre-activations of this thread's row, 32 hidden
                // units per chunk; chunk c + 1 is requested before chunk c is
                // used, and chunk 0 before the accumulator is ready
                const int grow = t.m_blk * BM + r;
                const bool valid = grow < t.rows;
                const size_t orow = static_cast<size_t>(t.row0) + static_cast<size_t>(grow);
                const size_t ld = 2 * static_cast<size_t>(p.d_ff);
                auto chunk_off = [&](int c) {
                    const int j0 = t.n_blk * BN + c;
                    return orow * ld + static_cast<size_t>(j0 >> 7) * 256 + (j0 & 127);
                };
                auto chunk_ok = [&](int c) { return valid && t.n_blk * BN + c < p.d_ff; };
                uint4 na[4], nb[4];
                if (chunk_ok(0)) {
                    const uint4* pa = reinterpret_cast<const uint4*>(p.ab + chunk_off(0));
#pragma unroll
                    for (int i = 0; i < 4; ++i) { na[i] = pa[i]; nb[i] = pa[16 + i]; }
                }
                if (!wait_b(&ctl->tfull[acc], aph, ctl, p)) break;
                tc_fence_after();
                const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                    static_cast<uint32_t>(acc * ACC_COLS);
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    uint4 ca[4], cb[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) { ca[i] = na[i]; cb[i] = nb[i]; }
                    if (c + 32 < BN && chunk_ok(c + 32)) {
                        const uint4* pa = reinterpret_cast<const uint4*>(p.ab + chunk_off(c + 32));
#pragma unroll
                        for (int i = 0; i < 4; ++i) { na[i] = pa[i]; nb[i] = pa[16 + i]; }
                    }
                    uint32_t v[32];
                    tmem_ld32(tb + c, v);
                    if (chunk_ok(c)) {
                        uint4* qa = reinterpret_cast<uint4*>(p.out_bf16 + chunk_off(c));
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            float a[8], b[8];
                            unpack8(ca[i], a);
                            unpack8(cb[i], b);
                            uint32_t da[4], db[4];
#pragma unroll
                            for (int e2 = 0; e2 < 4; ++e2) {
                                float rda[2], rdb[2];
#pragma unroll
                                for (int h = 0; h < 2; ++h) {
                                    const int e = 2 * e2 + h;
                                    const float dh = __uint_as_float(v[8 * i + e]);
                                    const float sg = 1.f / (1.f + __expf(-a[e]));
                                    rda[h] = dh * b[e] * (sg * (1.f + a[e] * (1.f - sg)));
                                    rdb[h] = dh * (a[e] * sg);
                                }
                                da[e2] = pack2(rda[0], rda[1]);
                                db[e2] = pack2(rdb[0], rdb[1]);
                            }
                            qa[i] = make_uint4(da[0], da[1], da[2], da[3]);
                            qa[16 + i] = make_uint4(db[0], db[1], db[2], db[3]);
                        }
                    }
                }
            } else if (MODE == BW_DX) {
                if (!wait_b(&ctl->tfull[acc], aph, ctl, p)) break;
                tc_fence_after();
                const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                    static_cast<uint32_t>(acc * ACC_COLS);
                const int grow = t.m_blk * BM + r;
                const bool valid = grow < t.rows;
                const size_t orow = static_cast<size_t>(t.row0) + static_cast<size_t>(grow);
                __nv_bfloat16* out = p.out_bf16 + orow * static_cast<size_t>(p.N);
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    uint32_t v[32];
                    tmem_ld32(tb + c, v);
                    const int col = t.n_blk * BN + c;
                    if (valid && col < p.N) {
                        uint4* dst = reinterpret_cast<uint4*>(out + col);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_uint4(pack2(__uint_as_float(v[8 * i]), __uint_as_float(v[8 * i + 1])),
                                                pack2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3])),
                                                pack2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5])),
                                                pack2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7])));
                    }
                }
            } else {
                // weight gradients, fp32: BW_DW2 rows of dW2_e; BW_DW13 rows of
                // dW1_e (gate half of a 256-row AB group) or dW3_e (up half).
                // Each 32 x 32 block of the warp is written to shared memory in
                // the 128-byte-swizzled layout of the output map and stored by
                // one bulk tensor store; two buffers per warp let the next block
                // be written while the previous store still reads.
                if (!wait_b(&ctl->tfull[acc], aph, ctl, p)) break;
                tc_fence_after();
                const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                    static_cast<uint32_t>(acc * ACC_COLS);
                const bool empty_k = t.num_kb == 0;   // an expert without rows: its gradient is 0
                const CUtensorMap* mo;
                int orow;                              // first output row of this warp's block
                if (MODE == BW_DW2) {
                    mo = &mO0;
                    orow = t.g * p.M + t.m_blk * BM + q * 32;
                } else {
                    mo = (t.m_blk & 1) ? &mO1 : &mO0;
                    orow = t.g * p.d_ff + (t.m_blk >> 1) * 128 + q * 32;
                }
#pragma unroll 1
                for (int c = 0; c < BN; c += 32) {
                    uint32_t v[32];
                    if (!empty_k) tmem_ld32(tb + c, v);
                    const int col = t.n_blk * BN + c;
                    if (col >= p.N) continue;          // the same for the whole warp
                    uint8_t* buf = outbuf + (nstore & 1) * OUT_BLOCK;
                    if (lane == 0) bulk_wait_read<1>();   // the store two blocks back has read `buf`
                    __syncwarp();
                    uint8_t* rowp = buf + lane * 128;
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
                            empty_k ? make_uint4(0u, 0u, 0u, 0u)
                                    : make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(mo, smem_u32(buf), col, orow);
                        bulk_commit();
                    }
                    ++nstore;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->tempty[acc]);
            acc ^= 1;
            if (acc == 0) aph ^= 1u;
        }
        if (lane == 0) bulk_wait_all();   // every bulk store of this warp has completed
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

template <int MODE>
cudaError_t launch_bwd_mode(const CUtensorMap (&maps)[5], const BParams& bp, cudaStream_t st) {
    static bool attr_set[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!attr_set[dev]) {
        cudaError_t e = cudaFuncSetAttribute(tc_bwd_gemm<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             SMEM_BYTES);
        if (e != cudaSuccess) return e;
        attr_set[dev] = true;
    }
    const int grid = device_sm_count();
    if (grid <= 0) return cudaErrorInvalidDevice;
    return launch_k(tc_bwd_gemm<MODE>, dim3(grid), dim3(NUM_THREADS), (size_t)SMEM_BYTES, st, maps[0], maps[1],
                    maps[2], maps[3], maps[4], bp);
}

}  // namespace

cudaError_t launch_bwd_gemm(const BwdGemmArgs& a, cudaStream_t st) {
    CUtensorMap maps[5];
    const bool a_mn = a.mode == BW_DW2 || a.mode == BW_DW13;
    // K-major operands: boxes of 64 K x 128 rows; MN-major: 64 columns x 64 K rows
    if (!make_tmap(&maps[0], a.A, a.a_rows, a.a_cols, a_mn ? 64 : 128)) return cudaErrorInvalidValue;
    if (!make_tmap(&maps[1], a.B0, a.b_rows, a.b_cols, 64)) return cudaErrorInvalidValue;
    if (!make_tmap(&maps[2], a.B1 != nullptr ? a.B1 : a.B0, a.b_rows, a.b_cols, 64)) return cudaErrorInvalidValue;
    // weight-gradient outputs, fp32 [groups * rows][N] for bulk stores
    if (a.mode == BW_DW2) {
        if (!make_tmap_f32_store(&maps[3], a.out0, a.E * a.M, a.N)) return cudaErrorInvalidValue;
        maps[4] = maps[3];
    } else if (a.mode == BW_DW13) {
        if (!make_tmap_f32_store(&maps[3], a.out0, a.E * a.d_ff, a.N)) return cudaErrorInvalidValue;
        if (!make_tmap_f32_store(&maps[4], a.out1, a.E * a.d_ff, a.N)) return cudaErrorInvalidValue;
    } else {
        maps[3] = maps[0];
        maps[4] = maps[0];
    }
    BParams bp;
    bp.indptr = a.indptr;
    bp.tiles = a.tiles;
    bp.E = a.E;
    bp.M = a.M; bp.N = a.N; bp.K = a.K;
    bp.mt = ceil_div(a.M > 0 ? a.M : 1, BM);
    bp.nt = ceil_div(a.N, BN);
    bp.d = a.d; bp.d_ff = a.d_ff;
    bp.ab = static_cast<const __nv_bfloat16*>(a.ab);
    bp.out_bf16 = static_cast<__nv_bfloat16*>(a.out_bf16);
    bp.out0 = a.out0;
    bp.out1 = a.out1;
    bp.status = a.status;
    bp.timeout_ns = wait_limit_ns();
    bp.drain_ns = kDrainLimitNs;
    switch (a.mode) {
        case BW_DH: return launch_bwd_mode<BW_DH>(maps, bp, st);
        case BW_DX: return launch_bwd_mode<BW_DX>(maps, bp, st);
        case BW_DW2: return launch_bwd_mode<BW_DW2>(maps, bp, st);
        case BW_DW13: return launch_bwd_mode<BW_DW13>(maps, bp, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace moe
