// fp32 grouped GEMM on CUDA cores, for the fp32 path of the layer.
//
// Z = GroupGemm(data, indptr, weights) ("Lecture 21 · LLM: Mixture-of-Experts"
// §3.3): group e multiplies rows [indptr[e], indptr[e+1]) of the permuted
// activations by expert e's weights. SWIGLU mode computes both W1 and W3
// products of a 64-column slice and writes SiLU(a) * b ("Week 2 Day 2" §2.1
// SwiGLU experts); PLAIN mode writes the product. tcgen05 has no fp32-input
// MMA (its tf32 kind keeps 10 mantissa bits), so this path stays on FMA units
// to hold fp32 accuracy.
//
// A persistent grid walks the tile list built from the group sizes; tile
// (g, m, n) is 64 rows x 64 columns. Each thread owns a 4 x 4 block of
// outputs and sums k in ascending order (fixed order, deterministic).
#include "common.cuh"

namespace moe {

constexpr int kBK = 16;

__device__ __forceinline__ void find_group(const int32_t* tiles, int G, int tile, int& g) {
    int lo = 0, hi = G;
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (tiles[mid] <= tile) lo = mid; else hi = mid;
    }
    g = lo;
}

template <bool SWIGLU>
__global__ void __launch_bounds__(256) simt_gemm_kernel(GroupedArgs a) {
    __shared__ float As[kBK][kSimtTileM + 4];
    __shared__ float Bs[SWIGLU ? 2 : 1][kBK][kSimtTileN + 4];
    pdl_wait();
    pdl_launch();
    const int G = a.E + a.has_shared;
    const int total = a.tiles[G];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;   // 16 x 16 threads
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
        int g;
        find_group(a.tiles, G, tile, g);
        const int kind = g >= a.E ? 1 : 0;
        const int rows = kind ? a.T : a.indptr[g + 1] - a.indptr[g];
        const int row0 = kind ? 0 : a.indptr[g];
        const int mt = (rows + kSimtTileM - 1) / kSimtTileM;
        const int local = tile - a.tiles[g];
        const int n_blk = local / mt, m_blk = local % mt;
        const int N = a.N[kind], K = a.K[kind];
        const float* A = (const float*)a.A[kind];
        const int e = kind ? 0 : g;
        const float* B0 = (const float*)a.B[kind][0] + (size_t)e * N * K;
        const float* B1 = SWIGLU ? (const float*)a.B[kind][1] + (size_t)e * N * K : nullptr;

        float acc0[4][4] = {}, acc1[4][4] = {};
        for (int k0 = 0; k0 < K; k0 += kBK) {
            __syncthreads();
            for (int i = threadIdx.x; i < kSimtTileM * kBK; i += blockDim.x) {
                int r = i / kBK, kk = i % kBK;
                int gr = m_blk * kSimtTileM + r, gk = k0 + kk;
                float v = 0.f;
                if (gr < rows && gk < K) v = A[(size_t)(row0 + gr) * K + gk];
                As[kk][r] = v;
            }
            for (int i = threadIdx.x; i < kSimtTileN * kBK; i += blockDim.x) {
                int c = i / kBK, kk = i % kBK;
                int gc = n_blk * kSimtTileN + c, gk = k0 + kk;
                bool ok = gc < N && gk < K;
                Bs[0][kk][c] = ok ? B0[(size_t)gc * K + gk] : 0.f;
                if (SWIGLU) Bs[SWIGLU ? 1 : 0][kk][c] = ok ? B1[(size_t)gc * K + gk] : 0.f;
            }
            __syncthreads();
#pragma unroll
            for (int kk = 0; kk < kBK; ++kk) {
                float av[4], bv0[4], bv1[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) av[i] = As[kk][ty * 4 + i];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    bv0[j] = Bs[0][kk][tx * 4 + j];
                    if (SWIGLU) bv1[j] = Bs[SWIGLU ? 1 : 0][kk][tx * 4 + j];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        acc0[i][j] = fmaf(av[i], bv0[j], acc0[i][j]);
                        if (SWIGLU) acc1[i][j] = fmaf(av[i], bv1[j], acc1[i][j]);
                    }
            }
        }
        float* out = (float*)a.out[kind];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            int gr = m_blk * kSimtTileM + ty * 4 + i;
            if (gr >= rows) continue;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                int gc = n_blk * kSimtTileN + tx * 4 + j;
                if (gc >= N) continue;
                float v = acc0[i][j];
                if (SWIGLU) {
                    float h = v / (1.f + expf(-v));
                    v = h * acc1[i][j];
                }
                out[(size_t)(row0 + gr) * N + gc] = v;
            }
        }
    }
}

cudaError_t launch_simt_gemm(bool swiglu, const GroupedArgs& a, cudaStream_t st) {
    int grid = device_sm_count() * 4;
    if (grid <= 0) grid = 148 * 4;
    if (swiglu) return launch_k(simt_gemm_kernel<true>, dim3(grid), dim3(256), 0, st, a);
    return launch_k(simt_gemm_kernel<false>, dim3(grid), dim3(256), 0, st, a);
}

}  // namespace moe
