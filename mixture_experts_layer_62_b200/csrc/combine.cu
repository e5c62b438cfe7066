// Un-permute and mix ("Lecture 21 · LLM: Mixture-of-Experts" §3.2 step 4;
// "Week 2 Day 2: Mixture of Experts" §1.3, y = sum_{i in T} g_i f_i(x)),
// plus the always-on shared expert (same page §4.1).
//
// One warp per token. Every lane owns 16-byte column vectors of the row and
// accumulates in fp32: slot 0, 1, ..., k-1 (dropped slots skipped), then the
// shared-expert row; the sum is rounded once on the store. Each output row is
// written by exactly one warp, so no atomics are needed and the summation
// order is fixed.
#include "common.cuh"

namespace moe {

template <typename T> struct VecTraits;
template <> struct VecTraits<float> {
    static constexpr int N = 4;
    __device__ static void load(const void* p, float (&v)[4]) {
        float4 a = *reinterpret_cast<const float4*>(p);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    }
    __device__ static void store(void* p, const float (&v)[4]) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct VecTraits<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const void* p, float (&v)[8]) {
        uint4 u = *reinterpret_cast<const uint4*>(p);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(h[i]);
            v[2 * i] = f.x; v[2 * i + 1] = f.y;
        }
    }
    __device__ static void store(void* p, const float (&v)[8]) {
        uint4 u;
        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        *reinterpret_cast<uint4*>(p) = u;
    }
};

// With split-K partials (opart != null and *split2 > 1) an expert output row
// is the sum over the splits, s = 0, 1, ..., of the fp32 partial rows.
template <typename T>
__global__ void __launch_bounds__(256)
combine_kernel(const T* __restrict__ o, const int32_t* __restrict__ pos, const float* __restrict__ gate,
               const T* __restrict__ s, T* __restrict__ out, int Tn, int d, int k,
               const float* __restrict__ opart, long long opart_stride, const int32_t* __restrict__ split2) {
    using V = VecTraits<T>;
    constexpr int VN = V::N;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * (blockDim.x >> 5) + warp;
    if (t >= Tn) return;
    const int S = (opart != nullptr && split2 != nullptr) ? *split2 : 1;
    int p[MOE_MAX_K];
    float g[MOE_MAX_K];
#pragma unroll
    for (int j = 0; j < MOE_MAX_K; ++j) {
        if (j < k) {
            p[j] = pos[(size_t)t * k + j];
            g[j] = gate[(size_t)t * k + j];
        }
    }
    const int nvec = d / VN;
    for (int v = lane; v < nvec; v += 32) {
        float acc[VN];
#pragma unroll
        for (int i = 0; i < VN; ++i) acc[i] = 0.f;
#pragma unroll
        for (int j = 0; j < MOE_MAX_K; ++j) {
            if (j < k && p[j] >= 0) {
                float ov[VN];
                if (S > 1) {
#pragma unroll
                    for (int i = 0; i < VN; ++i) ov[i] = 0.f;
                    for (int sp = 0; sp < S; ++sp) {
                        const float* src = opart + (size_t)sp * opart_stride + (size_t)p[j] * d + (size_t)v * VN;
#pragma unroll
                        for (int i = 0; i < VN; i += 4) {
                            float4 q4 = *reinterpret_cast<const float4*>(src + i);
                            ov[i] += q4.x; ov[i + 1] += q4.y; ov[i + 2] += q4.z; ov[i + 3] += q4.w;
                        }
                    }
                } else {
                    V::load(o + (size_t)p[j] * d + (size_t)v * VN, ov);
                }
#pragma unroll
                for (int i = 0; i < VN; ++i) acc[i] = fmaf(g[j], ov[i], acc[i]);
            }
        }
        if (s != nullptr) {
            float sv[VN];
            V::load(s + (size_t)t * d + (size_t)v * VN, sv);
#pragma unroll
            for (int i = 0; i < VN; ++i) acc[i] += sv[i];
        }
        V::store(out + (size_t)t * d + (size_t)v * VN, acc);
    }
}

cudaError_t launch_combine(int dtype, const void* o, const int32_t* pos, const float* gate,
                           const void* s, void* out, int T, int d, int k, cudaStream_t st,
                           const float* opart, long long opart_stride, const int32_t* split2) {
    if (T == 0) return cudaSuccess;
    const int per_block = 8;
    dim3 grid(ceil_div(T, per_block)), block(per_block * 32);
    if (dtype == MOE_DTYPE_BF16)
        combine_kernel<__nv_bfloat16><<<grid, block, 0, st>>>(
            (const __nv_bfloat16*)o, pos, gate, (const __nv_bfloat16*)s, (__nv_bfloat16*)out, T, d, k, opart,
            opart_stride, split2);
    else
        combine_kernel<float><<<grid, block, 0, st>>>((const float*)o, pos, gate, (const float*)s,
                                                      (float*)out, T, d, k, nullptr, 0, nullptr);
    return cudaGetLastError();
}

// Split-K reduction of grouped GEMM 1/3: the partial rows hold, per 128
// output columns, 128 gate sums followed by 128 up sums (the accumulator
// layout of a SwiGLU tile). h[r][c] = SiLU(sum_s gate) * (sum_s up), summed
// s = 0, 1, ... in order. One block per row; nothing to do when the split
// factor chosen on the device is 1 (the GEMM then wrote h itself).
__global__ void __launch_bounds__(256)
swiglu_reduce_kernel(const float* __restrict__ part, long long split_stride, int ld,
                     const int32_t* __restrict__ split13, const int32_t* __restrict__ indptr, int E, int d_ff,
                     __nv_bfloat16* __restrict__ h) {
    const int S = *split13;
    if (S <= 1) return;
    const int r = blockIdx.x;
    if (r >= indptr[E]) return;
    for (int c = threadIdx.x; c < d_ff; c += blockDim.x) {
        const size_t col = (size_t)(c / 128) * 256 + (c % 128);
        float g = 0.f, u = 0.f;
        for (int sp = 0; sp < S; ++sp) {
            const float* row = part + (size_t)sp * split_stride + (size_t)r * ld;
            g += row[col];
            u += row[col + 128];
        }
        h[(size_t)r * d_ff + c] = __float2bfloat16_rn(g / (1.f + __expf(-g)) * u);
    }
}

cudaError_t launch_swiglu_reduce(const float* part, long long split_stride, int ld, const int32_t* split13,
                                 const int32_t* indptr, int E, int max_rows, int d_ff, void* h,
                                 cudaStream_t st) {
    if (max_rows <= 0) return cudaSuccess;
    swiglu_reduce_kernel<<<max_rows, 256, 0, st>>>(part, split_stride, ld, split13, indptr, E, d_ff,
                                                   (__nv_bfloat16*)h);
    return cudaGetLastError();
}

}  // namespace moe
