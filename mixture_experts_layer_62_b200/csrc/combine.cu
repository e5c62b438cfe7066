// Un-permute and mix ("Lecture 21 · LLM: Mixture-of-Experts" §3.2 step 4;
// "Week 2 Day 2: Mixture of Experts" §1.3, y = sum_{i in T} g_i f_i(x)),
// plus the always-on shared expert (same page §4.1).
//
// One warp per (token, slice of the row). Every lane owns 16-byte column
// vectors of the slice and accumulates in fp32: slot 0, 1, ..., k-1 (dropped
// slots skipped), then the shared-expert row; the sum is rounded once on the
// store. Each output element is written by exactly one lane, so no atomics
// are needed and the summation order is fixed.
#include "common.cuh"

namespace moe {

template <typename T> struct VecTraits;
template <> struct VecTraits<float> {
    static constexpr int N = 4;
    __device__ static void load(const void* p, float (&v)[4]) {
        float4 a = *reinterpret_cast<const float4*>(p);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    }
    __device__ static void unpack(const uint4& u, float (&v)[4]) {
        v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
        v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
    }
    __device__ static void store(void* p, const float (&v)[4]) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    }
};
template <> struct VecTraits<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void load(const void* p, float (&v)[8]) {
        uint4 u = *reinterpret_cast<const uint4*>(p);
        unpack(u, v);
    }
    __device__ static void unpack(const uint4& u, float (&v)[8]) {
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

// One warp per (token, slice of the row): a slice is 32 x vpl 16-byte
// vectors (vpl = 1 for small batches), so few tokens still spread over many
// warps.
constexpr int kCbVecPerLane = 2;
constexpr int kCbSlotGroup = 2;   // slots whose rows are requested together
constexpr int kCbWarps = 8;

template <typename T>
__global__ void __launch_bounds__(kCbWarps * 32, 4)
combine_kernel(const T* __restrict__ o, const int32_t* __restrict__ pos, const float* __restrict__ gate,
               const T* __restrict__ s, T* __restrict__ out, int Tn, int d, int k, int slices, int vpl, int rows,
               int32_t* __restrict__ status) {
    using V = VecTraits<T>;
    constexpr int VN = V::N;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long task = (long long)blockIdx.x * kCbWarps + warp;
    const int t = (int)(task / slices), sl = (int)(task % slices);
    if (t >= Tn) {
        pdl_wait();
        pdl_launch();
        return;
    }
    // lane j holds the slot-j position and gate of the warp's token (k <= 32);
    // they come from the routing, at least two launches back (both GEMMs run
    // after it), so they are read before the dependency wait; the expert
    // outputs are read after it
    int p_l = -1;
    float g_l = 0.f;
    if (lane < k) {
        p_l = pos[(size_t)t * k + lane];
        g_l = gate[(size_t)t * k + lane];
        if (kDebugChecks && p_l >= rows) {   // a position past o: recorded, the slot skipped
            if (sl == 0) debug_record_bounds(status);
            p_l = -1;
        }
    }
    pdl_wait();
    pdl_launch();
    const int nvec = d / VN;
    // the warp's vpl vector columns are processed together: for each pair of
    // slots, every row vector of the pair and of every column is requested
    // before any is accumulated (2 vpl loads in flight per lane); the
    // accumulation is still in slot order for each element
    float acc[kCbVecPerLane][VN];
#pragma unroll
    for (int i = 0; i < kCbVecPerLane; ++i)
#pragma unroll
        for (int e = 0; e < VN; ++e) acc[i][e] = 0.f;
    int vv[kCbVecPerLane];
    bool valid[kCbVecPerLane];
#pragma unroll
    for (int i = 0; i < kCbVecPerLane; ++i) {
        vv[i] = (sl * vpl + i) * 32 + lane;
        valid[i] = i < vpl && vv[i] < nvec;
    }
    for (int j0 = 0; j0 < k; j0 += kCbSlotGroup) {
        uint4 raw[kCbSlotGroup][kCbVecPerLane];
        int pj[kCbSlotGroup];
        float gj[kCbSlotGroup];
#pragma unroll
        for (int u = 0; u < kCbSlotGroup; ++u) {
            pj[u] = __shfl_sync(0xffffffffu, p_l, j0 + u);
            gj[u] = __shfl_sync(0xffffffffu, g_l, j0 + u);
#pragma unroll
            for (int i = 0; i < kCbVecPerLane; ++i) {
                raw[u][i] = make_uint4(0u, 0u, 0u, 0u);
                if (j0 + u < k && pj[u] >= 0 && valid[i])
                    raw[u][i] = *reinterpret_cast<const uint4*>(o + (size_t)pj[u] * d + (size_t)vv[i] * VN);
            }
        }
#pragma unroll
        for (int u = 0; u < kCbSlotGroup; ++u) {
            if (j0 + u < k && pj[u] >= 0) {
#pragma unroll
                for (int i = 0; i < kCbVecPerLane; ++i) {
                    float ov[VN];
                    V::unpack(raw[u][i], ov);
#pragma unroll
                    for (int e = 0; e < VN; ++e) acc[i][e] = fmaf(gj[u], ov[e], acc[i][e]);
                }
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kCbVecPerLane; ++i) {
        if (!valid[i]) continue;
        if (s != nullptr) {
            float sv[VN];
            V::load(s + (size_t)t * d + (size_t)vv[i] * VN, sv);
#pragma unroll
            for (int e = 0; e < VN; ++e) acc[i][e] += sv[e];
        }
        V::store(out + (size_t)t * d + (size_t)vv[i] * VN, acc[i]);
    }
}

cudaError_t launch_combine(int dtype, const void* o, const int32_t* pos, const float* gate,
                           const void* s, void* out, int T, int d, int k, int rows, int32_t* status,
                           cudaStream_t st) {
    if (T == 0) return cudaSuccess;
    const int vn = dtype == MOE_DTYPE_BF16 ? 8 : 4;
    // small batches: one vector per lane per warp, so the few rows are spread
    // over more warps
    const int vpl = T < 256 ? 1 : kCbVecPerLane;
    const int slices = ceil_div(d / vn, 32 * vpl);
    const long long tasks = (long long)T * slices;
    const unsigned grid = (unsigned)((tasks + kCbWarps - 1) / kCbWarps);
    if (dtype == MOE_DTYPE_BF16)
        return launch_k(combine_kernel<__nv_bfloat16>, dim3(grid), dim3(kCbWarps * 32), 0, st,
                        (const __nv_bfloat16*)o, pos, gate, (const __nv_bfloat16*)s, (__nv_bfloat16*)out, T, d, k,
                        slices, vpl, rows, status);
    return launch_k(combine_kernel<float>, dim3(grid), dim3(kCbWarps * 32), 0, st, (const float*)o, pos, gate,
                    (const float*)s, (float*)out, T, d, k, slices, vpl, rows, status);
}

}  // namespace moe
