// Allocation-free entry point of the permutation stage.
//
// moe_permute needs a caller-provided workspace for two small scratch arrays
// (per-chunk expert counts and their expert-major scan). Some callers cannot
// allocate device memory at the point where they run the layer: a plugin of an
// inference runtime that owns all device memory and hands the plugin only its
// input and output buffers, or a latency-critical loop where cudaMalloc could
// block or synchronise the device. moe_permute_noalloc runs the same kernels
// with that scratch in a fixed-size array of this file instead, so the caller
// passes inputs and outputs only.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds it (1 MiB) until the process exits. In host code its name is
// only a host-side stand-in, not a device address, so the device address is
// looked up with cudaGetSymbolAddress once per device, with that device
// current, on the first call made on that device.
#include <cmath>
#include <mutex>

#include "common.cuh"

namespace {

// Scratch capacity: E * kk * ceil(T / 32) entries for each of the two arrays
// (kk = k under the slot-priority drop order, else 1).
constexpr long long kMaxEntries = 1LL << 17;
constexpr int kMaxDevices = 64;

__device__ __align__(256) int32_t g_permute_scratch[2 * kMaxEntries];

struct DeviceScratch {
    std::once_flag once;
    int32_t* ptr = nullptr;
    cudaError_t err = cudaSuccess;
};
DeviceScratch g_scratch[kMaxDevices];

// Device address of the scratch array on the current device (looked up once
// per device); nullptr on failure.
int32_t* scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    DeviceScratch& s = g_scratch[dev];
    std::call_once(s.once, [&s] {
        void* ptr = nullptr;
        s.err = cudaGetSymbolAddress(&ptr, g_permute_scratch);
        if (s.err == cudaSuccess) s.ptr = static_cast<int32_t*>(ptr);
    });
    return s.err == cudaSuccess ? s.ptr : nullptr;
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

// The problem checks of the other entry points, restated for this one.
int check(const moe_problem* p) {
    if (p == nullptr) return MOE_ERR_INVALID_ARG;
    if (p->T < 0 || p->d <= 0 || p->d_ff <= 0 || p->E < 1 || p->E > MOE_MAX_E || p->k < 1 || p->k > p->E ||
        p->k > MOE_MAX_K || p->d_ff_shared < 0)
        return MOE_ERR_INVALID_ARG;
    if (p->dtype != MOE_DTYPE_F32 && p->dtype != MOE_DTYPE_BF16) return MOE_ERR_INVALID_ARG;
    if (p->bias_mode < MOE_BIAS_NONE || p->bias_mode > MOE_BIAS_PROB) return MOE_ERR_INVALID_ARG;
    if (!(p->capacity_factor == p->capacity_factor)) return MOE_ERR_INVALID_ARG;
    if ((long long)p->T * p->k >= (1LL << 30)) return MOE_ERR_UNSUPPORTED;
    if (p->dtype == MOE_DTYPE_BF16 ? (p->d % 8 != 0) : (p->d % 4 != 0)) return MOE_ERR_UNSUPPORTED;
    return MOE_OK;
}

}  // namespace

extern "C" int moe_permute_noalloc(const moe_problem* p, const void* x, const int32_t* idx, int32_t* pos,
                                   int32_t* indptr, int32_t* row_token, void* xp, void* stats, void* stream) {
    int rc = check(p);
    if (rc != MOE_OK) return rc;
    if (!idx || !pos || !indptr || !stats) return MOE_ERR_INVALID_ARG;
    if (xp && (!x || !aligned16(x) || !aligned16(xp))) return MOE_ERR_INVALID_ARG;
    if (!aligned16(stats)) return MOE_ERR_INVALID_ARG;
    const long long nb = (p->T + moe::kChunk - 1) / moe::kChunk;
    if (p->gate_mode != MOE_GATE_SELECTED && p->gate_mode != MOE_GATE_FULL) return MOE_ERR_INVALID_ARG;
    if (p->drop_order != MOE_DROP_TOKEN && p->drop_order != MOE_DROP_SLOT) return MOE_ERR_INVALID_ARG;
    const int kk = moe::count_slots(*p);
    if (kk > 1 && p->E * p->k > moe::kMaxSlotCounts) return MOE_ERR_UNSUPPORTED;
    if ((long long)p->E * kk * nb > kMaxEntries) return MOE_ERR_UNSUPPORTED;   // beyond the static scratch
    if (p->pad_rows != 0) return MOE_ERR_UNSUPPORTED;                         // dense rows only

    int32_t* scratch = scratch_on_current_device();
    if (scratch == nullptr) return MOE_ERR_CUDA;
    int32_t* blockcnt = scratch;                 // written in full by the histogram
    int32_t* blockoff = scratch + kMaxEntries;   // written in full by the scan
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    double cf = (double)p->capacity_factor;
    int C = -1;
    if (cf > 0.0) {
        double c = std::ceil(cf * (double)p->T * (double)p->k / (double)p->E);
        C = c > 2147483647.0 ? -1 : (int)c;
    }
    if (p->T == 0) {
        if (moe::launch_zero_stats(stats, p->E, C, st) != cudaSuccess) return MOE_ERR_CUDA;
        if (cudaMemsetAsync(indptr, 0, sizeof(int32_t) * (size_t)(p->E + 1), st) != cudaSuccess) return MOE_ERR_CUDA;
        return MOE_OK;
    }
    if (cudaMemsetAsync(stats, 0, sizeof(int32_t), st) != cudaSuccess) return MOE_ERR_CUDA;
    if (moe::launch_hist(idx, p->T, p->k, kk, p->E, blockcnt, st) != cudaSuccess) return MOE_ERR_CUDA;
    moe::ScanArgs sa = {};
    sa.T = p->T; sa.k = p->k; sa.E = p->E; sa.capacity = C; sa.kk = kk;
    sa.blockcnt = blockcnt; sa.blockoff = blockoff; sa.blockpsum = nullptr;
    sa.indptr = indptr; sa.stats = stats;
    if (moe::launch_scan(sa, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (moe::launch_permute_gather(p->dtype, x, idx, blockoff, indptr, p->T, p->d, p->E, p->k, kk, C, pos,
                                   row_token, xp, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}
