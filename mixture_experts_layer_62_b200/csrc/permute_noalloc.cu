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
#include <mutex>

#include "common.cuh"

namespace {

// Scratch capacity: E * kk * ceil(T / 32) entries for each of the two arrays
// (kk = k under the slot-priority drop order, else 1).
constexpr long long kMaxEntries = 1LL << 17;
constexpr int kMaxDevices = 64;

__device__ __align__(256) int32_t g_permute_scratch[2 * kMaxEntries];

// Device address of the scratch array, per device. A successful lookup is
// kept for the life of the process; a failed one is not, so a later call on
// that device tries again instead of failing for the rest of the process.
std::mutex g_scratch_mutex;
int32_t* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device; nullptr if the
// lookup failed.
int32_t* scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_permute_scratch) != cudaSuccess) {
            cudaGetLastError();   // the failure is reported by the return code, not left pending
            return nullptr;
        }
        g_scratch_ptr[dev] = static_cast<int32_t*>(ptr);
    }
    return g_scratch_ptr[dev];
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

}  // namespace

extern "C" int moe_permute_noalloc(const moe_problem* p, const void* x, const int32_t* idx, int32_t* pos,
                                   int32_t* indptr, int32_t* row_token, void* xp, void* stats, void* stream) {
    int rc = moe::check_problem(p);   // the checks of moe_permute
    if (rc != MOE_OK) return rc;
    if (!idx || !pos || !indptr || !stats) return MOE_ERR_INVALID_ARG;
    if (xp && (!x || !aligned16(x) || !aligned16(xp))) return MOE_ERR_INVALID_ARG;
    if (!aligned16(stats)) return MOE_ERR_INVALID_ARG;
    const long long nb = (p->T + moe::kChunk - 1) / moe::kChunk;
    const int kk = moe::count_slots(*p);
    if ((long long)p->E * kk * nb > kMaxEntries) return MOE_ERR_UNSUPPORTED;   // beyond the static scratch
    if (p->pad_rows != 0) return MOE_ERR_UNSUPPORTED;                         // dense rows only

    int32_t* scratch = scratch_on_current_device();
    if (scratch == nullptr) return MOE_ERR_CUDA;
    int32_t* blockcnt = scratch;                 // written in full by the histogram
    int32_t* blockoff = scratch + kMaxEntries;   // written in full by the scan
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int C = moe::capacity_of(p);
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
