// fathom_scan_topk_noalloc: one decode step's candidate scan and top-k with
// no caller-provided scratch.
//
// Some callers cannot allocate device memory at the point where they run
// the scan: an operator plugged into another inference runtime that has
// already reserved the free device memory for its own KV-cache pool and
// hands the operator no allocator, or a serving loop that must not call
// cudaMalloc because it synchronises the device.  For them this entry
// point keeps the candidate buffer (thresholds, counters, sample scores
// and candidate entries) in a fixed array in the library's own device
// memory instead of a caller buffer.  The caller passes only the index,
// the plan, the queries and the output arrays.
//
// The array is a file-scope __device__ object: every device that loads
// the library holds FATHOM_NOALLOC_SCRATCH_BYTES of it until the process
// exits.  Host code cannot use the array's name as a device address, so
// the first call on each device looks the address up with
// cudaGetSymbolAddress (with that device current) and caches it.
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace fathom {

// Defined in api.cu.
int topk_cand_args_check(int G, int64_t n, int k, const int32_t* idx, const int32_t* union_idx,
                         const int32_t* union_count);

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[FATHOM_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
void* g_scratch_addr[kMaxDevices];
cudaError_t g_scratch_err[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

// Device address of this device's scratch array (set up on first use).
int scratch_for_current_device(void** out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
    if (dev < 0 || dev >= kMaxDevices) return FATHOM_ERR_UNSUPPORTED;
    std::call_once(g_scratch_once[dev], [dev] {
        void* p = nullptr;
        g_scratch_err[dev] = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        g_scratch_addr[dev] = (g_scratch_err[dev] == cudaSuccess) ? p : nullptr;
    });
    if (g_scratch_err[dev] != cudaSuccess) return cuda_status(g_scratch_err[dev]);
    *out = g_scratch_addr[dev];
    return FATHOM_OK;
}

}  // namespace
}  // namespace fathom

extern "C" int fathom_scan_topk_noalloc(const uint64_t* planes, const uint16_t* scales, int64_t H, int D,
                                        int64_t n, int64_t nb_stride, const uint16_t* active,
                                        const int32_t* n_active, const float* q, int G, int k, int32_t* idx,
                                        int32_t* union_idx, int32_t* union_count, fathom_stream_t stream)
{
    using namespace fathom;
    if (H < 0 || n < 0 || G < 1 || G > kMaxG) return H < 0 || n < 0 ? FATHOM_ERR_INVALID_ARG : FATHOM_ERR_UNSUPPORTED;
    if (H == 0) return FATHOM_OK;
    if (k < 1 || k > n) return FATHOM_ERR_INVALID_ARG;
    // The top-k outputs are checked before the scan enqueues anything.
    int st = topk_cand_args_check(G, n, k, idx, union_idx, union_count);
    if (st != FATHOM_OK) return st;
    const size_t need = fathom_scan_cand_bytes(H, G, n, k);
    if (need == 0) return FATHOM_ERR_INVALID_ARG;
    if (need > FATHOM_NOALLOC_SCRATCH_BYTES) return FATHOM_ERR_WORKSPACE;
    void* scratch = nullptr;
    st = scratch_for_current_device(&scratch);
    if (st != FATHOM_OK) return st;
    nvtxRangePushA("fathom_scan_topk_noalloc");
    // The threshold pass resets the counters it needs, so the array's
    // leftover contents from an earlier call do not matter.
    st = fathom_scan(planes, scales, H, D, n, nb_stride, active, n_active, q, G, FATHOM_SCAN_CANDIDATE, nullptr,
                     scratch, need, k, stream);
    if (st == FATHOM_OK)
        st = fathom_topk(nullptr, scratch, H, G, n, k, idx, union_idx, union_count, nullptr, 0, stream);
    nvtxRangePop();
    return st;
}
