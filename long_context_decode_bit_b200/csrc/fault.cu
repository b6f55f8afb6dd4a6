// Device fault word: set by a kernel whose bounded wait gave up (bit 0), or,
// in the debug build, whose bounds check failed (bit 1).
//
// The scan's shared-memory ring waits on mbarriers with a poll limit.  A wait
// that runs out (which a correct launch never does) makes the kernel set
// this word and leave its loop instead of spinning for ever; the scores of
// that launch are then void.  The union kernel turns a set word into
// FATHOM_ERR_TIMEOUT in union_count, and fathom_device_status() reads it from
// the host.  The word stays set until fathom_device_status(clear = 1).
//
// Host code cannot use a __device__ object's name as a device address, so
// the first use on each device looks it up with cudaGetSymbolAddress (with
// that device current) and caches it.
#include <mutex>

#include "common.cuh"

namespace fathom {
namespace {

__device__ int32_t g_device_fault;

constexpr int kMaxDevices = 128;
int32_t* g_fault_addr[kMaxDevices];
cudaError_t g_fault_err[kMaxDevices];
std::once_flag g_fault_once[kMaxDevices];

}  // namespace

int device_fault_word(int32_t** out)
{
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_status(e);
    if (dev < 0 || dev >= kMaxDevices) return FATHOM_ERR_UNSUPPORTED;
    std::call_once(g_fault_once[dev], [dev] {
        void* p = nullptr;
        g_fault_err[dev] = cudaGetSymbolAddress(&p, g_device_fault);
        g_fault_addr[dev] = (g_fault_err[dev] == cudaSuccess) ? static_cast<int32_t*>(p) : nullptr;
    });
    if (g_fault_err[dev] != cudaSuccess) return cuda_status(g_fault_err[dev]);
    *out = g_fault_addr[dev];
    return FATHOM_OK;
}

}  // namespace fathom

extern "C" int fathom_device_status(int clear, fathom_stream_t stream)
{
    using namespace fathom;
    int32_t* w = nullptr;
    int st = device_fault_word(&w);
    if (st) return st;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, w, sizeof(v), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e);
    if (clear && v) {
        e = cudaMemsetAsync(w, 0, sizeof(v), s);
        if (e == cudaSuccess) e = cudaStreamSynchronize(s);
        if (e != cudaSuccess) return cuda_status(e);
    }
    return (v & kFaultTimeout) ? FATHOM_ERR_TIMEOUT : ((v & kFaultBounds) ? FATHOM_ERR_BOUNDS : FATHOM_OK);
}
