// Per-device launch facts, looked up once and kept: the SM count (for grid
// sizing) and each kernel's raised dynamic shared memory limit.  Entry
// points run on every decode step, so none of them should pay a driver
// query that has the same answer every time.
#include <mutex>

#include "common.cuh"

namespace fathom {
namespace {

constexpr int kMaxDevices = 128;
int g_sms[kMaxDevices];
cudaError_t g_sms_err[kMaxDevices];
std::once_flag g_sms_once[kMaxDevices];

// (kernel, device) -> dynamic shared memory bytes the limit was raised to.
struct SmemLimit {
    const void* func;
    int dev;
    size_t bytes;
};
constexpr int kMaxLimits = 1024;
SmemLimit g_limits[kMaxLimits];
int g_n_limits = 0;
std::mutex g_limits_mu;

int current_device(int* dev)
{
    const cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_status(e);
    if (*dev < 0 || *dev >= kMaxDevices) return FATHOM_ERR_UNSUPPORTED;
    return FATHOM_OK;
}

}  // namespace

int device_sm_count(int* sms)
{
    int dev = -1;
    const int st = current_device(&dev);
    if (st) return st;
    std::call_once(g_sms_once[dev], [dev] {
        int v = 0;
        g_sms_err[dev] = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        g_sms[dev] = v;
    });
    if (g_sms_err[dev] != cudaSuccess) return cuda_status(g_sms_err[dev]);
    *sms = g_sms[dev];
    return FATHOM_OK;
}

int ensure_dynamic_smem(const void* func, size_t bytes)
{
    if (bytes <= 48 * 1024) return FATHOM_OK;   // within the default limit
    int dev = -1;
    const int st = current_device(&dev);
    if (st) return st;
    std::lock_guard<std::mutex> lock(g_limits_mu);
    SmemLimit* hit = nullptr;
    for (int i = 0; i < g_n_limits; ++i)
        if (g_limits[i].func == func && g_limits[i].dev == dev) hit = &g_limits[i];
    if (hit && hit->bytes >= bytes) return FATHOM_OK;
    const cudaError_t e =
        cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
    if (e != cudaSuccess) return cuda_status(e);
    if (hit) {
        hit->bytes = bytes;
    } else if (g_n_limits < kMaxLimits) {
        g_limits[g_n_limits++] = SmemLimit{func, dev, bytes};
    }
    return FATHOM_OK;
}

}  // namespace fathom
