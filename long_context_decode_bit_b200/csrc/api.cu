// extern "C" entry points of libfathom.so (declared in include/fathom.h):
// argument validation on the host, then the launches.  No allocation.  The
// library's state is the per-thread last CUDA error code, one fault word per
// device (fault.cu) and the scratch array of the allocation-free entry point
// (noalloc.cu).  Every entry point that enqueues work opens an NVTX range
// named after it, so that a trace shows the library's calls on the host
// timeline (a no-op unless a profiler is attached).
#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace fathom {

int launch_pack(const void* keys, int key_dtype, int64_t H, int64_t n, int D, int64_t stride_h,
                int64_t stride_tok, uint64_t* planes, uint16_t* scales, int64_t nb_stride, cudaStream_t stream);
int launch_pack_rotated(const void* keys, int key_dtype, int64_t H, int64_t n, int D, int64_t stride_h,
                        int64_t stride_tok, const float* U, uint64_t* planes, uint16_t* scales, int64_t nb_stride,
                        cudaStream_t stream);
int launch_plan(const float* sigma2, const float* q, int64_t H, int G, int D, const int32_t* budget_bits,
                int32_t budget_flat, uint8_t* depth, uint16_t* active, int32_t* n_active, float* theta,
                cudaStream_t stream);
int launch_plan_fixed(const float* q, int64_t H, int G, int D, int r, int bits, uint8_t* depth, uint16_t* active,
                      int32_t* n_active, cudaStream_t stream);
int launch_scan(const uint64_t* planes, const uint16_t* scales, int64_t H, int D, int64_t n, int64_t nb_stride,
                const uint16_t* active, const int32_t* n_active, const float* q, int G, int mode, float* scores,
                void* cand, int k, bool nib, cudaStream_t stream);
int launch_topk(const float* scores, const void* cand, int64_t H, int G, int64_t n, int k, int32_t* idx,
                int32_t* union_idx, int32_t* union_count, cudaStream_t stream);
int launch_scan_tm(const uint8_t* store, const uint16_t* scales, int64_t H, int D, int64_t n, int64_t nb_stride,
                   const uint16_t* active, const int32_t* n_active, const float* q, int G, int mode, float* scores,
                   void* cand, int k, cudaStream_t stream);
int launch_tm_from_planes(const uint64_t* planes, int64_t H, int D, int64_t n, int64_t nb_stride, uint8_t* store,
                          cudaStream_t stream);

int launch_dequant_rows(const uint64_t* planes, const uint16_t* scales, int64_t H, int D, int64_t n,
                        int64_t nb_stride, const int32_t* rows, int64_t M, const int32_t* row_count, int bits,
                        float* out, cudaStream_t stream);

size_t layer_budgets_workspace_bytes(int64_t H, int D);
int launch_layer_budgets(const float* sigma2, const float* q, int64_t H, int G, int D, int layers, int64_t total_bits,
                         int32_t* budget, void* ws, cudaStream_t stream);
size_t calibrate_workspace_bytes(int64_t H, int D, bool with_cov);
int launch_calibrate(const void* keys, int key_dtype, int64_t H, int64_t n, int D, int64_t sh, int64_t st,
                     float* mean, float* sigma2, float* cov, void* ws, cudaStream_t stream);

size_t union_attention_workspace_bytes(int64_t H, int G, int D, int64_t M);
int launch_union_attention(const void* k, const void* v, int kv_dtype, int64_t H, int64_t n, int D, int64_t sh,
                           int64_t st, const float* q, int G, const int32_t* uni, const int32_t* count, int64_t M,
                           float scale, float* out, void* ws, cudaStream_t stream);

static thread_local int g_last_cuda_error = 0;

// NVTX range over one library call.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

int cuda_status(cudaError_t e)
{
    if (e == cudaSuccess) return FATHOM_OK;
    g_last_cuda_error = static_cast<int>(e);
    return FATHOM_ERR_CUDA;
}

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// A pointer the current device can dereference: device or managed memory,
// or page-locked host memory mapped into the device's address space.
int check_device_ptr(const void* p)
{
    if (!p) return FATHOM_ERR_INVALID_ARG;
    cudaPointerAttributes attr;
    const cudaError_t e = cudaPointerGetAttributes(&attr, p);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return FATHOM_ERR_INVALID_ARG;
    }
    switch (attr.type) {
        case cudaMemoryTypeDevice:
        case cudaMemoryTypeManaged:
            return FATHOM_OK;
        case cudaMemoryTypeHost:
            return attr.devicePointer == p ? FATHOM_OK : FATHOM_ERR_INVALID_ARG;
        default:
            return FATHOM_ERR_INVALID_ARG;
    }
}

bool dims_ok(int D, int G) { return D >= 32 && D <= kMaxD && D % 32 == 0 && G >= 1 && G <= kMaxG; }

#define FATHOM_TRY_IN(expr)              \
    do {                                 \
        const int _st = (expr);          \
        if (_st != FATHOM_OK) return _st; \
    } while (0)

// Store layouts a scan reads: bit planes, channel-major nibbles, token-major nibble rows.
enum StoreLayout { kPlanesLayout = 0, kNibblesLayout = 1, kTokenMajorLayout = 2 };

int scan_entry(const void* planes, const uint16_t* scales, int64_t H, int D, int64_t n, int64_t nb_stride,
               const uint16_t* active, const int32_t* n_active, const float* q, int G, int mode, float* scores,
               void* cand, size_t cand_bytes, int k, StoreLayout layout, fathom_stream_t stream)
{
    if (H < 0 || H > 65535 || n < 0 || n >= (1LL << 31)) return FATHOM_ERR_INVALID_ARG;
    if (!dims_ok(D, G)) return FATHOM_ERR_UNSUPPORTED;
    if (mode < FATHOM_SCAN_DENSE || mode > FATHOM_SCAN_FILTER) return FATHOM_ERR_INVALID_ARG;
    if (H == 0 || n == 0) return FATHOM_OK;
    const int64_t nb = ceil_div(n, kBlockTokens);
    if (nb_stride < nb) return FATHOM_ERR_INVALID_ARG;
    if ((nb_stride & 7) || !aligned(planes, 16) || !aligned(scales, 16) || !aligned(active, 2) ||
        !aligned(n_active, 4) || !aligned(q, 4))
        return FATHOM_ERR_UNSUPPORTED;
    FATHOM_TRY_IN(check_device_ptr(planes));
    FATHOM_TRY_IN(check_device_ptr(scales));
    FATHOM_TRY_IN(check_device_ptr(active));
    FATHOM_TRY_IN(check_device_ptr(n_active));
    FATHOM_TRY_IN(check_device_ptr(q));
    if (mode == FATHOM_SCAN_DENSE) {
        if (!aligned(scores, 4)) return FATHOM_ERR_UNSUPPORTED;
        FATHOM_TRY_IN(check_device_ptr(scores));
    } else {
        if (k < 1 || k > n) return FATHOM_ERR_INVALID_ARG;
        if (k > kMaxCandK) return FATHOM_ERR_UNSUPPORTED;
        if (!aligned(cand, 16)) return FATHOM_ERR_UNSUPPORTED;
        FATHOM_TRY_IN(check_device_ptr(cand));
        if (cand_bytes < cand_layout(H, G, n, k).total) return FATHOM_ERR_WORKSPACE;
    }
    if (layout == kTokenMajorLayout)
        return launch_scan_tm(static_cast<const uint8_t*>(planes), scales, H, D, n, nb_stride, active, n_active, q, G,
                              mode, scores, cand, k, reinterpret_cast<cudaStream_t>(stream));
    return launch_scan(static_cast<const uint64_t*>(planes), scales, H, D, n, nb_stride, active, n_active, q, G, mode,
                       scores, cand, k, layout == kNibblesLayout, reinterpret_cast<cudaStream_t>(stream));
}

// One thread per (group, channel, block): the four plane words -> the four
// nibble words of the same codes.
__global__ void nibbles_kernel(const uint64_t* __restrict__ planes, int64_t rows, int64_t nb, int64_t nb_stride,
                               uint64_t* __restrict__ nib)
{
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= rows * nb) return;
    const int64_t r = t / nb, b = t % nb;   // r = h * D + j
    uint64_t p[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) p[q] = planes[(r * 4 + q) * nb_stride + b];
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint64_t out = 0;
        for (int e = 0; e < 16; ++e) {
            const int i = 16 * w + e;
            uint64_t c = 0;
#pragma unroll
            for (int q = 0; q < 4; ++q) c |= ((p[q] >> i) & 1ull) << (3 - q);
            out |= c << (4 * e);
        }
        nib[(r * 4 + w) * nb_stride + b] = out;
    }
}


}  // namespace

// Checks of fathom_topk's output arguments and limits for the candidate
// path, shared with fathom_scan_topk_noalloc so that it rejects bad outputs
// before it enqueues anything.
int topk_cand_args_check(int G, int64_t n, int k, const int32_t* idx, const int32_t* union_idx,
                         const int32_t* union_count)
{
    if (G < 1 || G > kMaxG) return FATHOM_ERR_UNSUPPORTED;
    if (k < 1 || k > n) return FATHOM_ERR_INVALID_ARG;
    if (k > kMaxK || k > kMaxCandK || static_cast<int64_t>(G) * k > kMaxUnion) return FATHOM_ERR_UNSUPPORTED;
    if (!aligned(idx, 4) || !aligned(union_idx, 4) || !aligned(union_count, 4)) return FATHOM_ERR_UNSUPPORTED;
    FATHOM_TRY_IN(check_device_ptr(idx));
    FATHOM_TRY_IN(check_device_ptr(union_idx));
    FATHOM_TRY_IN(check_device_ptr(union_count));
    return FATHOM_OK;
}

}  // namespace fathom

using namespace fathom;

#define FATHOM_TRY(expr)                 \
    do {                                 \
        const int _st = (expr);          \
        if (_st != FATHOM_OK) return _st; \
    } while (0)

extern "C" {

int fathom_version(void) { return 10000; }

const char* fathom_status_string(int status)
{
    switch (status) {
        case FATHOM_OK: return "ok";
        case FATHOM_ERR_INVALID_ARG: return "invalid argument";
        case FATHOM_ERR_UNSUPPORTED: return "unsupported size or alignment";
        case FATHOM_ERR_CUDA: return "CUDA error";
        case FATHOM_ERR_WORKSPACE: return "buffer too small";
        case FATHOM_ERR_TIMEOUT: return "device wait timed out";
        case FATHOM_ERR_OVERFLOW: return "candidate pass could not prove the top-k exact";
        case FATHOM_ERR_BOUNDS: return "device bounds check failed (debug build)";
        default: return "unknown status";
    }
}

int fathom_last_cuda_error(void) { return g_last_cuda_error; }

int64_t fathom_nb_stride(int64_t n)
{
    if (n <= 0) return 0;
    return ceil_div(ceil_div(n, kBlockTokens), 16) * 16;
}

int fathom_pack(const void* keys, int key_dtype, int64_t H, int64_t n, int D, int64_t key_stride_h,
                int64_t key_stride_tok, uint64_t* planes, uint16_t* scales, int64_t nb_stride,
                fathom_stream_t stream)
{
    NvtxRange range("fathom_pack");
    if (H < 0 || n < 0 || n >= (1LL << 31)) return FATHOM_ERR_INVALID_ARG;
    if (key_dtype != FATHOM_KEYS_F32 && key_dtype != FATHOM_KEYS_BF16) return FATHOM_ERR_INVALID_ARG;
    if (!dims_ok(D, 1)) return FATHOM_ERR_UNSUPPORTED;
    if (H == 0 || n == 0) return FATHOM_OK;
    const int64_t nb = ceil_div(n, kBlockTokens);
    if (nb_stride < nb || (nb_stride & 1)) return FATHOM_ERR_INVALID_ARG;
    if (key_stride_tok < D || (H > 1 && key_stride_h < n * key_stride_tok)) return FATHOM_ERR_INVALID_ARG;
    if (H > 65535 / (D / 32)) return FATHOM_ERR_UNSUPPORTED;
    if (!aligned(planes, 8) || !aligned(scales, 2) || !aligned(keys, key_dtype == FATHOM_KEYS_F32 ? 4 : 2))
        return FATHOM_ERR_UNSUPPORTED;
    FATHOM_TRY(check_device_ptr(keys));
    FATHOM_TRY(check_device_ptr(planes));
    FATHOM_TRY(check_device_ptr(scales));
    return launch_pack(keys, key_dtype, H, n, D, key_stride_h, key_stride_tok, planes, scales, nb_stride,
                       reinterpret_cast<cudaStream_t>(stream));
}

int fathom_pack_rotated(const void* keys, int key_dtype, int64_t H, int64_t n, int D, int64_t key_stride_h,
                        int64_t key_stride_tok, const float* U, uint64_t* planes, uint16_t* scales,
                        int64_t nb_stride, fathom_stream_t stream)
{
    NvtxRange range("fathom_pack_rotated");
    if (H < 0 || n < 0 || n >= (1LL << 31)) return FATHOM_ERR_INVALID_ARG;
    if (key_dtype != FATHOM_KEYS_F32 && key_dtype != FATHOM_KEYS_BF16) return FATHOM_ERR_INVALID_ARG;
    if (!dims_ok(D, 1)) return FATHOM_ERR_UNSUPPORTED;
    if (H == 0 || n == 0) return FATHOM_OK;
    const int64_t nb = ceil_div(n, kBlockTokens);
    if (nb_stride < nb || (nb_stride & 1)) return FATHOM_ERR_INVALID_ARG;
    if (key_stride_tok < D || (H > 1 && key_stride_h < n * key_stride_tok)) return FATHOM_ERR_INVALID_ARG;
    if (H * (D % 128 == 0 ? D / 128 : (D % 64 == 0 ? D / 64 : D / 32)) > 65535) return FATHOM_ERR_UNSUPPORTED;
    if (!aligned(planes, 8) || !aligned(scales, 2) || !aligned(U, 4) ||
        !aligned(keys, key_dtype == FATHOM_KEYS_F32 ? 4 : 2))
        return FATHOM_ERR_UNSUPPORTED;
    FATHOM_TRY(check_device_ptr(keys));
    FATHOM_TRY(check_device_ptr(U));
    FATHOM_TRY(check_device_ptr(planes));
    FATHOM_TRY(check_device_ptr(scales));
    return launch_pack_rotated(keys, key_dtype, H, n, D, key_stride_h, key_stride_tok, U, planes, scales, nb_stride,
                               reinterpret_cast<cudaStream_t>(stream));
}

size_t fathom_layer_budgets_workspace_bytes(int64_t H, int D)
{
    if (H <= 0 || !dims_ok(D, 1)) return 0;
    return layer_budgets_workspace_bytes(H, D);
}

int fathom_layer_budgets(const float* sigma2, const float* q, int64_t H, int G, int D, int layers,
                         int64_t total_bits, int32_t* budget_bits, void* workspace, size_t ws_bytes,
                         fathom_stream_t stream)
{
    NvtxRange range("fathom_layer_budgets");
    if (H < 0 || H > 0x7FFFFFFF || layers < 1 || layers > 1024 || total_bits < 0) return FATHOM_ERR_INVALID_ARG;
    if (!dims_ok(D, G)) return FATHOM_ERR_UNSUPPORTED;
    if (H == 0) return FATHOM_OK;
    if (H % layers) return FATHOM_ERR_INVALID_ARG;
    if (ws_bytes < layer_budgets_workspace_bytes(H, D)) return FATHOM_ERR_WORKSPACE;
    if (!aligned(sigma2, 4) || !aligned(q, 4) || !aligned(budget_bits, 4) || !aligned(workspace, 256))
        return FATHOM_ERR_UNSUPPORTED;
    FATHOM_TRY(check_device_ptr(sigma2));
    FATHOM_TRY(check_device_ptr(q));
    FATHOM_TRY(check_device_ptr(budget_bits));
    FATHOM_TRY(check_device_ptr(workspace));
    return launch_layer_budgets(sigma2, q, H, G, D, layers, total_bits, budget_bits, workspace,
                                reinterpret_cast<cudaStream_t>(stream));
}

size_t fathom_calibrate_workspace_bytes(int64_t H, int D, int with_cov)
{
    if (H <= 0 || !dims_ok(D, 1)) return 0;
    return calibrate_workspace_bytes(H, D, with_cov != 0);
}

int fathom_calibrate(const void* keys, int key_dtype, int64_t H, int64_t n, int D, int64_t key_stride_h,
                     int64_t key_stride_tok, float* mean, float* sigma2, float* cov, void* workspace, size_t ws_bytes,
                     fathom_stream_t stream)
{
    NvtxRange range("fathom_calibrate");
    if (H < 0 || n < 0 || n >= (1LL << 40)) return FATHOM_ERR_INVALID_ARG;
    if (key_dtype != FATHOM_KEYS_F32 && key_dtype != FATHOM_KEYS_BF16) return FATHOM_ERR_INVALID_ARG;
    if (!dims_ok(D, 1)) return FATHOM_ERR_UNSUPPORTED;
    if (H == 0) return FATHOM_OK;
    if (H > 65535) return FATHOM_ERR_UNSUPPORTED;
    if (key_stride_tok < D || (H > 1 && key_stride_h < n * key_stride_tok)) return FATHOM_ERR_INVALID_ARG;
    if (!sigma2) return FATHOM_ERR_INVALID_ARG;
    if (ws_bytes < calibrate_workspace_bytes(H, D, cov != nullptr)) return FATHOM_ERR_WORKSPACE;
    if (!aligned(keys, key_dtype == FATHOM_KEYS_F32 ? 4 : 2) || !aligned(sigma2, 4) || (mean && !aligned(mean, 4)) ||
        (cov && !aligned(cov, 4)) || !aligned(workspace, 256))
        return FATHOM_ERR_UNSUPPORTED;
    if (n > 0) FATHOM_TRY(check_device_ptr(keys));
    FATHOM_TRY(check_device_ptr(sigma2));
    FATHOM_TRY(check_device_ptr(workspace));
    if (mean) FATHOM_TRY(check_device_ptr(mean));
    if (cov) FATHOM_TRY(check_device_ptr(cov));
    return launch_calibrate(keys, key_dtype, H, n, D, key_stride_h, key_stride_tok, mean, sigma2, cov, workspace,
                            reinterpret_cast<cudaStream_t>(stream));
}

size_t fathom_union_attention_workspace_bytes(int64_t H, int G, int D, int64_t M)
{
    if (H <= 0 || M < 1 || M > 65536 || !dims_ok(D, G)) return 0;
    return union_attention_workspace_bytes(H, G, D, M);
}

int fathom_union_attention(const void* k_cache, const void* v_cache, int kv_dtype, int64_t H, int64_t n, int D,
                           int64_t kv_stride_h, int64_t kv_stride_tok, const float* q, int G, const int32_t* union_idx,
                           const int32_t* union_count, int64_t M, float scale, float* out, void* workspace,
                           size_t ws_bytes, fathom_stream_t stream)
{
    NvtxRange range("fathom_union_attention");
    if (H < 0 || n < 0 || n >= (1LL << 31) || M < 1 || M > 65536) return FATHOM_ERR_INVALID_ARG;
    if (kv_dtype != FATHOM_KEYS_F32 && kv_dtype != FATHOM_KEYS_BF16) return FATHOM_ERR_INVALID_ARG;
    if (!dims_ok(D, G)) return FATHOM_ERR_UNSUPPORTED;
    if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return FATHOM_ERR_INVALID_ARG;
    if (H == 0) return FATHOM_OK;
    if (H > 65535) return FATHOM_ERR_UNSUPPORTED;
    if (kv_stride_tok < D || (H > 1 && kv_stride_h < n * kv_stride_tok)) return FATHOM_ERR_INVALID_ARG;
    if (ws_bytes < union_attention_workspace_bytes(H, G, D, M)) return FATHOM_ERR_WORKSPACE;
    const size_t ea = kv_dtype == FATHOM_KEYS_F32 ? 4 : 2;
    if (!aligned(k_cache, ea) || !aligned(v_cache, ea) || !aligned(q, 4) || !aligned(union_idx, 4) ||
        !aligned(union_count, 4) || !aligned(out, 4) || !aligned(workspace, 256))
        return FATHOM_ERR_UNSUPPORTED;
    FATHOM_TRY(check_device_ptr(k_cache));
    FATHOM_TRY(check_device_ptr(v_cache));
    FATHOM_TRY(check_device_ptr(q));
    FATHOM_TRY(check_device_ptr(union_idx));
    FATHOM_TRY(check_device_ptr(union_count));
    FATHOM_TRY(check_device_ptr(out));
    FATHOM_TRY(check_device_ptr(workspace));
    return launch_union_attention(k_cache, v_cache, kv_dtype, H, n, D, kv_stride_h, kv_stride_tok, q, G, union_idx,
                                  union_count, M, scale, out, workspace, reinterpret_cast<cudaStream_t>(stream));
}

int fathom_plan(const float* sigma2, const float* q, int64_t H, int G, int D, const int32_t* budget_bits,
                int32_t budget_flat, uint8_t* depth, uint16_t* active, int32_t* n_active, float* theta,
                fathom_stream_t stream)
{
    NvtxRange range("fathom_plan");
    if (H < 0 || H > 0x7FFFFFFF) return FATHOM_ERR_INVALID_ARG;
    if (!dims_ok(D, G)) return FATHOM_ERR_UNSUPPORTED;
    if (!budget_bits && (budget_flat < 0 || budget_flat > 4 * D)) return FATHOM_ERR_INVALID_ARG;
    if (H == 0) return FATHOM_OK;
    if (!aligned(sigma2, 4) || !aligned(q, 4) || !aligned(active, 2) || !aligned(n_active, 4) ||
        (budget_bits && !aligned(budget_bits, 4)) || (theta && !aligned(theta, 4)))
        return FATHOM_ERR_UNSUPPORTED;
    FATHOM_TRY(check_device_ptr(sigma2));
    FATHOM_TRY(check_device_ptr(q));
    FATHOM_TRY(check_device_ptr(depth));
    FATHOM_TRY(check_device_ptr(active));
    FATHOM_TRY(check_device_ptr(n_active));
    if (budget_bits) FATHOM_TRY(check_device_ptr(budget_bits));
    if (theta) FATHOM_TRY(check_device_ptr(theta));
    return launch_plan(sigma2, q, H, G, D, budget_bits, budget_flat, depth, active, n_active, theta,
                       reinterpret_cast<cudaStream_t>(stream));
}

int fathom_plan_fixed(const float* q, int64_t H, int G, int D, int r, int bits, uint8_t* depth, uint16_t* active,
                      int32_t* n_active, fathom_stream_t stream)
{
    NvtxRange range("fathom_plan_fixed");
    if (H < 0 || H > 0x7FFFFFFF) return FATHOM_ERR_INVALID_ARG;
    if (!dims_ok(D, G)) return FATHOM_ERR_UNSUPPORTED;
    if (r < 0 || r > D || bits < 1 || bits > kPlanes) return FATHOM_ERR_INVALID_ARG;
    if (H == 0) return FATHOM_OK;
    if (!aligned(q, 4) || !aligned(active, 2) || !aligned(n_active, 4)) return FATHOM_ERR_UNSUPPORTED;
    FATHOM_TRY(check_device_ptr(q));
    FATHOM_TRY(check_device_ptr(depth));
    FATHOM_TRY(check_device_ptr(active));
    FATHOM_TRY(check_device_ptr(n_active));
    return launch_plan_fixed(q, H, G, D, r, bits, depth, active, n_active, reinterpret_cast<cudaStream_t>(stream));
}

size_t fathom_scan_cand_bytes(int64_t H, int G, int64_t n, int k)
{
    if (H <= 0 || G < 1 || G > kMaxG || n <= 0 || k < 1 || k > n) return 0;
    return cand_layout(H, G, n, k).total;
}

int fathom_scan(const uint64_t* planes, const uint16_t* scales, int64_t H, int D, int64_t n, int64_t nb_stride,
                const uint16_t* active, const int32_t* n_active, const float* q, int G, int mode, float* scores,
                void* cand, size_t cand_bytes, int k, fathom_stream_t stream)
{
    NvtxRange range("fathom_scan");
    return fathom::scan_entry(planes, scales, H, D, n, nb_stride, active, n_active, q, G, mode, scores, cand, cand_bytes, k,
                              fathom::kPlanesLayout, stream);
}

int fathom_scan_nibbles(const uint64_t* nibbles, const uint16_t* scales, int64_t H, int D, int64_t n,
                        int64_t nb_stride, const uint16_t* active, const int32_t* n_active, const float* q, int G,
                        int mode, float* scores, void* cand, size_t cand_bytes, int k, fathom_stream_t stream)
{
    NvtxRange range("fathom_scan_nibbles");
    return fathom::scan_entry(nibbles, scales, H, D, n, nb_stride, active, n_active, q, G, mode, scores, cand, cand_bytes, k,
                              fathom::kNibblesLayout, stream);
}

int fathom_scan_nibbles_tm(const uint8_t* store, const uint16_t* scales, int64_t H, int D, int64_t n,
                           int64_t nb_stride, const uint16_t* active, const int32_t* n_active, const float* q, int G,
                           int mode, float* scores, void* cand, size_t cand_bytes, int k, fathom_stream_t stream)
{
    NvtxRange range("fathom_scan_nibbles_tm");
    return fathom::scan_entry(store, scales, H, D, n, nb_stride, active, n_active, q, G, mode, scores, cand, cand_bytes,
                              k, fathom::kTokenMajorLayout, stream);
}

int fathom_nibbles_tm_from_planes(const uint64_t* planes, int64_t H, int D, int64_t n, int64_t nb_stride,
                                  uint8_t* store, fathom_stream_t stream)
{
    NvtxRange range("fathom_nibbles_tm_from_planes");
    if (H < 0 || n < 0 || n >= (1LL << 31)) return FATHOM_ERR_INVALID_ARG;
    if (!dims_ok(D, 1)) return FATHOM_ERR_UNSUPPORTED;
    if (H == 0 || n == 0) return FATHOM_OK;
    const int64_t nb = ceil_div(n, kBlockTokens);
    if (nb_stride < nb) return FATHOM_ERR_INVALID_ARG;
    if (!aligned(planes, 8) || !aligned(store, 16)) return FATHOM_ERR_UNSUPPORTED;
    FATHOM_TRY(check_device_ptr(planes));
    FATHOM_TRY(check_device_ptr(store));
    return launch_tm_from_planes(planes, H, D, n, nb_stride, store, reinterpret_cast<cudaStream_t>(stream));
}

int fathom_nibbles_from_planes(const uint64_t* planes, int64_t H, int D, int64_t n, int64_t nb_stride,
                               uint64_t* nibbles, fathom_stream_t stream)
{
    NvtxRange range("fathom_nibbles_from_planes");
    if (H < 0 || n < 0 || n >= (1LL << 31)) return FATHOM_ERR_INVALID_ARG;
    if (!dims_ok(D, 1)) return FATHOM_ERR_UNSUPPORTED;
    if (H == 0 || n == 0) return FATHOM_OK;
    const int64_t nb = ceil_div(n, kBlockTokens);
    if (nb_stride < nb) return FATHOM_ERR_INVALID_ARG;
    if (!aligned(planes, 8) || !aligned(nibbles, 8)) return FATHOM_ERR_UNSUPPORTED;
    FATHOM_TRY(check_device_ptr(planes));
    FATHOM_TRY(check_device_ptr(nibbles));
    const int64_t total = H * D * nb;
    fathom::nibbles_kernel<<<static_cast<unsigned>(ceil_div(total, 256)), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        planes, H * D, nb, nb_stride, nibbles);
    return launch_status();
}

size_t fathom_topk_workspace_bytes(int64_t H, int G, int64_t n, int k)
{
    (void)H; (void)G; (void)n; (void)k;
    return 0;
}

int fathom_topk(const float* scores, const void* cand, int64_t H, int G, int64_t n, int k, int32_t* idx,
                int32_t* union_idx, int32_t* union_count, void* workspace, size_t ws_bytes,
                fathom_stream_t stream)
{
    NvtxRange range("fathom_topk");
    (void)workspace; (void)ws_bytes;
    if (H < 0 || H > 65535 || n < 0 || n >= (1LL << 31)) return FATHOM_ERR_INVALID_ARG;
    if (G < 1 || G > kMaxG) return FATHOM_ERR_UNSUPPORTED;
    if ((scores == nullptr) == (cand == nullptr)) return FATHOM_ERR_INVALID_ARG;
    if (H == 0) return FATHOM_OK;
    if (k < 1 || k > n) return FATHOM_ERR_INVALID_ARG;
    if (k > kMaxK || static_cast<int64_t>(G) * k > kMaxUnion) return FATHOM_ERR_UNSUPPORTED;
    if (!aligned(idx, 4) || !aligned(union_idx, 4) || !aligned(union_count, 4)) return FATHOM_ERR_UNSUPPORTED;
    if (scores) {
        if (!aligned(scores, 4)) return FATHOM_ERR_UNSUPPORTED;
        FATHOM_TRY(check_device_ptr(scores));
    } else {
        if (k > kMaxCandK) return FATHOM_ERR_UNSUPPORTED;
        if (!aligned(cand, 16)) return FATHOM_ERR_UNSUPPORTED;
        FATHOM_TRY(check_device_ptr(cand));
    }
    FATHOM_TRY(check_device_ptr(idx));
    FATHOM_TRY(check_device_ptr(union_idx));
    FATHOM_TRY(check_device_ptr(union_count));
    return launch_topk(scores, cand, H, G, n, k, idx, union_idx, union_count,
                       reinterpret_cast<cudaStream_t>(stream));
}

int fathom_dequant_rows(const uint64_t* planes, const uint16_t* scales, int64_t H, int D, int64_t n,
                        int64_t nb_stride, const int32_t* rows, int64_t M, const int32_t* row_count, int bits,
                        float* out, fathom_stream_t stream)
{
    NvtxRange range("fathom_dequant_rows");
    if (H < 0 || H > 65535 || n < 0 || n >= (1LL << 31) || M < 0 || M > (1LL << 24)) return FATHOM_ERR_INVALID_ARG;
    if (!dims_ok(D, 1)) return FATHOM_ERR_UNSUPPORTED;
    if (bits < 1 || bits > kPlanes) return FATHOM_ERR_INVALID_ARG;
    if (H == 0 || M == 0) return FATHOM_OK;
    if (nb_stride < ceil_div(n, kBlockTokens)) return FATHOM_ERR_INVALID_ARG;
    if (!aligned(planes, 8) || !aligned(scales, 2) || !aligned(rows, 4) || !aligned(out, 4) ||
        (row_count && !aligned(row_count, 4)))
        return FATHOM_ERR_UNSUPPORTED;
    FATHOM_TRY(check_device_ptr(planes));
    FATHOM_TRY(check_device_ptr(scales));
    FATHOM_TRY(check_device_ptr(rows));
    FATHOM_TRY(check_device_ptr(out));
    if (row_count) FATHOM_TRY(check_device_ptr(row_count));
    return launch_dequant_rows(planes, scales, H, D, n, nb_stride, rows, M, row_count, bits, out,
                               reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
