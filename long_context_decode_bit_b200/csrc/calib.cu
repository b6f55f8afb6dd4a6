// fathom_calibrate: per-KV-head key statistics from the session's own keys.
//
// The plan's importance w_j = sigma_j^2 * sum_g q_{g,j}^2 needs the per-channel
// key variance sigma_j^2, measured once on calibration keys (Fathom, section
// "方法二"); the pages also compute the statistics from a session's own
// prefill keys, one covariance per KV head, in under a millisecond at 100k
// tokens (experiments section, calibration-domain paragraph), and a rotated
// basis is the eigenbasis of that covariance (multi-model paragraph).
//
// What is computed, per group h over its first n keys:
//   mean_j  = (1/n) sum_i k_ij
//   var_j   = (1/n) sum_i (k_ij - mean_j)^2        (population variance)
//   cov_ab  = (1/n) sum_i (k_ia - mean_a)(k_ib - mean_b)   (optional)
// in double precision, rounded once to fp32 at the end.  The sums run over
// k - k_0 (the group's first key), which keeps the one-pass form
// E[x^2] - E[x]^2 free of cancellation for keys far from zero.
//
// Layout: `calib_diag_kernel` streams each group's keys once, a CTA per
// chunk of tokens, and adds per-channel double sums into the workspace
// with double atomics.  `calib_cov_kernel` stages tiles of 32 shifted keys
// in shared memory as doubles; each thread owns an 8 x 8 block of the D x D
// matrix and does 64 double FMAs per key.  `calib_finalize_kernel` turns the
// sums into the fp32 outputs.
#include "common.cuh"

namespace fathom {

namespace {

constexpr int kCalThreads = 256;
constexpr int kCovTile = 32;           // keys per shared-memory tile
constexpr int64_t kDiagChunk = 2048;   // keys per CTA, diagonal pass
constexpr int64_t kCovChunk = 1024;    // keys per CTA, covariance pass

template <int DT>
__device__ __forceinline__ double key_value(const void* keys, int64_t off)
{
    if (DT == FATHOM_KEYS_BF16)
        return static_cast<double>(__bfloat162float(static_cast<const __nv_bfloat16*>(keys)[off]));
    return static_cast<double>(static_cast<const float*>(keys)[off]);
}

// Per-channel sums of x = k - k_0 and x^2 over one chunk of one group.
template <int DT>
__global__ void __launch_bounds__(kCalThreads)
calib_diag_kernel(const void* __restrict__ keys, int64_t n, int D, int64_t sh, int64_t st, double* __restrict__ s1,
                  double* __restrict__ s2)
{
    __shared__ double r1[kCalThreads], r2[kCalThreads];
    const int64_t h = blockIdx.y;
    const int tid = threadIdx.x;
    const int rows = kCalThreads / D;          // keys per sweep of the CTA (D <= 256)
    const int r = tid / D, c = tid % D;
    const bool on = r < rows;
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * kDiagChunk;
    const int64_t i1 = min(n, i0 + kDiagChunk);
    double a1 = 0.0, a2 = 0.0;
    if (on) {
        const double k0 = key_value<DT>(keys, h * sh + c);
        for (int64_t i = i0 + r; i < i1; i += rows) {
            const double x = key_value<DT>(keys, h * sh + i * st + c) - k0;
            a1 += x;
            a2 = fma(x, x, a2);
        }
    }
    r1[tid] = a1;
    r2[tid] = a2;
    __syncthreads();
    if (tid < D) {
        double t1 = 0.0, t2 = 0.0;
        for (int q = 0; q < rows; ++q) {
            t1 += r1[q * D + tid];
            t2 += r2[q * D + tid];
        }
        atomicAdd(&s1[h * D + tid], t1);
        atomicAdd(&s2[h * D + tid], t2);
    }
}

// Sums of x_a x_b over one chunk of one group, x = k - k_0, for the 8 x 8
// blocks of the D x D matrix that this CTA's threads own.
template <int DT>
__global__ void __launch_bounds__(kCalThreads, 1)
calib_cov_kernel(const void* __restrict__ keys, int64_t n, int D, int64_t sh, int64_t st, double* __restrict__ s2)
{
    extern __shared__ double tile[];           // [kCovTile][D], then k_0 [D]
    double* k0 = tile + kCovTile * D;
    const int64_t h = blockIdx.y;
    const int tid = threadIdx.x;
    const int nbk = D / 8;
    const int blk = blockIdx.z * kCalThreads + tid;
    const bool on = blk < nbk * nbk;
    const int ra = on ? (blk / nbk) * 8 : 0, cb = on ? (blk % nbk) * 8 : 0;
    const int64_t i0 = static_cast<int64_t>(blockIdx.x) * kCovChunk;
    const int64_t i1 = min(n, i0 + kCovChunk);
    for (int c = tid; c < D; c += kCalThreads) k0[c] = key_value<DT>(keys, h * sh + c);
    double acc[8][8];
#pragma unroll
    for (int x = 0; x < 8; ++x)
#pragma unroll
        for (int y = 0; y < 8; ++y) acc[x][y] = 0.0;
    for (int64_t t0 = i0; t0 < i1; t0 += kCovTile) {
        __syncthreads();   // k_0 written / the previous tile consumed
        for (int e = tid; e < kCovTile * D; e += kCalThreads) {
            const int rr = e / D, c = e % D;
            const int64_t i = t0 + rr;
            tile[e] = i < i1 ? key_value<DT>(keys, h * sh + i * st + c) - k0[c] : 0.0;
        }
        __syncthreads();
        if (on) {
            for (int rr = 0; rr < kCovTile; ++rr) {
                const double* row = tile + rr * D;
                double a[8], b[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) {
                    a[x] = row[ra + x];
                    b[x] = row[cb + x];
                }
#pragma unroll
                for (int x = 0; x < 8; ++x)
#pragma unroll
                    for (int y = 0; y < 8; ++y) acc[x][y] = fma(a[x], b[y], acc[x][y]);
            }
        }
    }
    if (on) {
        double* dst = s2 + h * D * D;
#pragma unroll
        for (int x = 0; x < 8; ++x)
#pragma unroll
            for (int y = 0; y < 8; ++y) atomicAdd(&dst[(ra + x) * D + cb + y], acc[x][y]);
    }
}

// Sums -> fp32 mean, variance and covariance.
template <int DT>
__global__ void __launch_bounds__(kCalThreads)
calib_finalize_kernel(const void* __restrict__ keys, int64_t n, int D, int64_t sh, const double* __restrict__ s1,
                      const double* __restrict__ s2d, const double* __restrict__ s2, float* __restrict__ mean,
                      float* __restrict__ sigma2, float* __restrict__ cov)
{
    const int64_t h = blockIdx.x;
    const double inv = n > 0 ? 1.0 / static_cast<double>(n) : 0.0;
    for (int c = threadIdx.x; c < D; c += blockDim.x) {
        const double m1 = s1[h * D + c] * inv;   // mean of k - k_0
        const double v = fmax(s2d[h * D + c] * inv - m1 * m1, 0.0);
        sigma2[h * D + c] = static_cast<float>(n > 0 ? v : 0.0);
        if (mean) mean[h * D + c] = static_cast<float>(n > 0 ? key_value<DT>(keys, h * sh + c) + m1 : 0.0);
    }
    if (cov) {
        for (int e = threadIdx.x; e < D * D; e += blockDim.x) {
            const int a = e / D, b = e % D;
            const double ma = s1[h * D + a] * inv, mb = s1[h * D + b] * inv;
            cov[h * D * D + e] = static_cast<float>(n > 0 ? s2[h * D * D + e] * inv - ma * mb : 0.0);
        }
    }
}

struct CalLayout {
    size_t off_s1, off_s2d, off_s2, total;
};

CalLayout cal_layout(int64_t H, int D, bool with_cov)
{
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    CalLayout L{};
    L.off_s1 = 0;
    L.off_s2d = up(sizeof(double) * H * D);
    L.off_s2 = L.off_s2d + up(sizeof(double) * H * D);
    L.total = L.off_s2 + (with_cov ? up(sizeof(double) * H * D * D) : 0);
    return L;
}

template <int DT>
int launch_calibrate_t(const void* keys, int64_t H, int64_t n, int D, int64_t sh, int64_t st, float* mean,
                       float* sigma2, float* cov, void* ws, cudaStream_t stream)
{
    const CalLayout L = cal_layout(H, D, cov != nullptr);
    char* base = static_cast<char*>(ws);
    double* s1 = reinterpret_cast<double*>(base + L.off_s1);
    double* s2d = reinterpret_cast<double*>(base + L.off_s2d);
    double* s2 = reinterpret_cast<double*>(base + L.off_s2);
    cudaError_t e = cudaMemsetAsync(ws, 0, L.total, stream);
    if (e != cudaSuccess) return cuda_status(e);
    if (n > 0) {
        const dim3 gd(static_cast<unsigned>(ceil_div(n, kDiagChunk)), static_cast<unsigned>(H));
        calib_diag_kernel<DT><<<gd, kCalThreads, 0, stream>>>(keys, n, D, sh, st, s1, s2d);
        int status = launch_status();
        if (status) return status;
        if (cov) {
            const size_t smem = sizeof(double) * (kCovTile + 1) * D;
            status = ensure_dynamic_smem(reinterpret_cast<const void*>(calib_cov_kernel<DT>), smem);
            if (status) return status;
            const int nbk = D / 8;
            const dim3 gc(static_cast<unsigned>(ceil_div(n, kCovChunk)), static_cast<unsigned>(H),
                          static_cast<unsigned>(ceil_div(static_cast<int64_t>(nbk) * nbk, kCalThreads)));
            calib_cov_kernel<DT><<<gc, kCalThreads, smem, stream>>>(keys, n, D, sh, st, s2);
            status = launch_status();
            if (status) return status;
        }
    }
    calib_finalize_kernel<DT><<<static_cast<unsigned>(H), kCalThreads, 0, stream>>>(keys, n, D, sh, s1, s2d, s2, mean,
                                                                                   sigma2, cov);
    return launch_status();
}

}  // namespace

size_t calibrate_workspace_bytes(int64_t H, int D, bool with_cov) { return cal_layout(H, D, with_cov).total; }

int launch_calibrate(const void* keys, int key_dtype, int64_t H, int64_t n, int D, int64_t sh, int64_t st,
                     float* mean, float* sigma2, float* cov, void* ws, cudaStream_t stream)
{
    if (key_dtype == FATHOM_KEYS_BF16)
        return launch_calibrate_t<FATHOM_KEYS_BF16>(keys, H, n, D, sh, st, mean, sigma2, cov, ws, stream);
    return launch_calibrate_t<FATHOM_KEYS_F32>(keys, H, n, D, sh, st, mean, sigma2, cov, ws, stream);
}

}  // namespace fathom
