// fathom_dequant_rows: reconstruct whole key rows from the bit-plane index.
//
// The union of a KV head's winners is what a decode step fetches next; the
// pages note that a K cache kept as 4-bit channel-major planes could serve
// those winners' keys directly, at the price of gathering one token from
// D x 4 separate plane words (Fathom, section "边界", storage-overhead
// paragraph).  This kernel does that gather: for each listed token i and
// channel j it reads the first `bits` plane words of (j, block i/64) and the
// block scale and writes s * (2 c_t - 2^t + 1) / 2^t, exact in fp32.
//
// Layout: a CTA takes 32 consecutive rows of a group's list and all D
// channels.  Warp w walks channels w, w+8, ...; lane r reads row r of the
// tile, so for ascending lists the lanes of a warp read the same or nearby
// plane words.  Values go through shared memory so that each output row is
// written with coalesced stores.
#include "common.cuh"

namespace fathom {

namespace {

constexpr int kRowsPerCta = 32;
constexpr int kRowsThreads = 256;

__global__ void __launch_bounds__(kRowsThreads)
dequant_rows_kernel(const uint64_t* __restrict__ planes, const uint16_t* __restrict__ scales, int D, int64_t n,
                    int64_t nb_stride, const int32_t* __restrict__ rows, int64_t M,
                    const int32_t* __restrict__ row_count, int bits, float* __restrict__ out)
{
    extern __shared__ float tile[];   // [kRowsPerCta][D + 1]
    const int64_t h = blockIdx.y;
    const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kRowsPerCta;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int64_t count = M;
    if (row_count) {
        const int32_t c = row_count[h];
        count = c < 0 ? 0 : (c > M ? M : c);
    }
    const int64_t r = r0 + lane;
    int64_t tok = -1;
    if (r < count) {
        const int32_t t = rows[h * M + r];
        if (t >= 0 && t < n) tok = t;
    }
    const int64_t b = tok >= 0 ? tok >> 6 : 0;
    const int bit = static_cast<int>(tok & 63);
    const float unit = __uint_as_float(static_cast<uint32_t>(127 - bits) << 23);   // 2^-bits
    for (int j = warp; j < D; j += kRowsThreads / 32) {
        float v = 0.0f;
        if (tok >= 0) {
            const uint64_t* pw = planes + ((h * D + j) * kPlanes) * nb_stride + b;
            int code = 0;
            for (int p = 0; p < bits; ++p) code = (code << 1) | static_cast<int>((__ldg(pw + p * nb_stride) >> bit) & 1);
            const float s = __half2float(__ushort_as_half(__ldg(scales + (h * D + j) * nb_stride + b)));
            v = s * (static_cast<float>(2 * code - (1 << bits) + 1) * unit);   // exact: fp16 x small odd int x 2^-bits
        }
        tile[lane * (D + 1) + j] = v;
    }
    __syncthreads();
    for (int idx = tid; idx < kRowsPerCta * D; idx += kRowsThreads) {
        const int rr = idx / D, j = idx % D;
        if (r0 + rr < M) out[(h * M + r0 + rr) * D + j] = tile[rr * (D + 1) + j];
    }
}

}  // namespace

int launch_dequant_rows(const uint64_t* planes, const uint16_t* scales, int64_t H, int D, int64_t n,
                        int64_t nb_stride, const int32_t* rows, int64_t M, const int32_t* row_count, int bits,
                        float* out, cudaStream_t stream)
{
    const size_t smem = sizeof(float) * kRowsPerCta * (D + 1);
    const int st = ensure_dynamic_smem(reinterpret_cast<const void*>(dequant_rows_kernel), smem);
    if (st) return st;
    const dim3 grid(static_cast<unsigned>(ceil_div(M, kRowsPerCta)), static_cast<unsigned>(H));
    dequant_rows_kernel<<<grid, kRowsThreads, smem, stream>>>(planes, scales, D, n, nb_stride, rows, M, row_count,
                                                              bits, out);
    return launch_status();
}

}  // namespace fathom
