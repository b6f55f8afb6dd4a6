// fathom_pack: per-channel 4-bit codes with fp16 block scales, stored as
// channel-major bit planes (Fathom, bit-plane section "方法一").
//
// One CTA packs a tile of 4 consecutive 64-token blocks x 32 channels of one
// group.  The keys are read token-major (coalesced along channels) into
// shared memory; each warp then owns one channel at a time, forms the block
// maximum with a warp reduction, rounds it to fp16, computes the 64 codes
// (two per lane) and turns each plane into a 64-bit word with two ballots.
// The 16 plane words (4 planes x 4 blocks) of a channel are written by 16
// lanes so that each plane row receives 32 contiguous bytes.
#include "common.cuh"

namespace fathom {

namespace {

constexpr int kPackBlocks = 4;                         // 64-token blocks per tile
constexpr int kPackTokens = kPackBlocks * kBlockTokens; // 256
constexpr int kPackCh = 32;                            // channels per tile
constexpr int kPackThreads = 256;

// The 4-bit code floor(8k/s) + 8, clamped to 0..15, decided exactly: the fp32
// quotient is only a guess, corrected with products e*s that are exact in
// fp32 (|e| <= 17 has at most 5 bits, s is an fp16 value with 11).
__device__ __forceinline__ int code4(float k, float s)
{
    if (!(s > 0.0f) || isinf(s)) return 8;
    const float k8 = 8.0f * k;                 // exact
    float e = floorf(__fdiv_rn(k8, s));
    if (__fmul_rn(e, s) > k8) e -= 1.0f;
    else if (__fmul_rn(e + 1.0f, s) <= k8) e += 1.0f;
    int c = static_cast<int>(e) + 8;
    return min(15, max(0, c));
}

template <typename T>
__device__ __forceinline__ float load_key(const T* p);

template <>
__device__ __forceinline__ float load_key<float>(const float* p) { return __ldg(p); }

template <>
__device__ __forceinline__ float load_key<__nv_bfloat16>(const __nv_bfloat16* p)
{
    return __bfloat162float(__ldg(p));
}

template <typename T>
__global__ void __launch_bounds__(kPackThreads)
pack_kernel(const T* __restrict__ keys, int64_t H, int64_t n, int D, int64_t stride_h,
            int64_t stride_tok, uint64_t* __restrict__ planes, uint16_t* __restrict__ scales,
            int64_t nb_stride, int64_t nb)
{
    __shared__ float tile[kPackTokens][kPackCh + 1];

    const int chunks_per_group = D / kPackCh;
    const int64_t h = blockIdx.y / chunks_per_group;
    const int c0 = (blockIdx.y % chunks_per_group) * kPackCh;
    const int64_t b0 = static_cast<int64_t>(blockIdx.x) * kPackBlocks;
    const int64_t t0 = b0 * kBlockTokens;
    const int tid = threadIdx.x;

    // Stage keys: each warp reads one token row of 32 channels per step.
    const T* kg = keys + h * stride_h + c0;
    for (int idx = tid; idx < kPackTokens * kPackCh; idx += kPackThreads) {
        const int tok = idx / kPackCh, ch = idx % kPackCh;
        const int64_t i = t0 + tok;
        tile[tok][ch] = (i < n) ? load_key(kg + i * stride_tok + ch) : 0.0f;
    }
    __syncthreads();

    const int warp = tid >> 5, lane = tid & 31;
    for (int ch = warp; ch < kPackCh; ch += kPackThreads / 32) {
        const int j = c0 + ch;
        uint64_t my_word = 0;
        uint16_t my_scale = 0;
#pragma unroll
        for (int b = 0; b < kPackBlocks; ++b) {
            const int64_t ilo = t0 + b * kBlockTokens + lane;
            const bool vlo = ilo < n, vhi = (ilo + 32) < n;
            const float klo = tile[b * kBlockTokens + lane][ch];
            const float khi = tile[b * kBlockTokens + 32 + lane][ch];
            float m = fmaxf(vlo ? fabsf(klo) : 0.0f, vhi ? fabsf(khi) : 0.0f);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const __half s16 = __float2half_rn(m);
            const float s = __half2float(s16);
            const int clo = code4(klo, s), chi = code4(khi, s);
#pragma unroll
            for (int p = 0; p < kPlanes; ++p) {
                const uint32_t lo = __ballot_sync(0xffffffffu, vlo && ((clo >> (3 - p)) & 1));
                const uint32_t hi = __ballot_sync(0xffffffffu, vhi && ((chi >> (3 - p)) & 1));
                if (lane == p * kPackBlocks + b) my_word = (static_cast<uint64_t>(hi) << 32) | lo;
            }
            if (lane == b) my_scale = __half_as_ushort(s16);
        }
        const int64_t row = (h * D + j) * kPlanes;
        if (lane < kPlanes * kPackBlocks) {
            const int p = lane / kPackBlocks, b = lane % kPackBlocks;
            if (b0 + b < nb) planes[(row + p) * nb_stride + b0 + b] = my_word;
        }
        if (lane < kPackBlocks && b0 + lane < nb) scales[(h * D + j) * nb_stride + b0 + lane] = my_scale;
    }
}

}  // namespace

int launch_pack(const void* keys, int key_dtype, int64_t H, int64_t n, int D, int64_t stride_h,
                int64_t stride_tok, uint64_t* planes, uint16_t* scales, int64_t nb_stride,
                cudaStream_t stream)
{
    const int64_t nb = ceil_div(n, kBlockTokens);
    const dim3 grid(static_cast<unsigned>(ceil_div(nb, kPackBlocks)),
                    static_cast<unsigned>(H * (D / kPackCh)));
    if (key_dtype == FATHOM_KEYS_F32)
        pack_kernel<float><<<grid, kPackThreads, 0, stream>>>(
            static_cast<const float*>(keys), H, n, D, stride_h, stride_tok, planes, scales, nb_stride, nb);
    else
        pack_kernel<__nv_bfloat16><<<grid, kPackThreads, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(keys), H, n, D, stride_h, stride_tok, planes, scales,
            nb_stride, nb);
    return launch_status();
}

}  // namespace fathom
