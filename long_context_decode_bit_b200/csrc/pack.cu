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

// 16 bytes of keys (8 bf16 or 4 fp32 channels) as floats.
template <typename T>
__device__ __forceinline__ void load16(const T* p, float (&x)[16 / sizeof(T)]);

template <>
__device__ __forceinline__ void load16<float>(const float* p, float (&x)[4])
{
    const float4 v = __ldg(reinterpret_cast<const float4*>(p));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}

template <>
__device__ __forceinline__ void load16<__nv_bfloat16>(const __nv_bfloat16* p, float (&x)[8])
{
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
}

template <typename T, bool VEC>
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

    // Stage keys.  VEC (16-byte aligned rows): each thread reads 16-byte
    // pieces of token rows, all of its reads issued before the stores;
    // otherwise one element per read, a warp per token row.
    const T* kg = keys + h * stride_h + c0;
    if (VEC) {
        constexpr int E = 16 / sizeof(T);                 // channels per piece
        constexpr int kPieces = kPackTokens * kPackCh / E;
        constexpr int kPer = kPieces / kPackThreads;
        float x[kPer][E];
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int idx = tid + u * kPackThreads;
            const int tok = idx / (kPackCh / E), q = idx % (kPackCh / E);
            const int64_t i = t0 + tok;
            if (i < n) load16<T>(kg + i * stride_tok + q * E, x[u]);
            else
#pragma unroll
                for (int e = 0; e < E; ++e) x[u][e] = 0.0f;
        }
#pragma unroll
        for (int u = 0; u < kPer; ++u) {
            const int idx = tid + u * kPackThreads;
            const int tok = idx / (kPackCh / E), q = idx % (kPackCh / E);
#pragma unroll
            for (int e = 0; e < E; ++e) tile[tok][q * E + e] = x[u][e];
        }
    } else {
        for (int idx = tid; idx < kPackTokens * kPackCh; idx += kPackThreads) {
            const int tok = idx / kPackCh, ch = idx % kPackCh;
            const int64_t i = t0 + tok;
            tile[tok][ch] = (i < n) ? load_key(kg + i * stride_tok + ch) : 0.0f;
        }
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

// ---------------------------------------------------------------------
// fathom_pack_rotated: the index of the keys' coordinates in an orthonormal
// basis U (Fathom, section 基座选择: for models without QK-norm the keys
// are stored in the KLT basis and the queries rotated to match).
// Coordinate i of key k is y_i = sum_d k_d U[d][i], accumulated in fp32
// fused multiply-adds in the order d = 0, 1, ..., D-1 from +0: the order is
// part of the definition, so the codes are bit-exact against any evaluation
// of the same chain.  The rotated keys never reach device memory.
//
// One CTA owns C output coordinates of one group and walks the group's
// 64-token blocks; its D x C slice of U stays in shared memory.  Each
// block's keys are staged channel-major (a row of 64 tokens per channel).
// Warp w owns coordinates [w*C/8, (w+1)*C/8); a lane accumulates TOK
// consecutive tokens of one coordinate in registers (float4 reads of the
// staged keys, one U value per step), then quantises them exactly as
// fathom_pack does: the block maximum over the lanes that share the
// coordinate, the fp16 scale, the codes, and each lane's TOK bits of every
// plane word, joined by shuffles.  Cost: D fused multiply-adds per output
// coordinate per token, so the kernel is bound by the FP32 pipe, not HBM.
// ---------------------------------------------------------------------
constexpr int kRotThreads = 256;
constexpr int kRotRow = kBlockTokens + 4;   // staged key row: 64 tokens + pad (16-byte multiple)

template <int C>
size_t rot_smem_bytes(int D)
{
    return sizeof(float) * (static_cast<size_t>(D) * C + static_cast<size_t>(D) * kRotRow);
}

template <typename T, int C>
__global__ void __launch_bounds__(kRotThreads)
pack_rotated_kernel(const T* __restrict__ keys, int64_t n, int D, int64_t stride_h, int64_t stride_tok,
                    const float* __restrict__ U, uint64_t* __restrict__ planes, uint16_t* __restrict__ scales,
                    int64_t nb_stride, int64_t nb)
{
    constexpr int OPW = C / 8;                  // coordinates per warp
    constexpr int TOK = kBlockTokens * OPW / 32; // tokens per lane
    extern __shared__ __align__(16) float rsm[];
    float* Us = rsm;                            // [D][C]
    float* Xs = rsm + static_cast<size_t>(D) * C;   // [D][kRotRow]

    const int chunks = D / C;
    const int64_t h = blockIdx.y / chunks;
    const int c0 = (blockIdx.y % chunks) * C;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cl = warp * OPW + lane % OPW;     // coordinate of the lane within the chunk
    const int qg = lane / OPW;                  // token group of the lane
    const int tok0 = qg * TOK;

    const float* Uh = U + h * static_cast<int64_t>(D) * D;
    for (int i = tid; i < D * C; i += kRotThreads) Us[i] = Uh[static_cast<int64_t>(i / C) * D + c0 + i % C];
    const T* kh = keys + h * stride_h;
    const int j = c0 + cl;

    for (int64_t b = blockIdx.x; b < nb; b += gridDim.x) {
        const int64_t t0 = b * kBlockTokens;
        __syncthreads();   // the previous block's keys are no longer read (and U is staged)
        for (int i = tid; i < kBlockTokens * D; i += kRotThreads) {
            const int t = i / D, d = i % D;
            Xs[d * kRotRow + t] = (t0 + t < n) ? load_key(kh + (t0 + t) * stride_tok + d) : 0.0f;
        }
        __syncthreads();

        // Packed fp32x2 FMAs over token pairs: each half is one IEEE fused
        // multiply-add, so every coordinate still follows the stated chain.
        float2 acc2[TOK / 2];
#pragma unroll
        for (int t = 0; t < TOK / 2; ++t) acc2[t] = make_float2(0.0f, 0.0f);
#pragma unroll 2
        for (int d = 0; d < D; ++d) {
            const float u = Us[d * C + cl];
            const float2 uu = make_float2(u, u);
            const float4* xr = reinterpret_cast<const float4*>(Xs + d * kRotRow + tok0);
#pragma unroll
            for (int v = 0; v < TOK / 4; ++v) {
                const float4 x = xr[v];
                acc2[2 * v] = __ffma2_rn(make_float2(x.x, x.y), uu, acc2[2 * v]);
                acc2[2 * v + 1] = __ffma2_rn(make_float2(x.z, x.w), uu, acc2[2 * v + 1]);
            }
        }
        float acc[TOK];
#pragma unroll
        for (int t = 0; t < TOK / 2; ++t) {
            acc[2 * t] = acc2[t].x;
            acc[2 * t + 1] = acc2[t].y;
        }

        // Block maximum over the valid tokens, across the lanes of this coordinate.
        float m = 0.0f;
#pragma unroll
        for (int t = 0; t < TOK; ++t)
            if (t0 + tok0 + t < n) m = fmaxf(m, fabsf(acc[t]));
#pragma unroll
        for (int o = OPW; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const __half s16 = __float2half_rn(m);
        const float s = __half2float(s16);
        uint32_t piece[kPlanes] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int t = 0; t < TOK; ++t) {
            if (t0 + tok0 + t >= n) continue;
            const int c = code4(acc[t], s);
#pragma unroll
            for (int p = 0; p < kPlanes; ++p) piece[p] |= static_cast<uint32_t>((c >> (3 - p)) & 1) << t;
        }
        // Join the 64 / TOK pieces of each plane word (token group g at bit g*TOK).
        uint64_t word[kPlanes] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
        for (int g = 0; g < 32 / OPW; ++g)
#pragma unroll
            for (int p = 0; p < kPlanes; ++p)
                word[p] |= static_cast<uint64_t>(__shfl_sync(0xffffffffu, piece[p], lane % OPW + g * OPW))
                           << (g * TOK);
        if (qg == 0) {
            const int64_t row = (h * D + j) * kPlanes;
#pragma unroll
            for (int p = 0; p < kPlanes; ++p) planes[(row + p) * nb_stride + b] = word[p];
            scales[(h * D + j) * nb_stride + b] = __half_as_ushort(s16);
        }
    }
}

template <typename T, int C>
int launch_pack_rotated_t(const T* keys, int64_t H, int64_t n, int D, int64_t stride_h, int64_t stride_tok,
                          const float* U, uint64_t* planes, uint16_t* scales, int64_t nb_stride,
                          cudaStream_t stream)
{
    const size_t smem = rot_smem_bytes<C>(D);
    int st = ensure_dynamic_smem(reinterpret_cast<const void*>(pack_rotated_kernel<T, C>), smem);
    if (st) return st;
    int sms = 0;
    st = device_sm_count(&sms);
    if (st) return st;
    const int64_t nb = ceil_div(n, kBlockTokens);
    const int64_t rows = H * (D / C);
    const int per_sm = smem <= 110 * 1024 ? 2 : 1;
    int64_t gx = ceil_div(static_cast<int64_t>(sms) * per_sm * 2, rows);   // about two waves of CTAs
    gx = gx < 1 ? 1 : (gx > nb ? nb : gx);
    const dim3 grid(static_cast<unsigned>(gx), static_cast<unsigned>(rows));
    pack_rotated_kernel<T, C><<<grid, kRotThreads, smem, stream>>>(keys, n, D, stride_h, stride_tok, U, planes,
                                                                   scales, nb_stride, nb);
    return launch_status();
}

template <typename T>
int launch_pack_rotated_c(const T* keys, int64_t H, int64_t n, int D, int64_t stride_h, int64_t stride_tok,
                          const float* U, uint64_t* planes, uint16_t* scales, int64_t nb_stride,
                          cudaStream_t stream)
{
    if (D % 128 == 0)
        return launch_pack_rotated_t<T, 128>(keys, H, n, D, stride_h, stride_tok, U, planes, scales, nb_stride, stream);
    if (D % 64 == 0)
        return launch_pack_rotated_t<T, 64>(keys, H, n, D, stride_h, stride_tok, U, planes, scales, nb_stride, stream);
    return launch_pack_rotated_t<T, 32>(keys, H, n, D, stride_h, stride_tok, U, planes, scales, nb_stride, stream);
}

}  // namespace

int launch_pack_rotated(const void* keys, int key_dtype, int64_t H, int64_t n, int D, int64_t stride_h,
                        int64_t stride_tok, const float* U, uint64_t* planes, uint16_t* scales, int64_t nb_stride,
                        cudaStream_t stream)
{
    if (key_dtype == FATHOM_KEYS_F32)
        return launch_pack_rotated_c(static_cast<const float*>(keys), H, n, D, stride_h, stride_tok, U, planes,
                                     scales, nb_stride, stream);
    return launch_pack_rotated_c(static_cast<const __nv_bfloat16*>(keys), H, n, D, stride_h, stride_tok, U, planes,
                                 scales, nb_stride, stream);
}

int launch_pack(const void* keys, int key_dtype, int64_t H, int64_t n, int D, int64_t stride_h,
                int64_t stride_tok, uint64_t* planes, uint16_t* scales, int64_t nb_stride,
                cudaStream_t stream)
{
    const int64_t nb = ceil_div(n, kBlockTokens);
    const dim3 grid(static_cast<unsigned>(ceil_div(nb, kPackBlocks)),
                    static_cast<unsigned>(H * (D / kPackCh)));
    const int64_t esz = key_dtype == FATHOM_KEYS_F32 ? 4 : 2;
    const bool vec = (reinterpret_cast<uintptr_t>(keys) & 15) == 0 && (stride_tok * esz) % 16 == 0 &&
                     (stride_h * esz) % 16 == 0;
    if (key_dtype == FATHOM_KEYS_F32) {
        const float* k = static_cast<const float*>(keys);
        if (vec) pack_kernel<float, true><<<grid, kPackThreads, 0, stream>>>(k, H, n, D, stride_h, stride_tok, planes, scales, nb_stride, nb);
        else pack_kernel<float, false><<<grid, kPackThreads, 0, stream>>>(k, H, n, D, stride_h, stride_tok, planes, scales, nb_stride, nb);
    } else {
        const __nv_bfloat16* k = static_cast<const __nv_bfloat16*>(keys);
        if (vec) pack_kernel<__nv_bfloat16, true><<<grid, kPackThreads, 0, stream>>>(k, H, n, D, stride_h, stride_tok, planes, scales, nb_stride, nb);
        else pack_kernel<__nv_bfloat16, false><<<grid, kPackThreads, 0, stream>>>(k, H, n, D, stride_h, stride_tok, planes, scales, nb_stride, nb);
    }
    return launch_status();
}

}  // namespace fathom
