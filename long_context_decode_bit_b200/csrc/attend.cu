// fathom_union_attention: softmax attention of each query head over the
// union of its KV head's winners.
//
// A decode step fetches the KV rows of the union of the G heads' top-k (at
// most G*k rows per KV head; Fathom, byte-accounting section) and attends
// over them.  For group h, head g and union rows i:
//   s_i = scale * q_g . K_i,   out_g = sum_i softmax(s)_i V_i.
// K and V are the session's full-precision cache, [H][n][D] (fp32 or bf16).
//
// Layout (split over the union, as in split-K decoding): a CTA takes a
// chunk of up to kAttRows union rows of one group.
//   1. Warp w scores its rows four at a time (all four rows' loads issued
//      before the arithmetic): lane l reads channels l, l+32, ... of a row
//      (64-byte coalesced pieces), keeps G partial dots and reduces them
//      across the warp with butterfly shuffles.
//   2. Warp g turns head g's chunk scores into exp(s - m_g) and their sum.
//   3. Thread t accumulates channel t % D over the rows of its slice
//      (t / D) for all G heads; the slices are summed in shared memory.
// Each chunk leaves (m_g, l_g, o_g) in the workspace; the combine kernel
// rescales them by exp(m_chunk - m_max) and divides by the total weight.
// Everything is fp32 (expf, one rounding per operation).
#include "common.cuh"
#include "ring.cuh"

namespace fathom {

namespace {

constexpr int kAttRows = 256;
constexpr int kAttThreads = 256;
constexpr unsigned kFullMask = 0xffffffffu;

struct AttArgs {
    const void* k;
    const void* v;
    int64_t n, sh, st, M;
    int D;
    const float* q;
    const int32_t* uni;
    const int32_t* count;
    float scale;
    int chunks;
    float* pm;   // [H][chunks][G] chunk maxima
    float* pl;   // [H][chunks][G] chunk weight sums
    float* po;   // [H][chunks][G][D] chunk outputs (unnormalised)
    float* out;  // [H][G][D]
    bool fast;   // D = 128 with 16-byte aligned rows: attend_fast_kernel
};

template <int DT>
__device__ __forceinline__ float kv_at(const void* p, int64_t off)
{
    if (DT == FATHOM_KEYS_BF16) return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[off]);
    return static_cast<const float*>(p)[off];
}

template <int DT, int G>
__global__ void __launch_bounds__(kAttThreads)
attend_chunk_kernel(const AttArgs a)
{
    extern __shared__ __align__(16) float sm[];
    const int D = a.D;
    float* qs = sm;                           // [G][D], scaled
    float* sc = qs + G * D;                   // [G][kAttRows]: scores, then weights
    float* red = sc + G * kAttRows;           // [slices][G][D]
    int* rowi = reinterpret_cast<int*>(red + (kAttThreads / D) * G * D);   // [kAttRows]

    const int64_t h = blockIdx.y;
    const int c = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t cnt = min(max(static_cast<int64_t>(a.count[h]), int64_t{0}), a.M);
    const int64_t r0 = static_cast<int64_t>(c) * kAttRows;
    const int rows = static_cast<int>(max(int64_t{0}, min(static_cast<int64_t>(kAttRows), cnt - r0)));
    const int64_t pbase = (h * a.chunks + c) * G;

    for (int e = tid; e < G * D; e += kAttThreads) qs[e] = a.q[h * G * D + e] * a.scale;
    for (int r = tid; r < rows; r += kAttThreads) {
        const int32_t i = a.uni[h * a.M + r0 + r];
        rowi[r] = (i >= 0 && i < a.n) ? i : -1;   // an index outside the cache scores as absent
    }
    __syncthreads();

    // 1. scores: each warp takes kAttBatch rows at a time and issues all
    // their loads before the arithmetic, so that several rows are in flight.
    constexpr int kAttBatch = 4;
    const int chunks_d = D / 32;   // channels per lane
    for (int r0w = warp * kAttBatch; r0w < rows; r0w += (kAttThreads / 32) * kAttBatch) {
        float kv[kAttBatch][kMaxD / 32];
#pragma unroll
        for (int b = 0; b < kAttBatch; ++b) {
            const int r = r0w + b;
            const int i = r < rows ? rowi[r] : -1;
            const int64_t base = h * a.sh + static_cast<int64_t>(i < 0 ? 0 : i) * a.st;
#pragma unroll
            for (int cc = 0; cc < kMaxD / 32; ++cc)
                kv[b][cc] = (i >= 0 && cc < chunks_d) ? kv_at<DT>(a.k, base + lane + 32 * cc) : 0.0f;
        }
#pragma unroll
        for (int b = 0; b < kAttBatch; ++b) {
            const int r = r0w + b;
            float dot[G];
#pragma unroll
            for (int g = 0; g < G; ++g) dot[g] = 0.0f;
#pragma unroll
            for (int cc = 0; cc < kMaxD / 32; ++cc)
                if (cc < chunks_d)
#pragma unroll
                    for (int g = 0; g < G; ++g) dot[g] = fmaf(qs[g * D + lane + 32 * cc], kv[b][cc], dot[g]);
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) dot[g] += __shfl_xor_sync(kFullMask, dot[g], o);
            if (lane == 0 && r < rows)
#pragma unroll
                for (int g = 0; g < G; ++g) sc[g * kAttRows + r] = rowi[r] >= 0 ? dot[g] : -INFINITY;
        }
    }
    __syncthreads();

    // 2. per-head chunk maximum, weights and their sum (warp g for head g)
    if (warp < G) {
        float* s = sc + warp * kAttRows;
        float m = -INFINITY;
        for (int r = lane; r < rows; r += 32) m = fmaxf(m, s[r]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
        float l = 0.0f;
        for (int r = lane; r < rows; r += 32) {
            const float p = m == -INFINITY ? 0.0f : expf(s[r] - m);
            s[r] = p;
            l += p;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(kFullMask, l, o);
        if (lane == 0) {
            a.pm[pbase + warp] = m;
            a.pl[pbase + warp] = l;
        }
    }
    __syncthreads();

    // 3. weighted value rows
    const int slices = kAttThreads / D;
    const int d = tid % D, sl = tid / D;
    if (sl < slices) {
        float acc[G];
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] = 0.0f;
#pragma unroll 8
        for (int r = sl; r < rows; r += slices) {
            const int i = rowi[r];
            const float vv = i >= 0 ? kv_at<DT>(a.v, h * a.sh + static_cast<int64_t>(i) * a.st + d) : 0.0f;
#pragma unroll
            for (int g = 0; g < G; ++g) acc[g] = fmaf(sc[g * kAttRows + r], vv, acc[g]);
        }
#pragma unroll
        for (int g = 0; g < G; ++g) red[(sl * G + g) * D + d] = acc[g];
    }
    __syncthreads();
    for (int e = tid; e < G * D; e += kAttThreads) {
        float t = 0.0f;
        for (int s2 = 0; s2 < slices; ++s2) t += red[s2 * G * D + e];
        a.po[pbase * D + e] = t;
    }
}

// The same chunk for D = 128 with vector loads and the value rows staged.
// Lane l owns channels 4l .. 4l+3 of every row (one 8-byte bf16 or 16-byte
// fp32 read per row per lane, a whole row per warp instruction); a warp
// scores 8 rows per batch.  When the chunk's value rows fit in 64 KB (bf16),
// the CTA starts copying them into shared memory with 16-byte cp.async
// before it reads the key rows, so the two fetches overlap; the value pass
// then reads shared memory.  Thread t sums rows t/32, t/32 + 8, ... for
// channels 4(t%32) .. +3 and the 8 slices are added in shared memory.
constexpr int kFastD = 128;
constexpr int kFastSlices = kAttThreads / 32;
constexpr int kFastBatch = 8;

template <int DT>
__device__ __forceinline__ void load4(const void* base, int64_t elem, float (&x)[4])
{
    if (DT == FATHOM_KEYS_BF16) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(static_cast<const __nv_bfloat16*>(base) + elem));
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else {
        const float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + elem));
        x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
    }
}

template <int DT>
__device__ __forceinline__ void lds4(const unsigned char* row, int lane, float (&x)[4])
{
    if (DT == FATHOM_KEYS_BF16) {
        const uint2 u = *reinterpret_cast<const uint2*>(row + 8 * lane);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        x[0] = a.x; x[1] = a.y; x[2] = b.x; x[3] = b.y;
    } else {
        const float4 f = *reinterpret_cast<const float4*>(row + 16 * lane);
        x[0] = f.x; x[1] = f.y; x[2] = f.z; x[3] = f.w;
    }
}

template <int DT, int G>
__host__ __device__ constexpr bool fast_stages_v() { return DT == FATHOM_KEYS_BF16; }   // 256 rows x 256 B

template <int DT, int G>
__host__ __device__ constexpr size_t fast_smem_bytes()
{
    constexpr size_t esz = DT == FATHOM_KEYS_BF16 ? 2 : 4;
    constexpr size_t stage = fast_stages_v<DT, G>() ? kAttRows * kFastD * esz : 0;
    constexpr size_t red = sizeof(float) * kFastSlices * G * kFastD;
    return sizeof(float) * (G * kFastD + G * kAttRows) + sizeof(int) * kAttRows + (stage > red ? stage : red);
}

template <int DT, int G>
__global__ void __launch_bounds__(kAttThreads)
attend_fast_kernel(const AttArgs a)
{
    extern __shared__ __align__(16) float sm[];
    constexpr int D = kFastD;
    constexpr size_t esz = DT == FATHOM_KEYS_BF16 ? 2 : 4;
    float* qs = sm;                                             // [G][D], scaled
    float* sc = qs + G * D;                                     // [G][kAttRows]
    int* rowi = reinterpret_cast<int*>(sc + G * kAttRows);      // [kAttRows]
    unsigned char* vs = reinterpret_cast<unsigned char*>(rowi + kAttRows);   // staged V rows, then the slice sums
    float* red = reinterpret_cast<float*>(vs);

    const int64_t h = blockIdx.y;
    const int c = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t cnt = min(max(static_cast<int64_t>(a.count[h]), int64_t{0}), a.M);
    const int64_t r0 = static_cast<int64_t>(c) * kAttRows;
    const int rows = static_cast<int>(max(int64_t{0}, min(static_cast<int64_t>(kAttRows), cnt - r0)));
    const int64_t pbase = (h * a.chunks + c) * G;

    for (int e = tid; e < G * D; e += kAttThreads) qs[e] = a.q[h * G * D + e] * a.scale;
    for (int r = tid; r < rows; r += kAttThreads) {
        const int32_t i = a.uni[h * a.M + r0 + r];
        rowi[r] = (i >= 0 && i < a.n) ? i : -1;
    }
    __syncthreads();

    if (fast_stages_v<DT, G>()) {
        // 16-byte pieces of the value rows (row r at vs + r * D * esz); absent rows are zero-filled.
        constexpr int pieces = D * esz / 16;
        for (int e = tid; e < rows * pieces; e += kAttThreads) {
            const int r = e / pieces, pc = e % pieces;
            const int i = rowi[r];
            const unsigned char* src = static_cast<const unsigned char*>(a.v) +
                                       (h * a.sh + static_cast<int64_t>(i < 0 ? 0 : i) * a.st) * esz + pc * 16;
            cp_async16(vs + (static_cast<size_t>(r) * D * esz + pc * 16), src, i < 0 ? 0 : 16);
        }
    }

    // 1. scores, 8 rows per warp per batch, all loads issued first
    for (int rb = warp * kFastBatch; rb < rows; rb += kFastSlices * kFastBatch) {
        float kv[kFastBatch][4];
#pragma unroll
        for (int b = 0; b < kFastBatch; ++b) {
            const int r = rb + b;
            const int i = r < rows ? rowi[r] : -1;
            if (i >= 0) load4<DT>(a.k, h * a.sh + static_cast<int64_t>(i) * a.st + 4 * lane, kv[b]);
            else kv[b][0] = kv[b][1] = kv[b][2] = kv[b][3] = 0.0f;
        }
#pragma unroll
        for (int b = 0; b < kFastBatch; ++b) {
            const int r = rb + b;
            float dot[G];
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float4 qq = *reinterpret_cast<const float4*>(qs + g * D + 4 * lane);
                dot[g] = fmaf(qq.x, kv[b][0], fmaf(qq.y, kv[b][1], fmaf(qq.z, kv[b][2], qq.w * kv[b][3])));
            }
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) dot[g] += __shfl_xor_sync(kFullMask, dot[g], o);
            if (lane == 0 && r < rows)
#pragma unroll
                for (int g = 0; g < G; ++g) sc[g * kAttRows + r] = rowi[r] >= 0 ? dot[g] : -INFINITY;
        }
    }
    __syncthreads();

    // 2. per-head chunk maximum, weights and their sum (warp g for head g)
    if (warp < G) {
        float* s = sc + warp * kAttRows;
        float m = -INFINITY;
        for (int r = lane; r < rows; r += 32) m = fmaxf(m, s[r]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
        float l = 0.0f;
        for (int r = lane; r < rows; r += 32) {
            const float p = m == -INFINITY ? 0.0f : expf(s[r] - m);
            s[r] = p;
            l += p;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(kFullMask, l, o);
        if (lane == 0) {
            a.pm[pbase + warp] = m;
            a.pl[pbase + warp] = l;
        }
    }
    if (fast_stages_v<DT, G>()) cp_async_wait_all();
    __syncthreads();

    // 3. weighted value rows: slice `warp` takes rows warp, warp + 8, ...
    float acc[4][G];
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
        for (int g = 0; g < G; ++g) acc[e][g] = 0.0f;
#pragma unroll 4
    for (int r = warp; r < rows; r += kFastSlices) {
        float vv[4];
        if (fast_stages_v<DT, G>()) {
            lds4<DT>(vs + static_cast<size_t>(r) * D * esz, lane, vv);
        } else {
            const int i = rowi[r];
            if (i >= 0) load4<DT>(a.v, h * a.sh + static_cast<int64_t>(i) * a.st + 4 * lane, vv);
            else vv[0] = vv[1] = vv[2] = vv[3] = 0.0f;
        }
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float p = sc[g * kAttRows + r];
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[e][g] = fmaf(p, vv[e], acc[e][g]);
        }
    }
    __syncthreads();   // every read of the staged rows is done: the area takes the slice sums
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 4; ++e) red[(warp * G + g) * D + 4 * lane + e] = acc[e][g];
    __syncthreads();
    for (int e = tid; e < G * D; e += kAttThreads) {
        float t = 0.0f;
#pragma unroll
        for (int s2 = 0; s2 < kFastSlices; ++s2) t += red[s2 * G * D + e];
        a.po[pbase * D + e] = t;
    }
}

// Chunks -> normalised output.
template <int G>
__global__ void __launch_bounds__(kAttThreads)
attend_combine_kernel(const AttArgs a)
{
    const int64_t h = blockIdx.x;
    const int D = a.D;
    for (int e = threadIdx.x; e < G * D; e += kAttThreads) {
        const int g = e / D;
        float m = -INFINITY;
        for (int c = 0; c < a.chunks; ++c) m = fmaxf(m, a.pm[(h * a.chunks + c) * G + g]);
        float l = 0.0f, o = 0.0f;
        if (m != -INFINITY) {
            for (int c = 0; c < a.chunks; ++c) {
                const int64_t pc = (h * a.chunks + c) * G + g;
                const float f = a.pm[pc] == -INFINITY ? 0.0f : expf(a.pm[pc] - m);
                l = fmaf(a.pl[pc], f, l);
                o = fmaf(a.po[pc * D + (e % D)], f, o);
            }
        }
        a.out[h * G * D + e] = l > 0.0f ? o / l : 0.0f;
    }
}

template <int DT, int G>
int launch_attend_g(AttArgs a, int64_t H, cudaStream_t stream)
{
    if (a.fast) {
        const size_t smem = fast_smem_bytes<DT, G>();
        int st = ensure_dynamic_smem(reinterpret_cast<const void*>(attend_fast_kernel<DT, G>), smem);
        if (st) return st;
        attend_fast_kernel<DT, G><<<dim3(a.chunks, static_cast<unsigned>(H)), kAttThreads, smem, stream>>>(a);
        st = launch_status();
        if (st) return st;
        attend_combine_kernel<G><<<static_cast<unsigned>(H), kAttThreads, 0, stream>>>(a);
        return launch_status();
    }
    const int slices = kAttThreads / a.D;
    const size_t smem = sizeof(float) * (G * a.D + G * kAttRows + slices * G * a.D) + sizeof(int) * kAttRows;
    int st = ensure_dynamic_smem(reinterpret_cast<const void*>(attend_chunk_kernel<DT, G>), smem);
    if (st) return st;
    attend_chunk_kernel<DT, G><<<dim3(a.chunks, static_cast<unsigned>(H)), kAttThreads, smem, stream>>>(a);
    st = launch_status();
    if (st) return st;
    attend_combine_kernel<G><<<static_cast<unsigned>(H), kAttThreads, 0, stream>>>(a);
    return launch_status();
}

template <int DT>
int launch_attend_dt(const AttArgs& a, int64_t H, int G, cudaStream_t stream)
{
    switch (G) {
        case 1: return launch_attend_g<DT, 1>(a, H, stream);
        case 2: return launch_attend_g<DT, 2>(a, H, stream);
        case 3: return launch_attend_g<DT, 3>(a, H, stream);
        case 4: return launch_attend_g<DT, 4>(a, H, stream);
        case 5: return launch_attend_g<DT, 5>(a, H, stream);
        case 6: return launch_attend_g<DT, 6>(a, H, stream);
        case 7: return launch_attend_g<DT, 7>(a, H, stream);
        default: return launch_attend_g<DT, 8>(a, H, stream);
    }
}

int att_chunks(int64_t M) { return static_cast<int>(ceil_div(M < 1 ? 1 : M, kAttRows)); }

}  // namespace

size_t union_attention_workspace_bytes(int64_t H, int G, int D, int64_t M)
{
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    const size_t cg = static_cast<size_t>(H) * att_chunks(M) * G;
    return 2 * up(sizeof(float) * cg) + up(sizeof(float) * cg * D);
}

int launch_union_attention(const void* k, const void* v, int kv_dtype, int64_t H, int64_t n, int D, int64_t sh,
                           int64_t st, const float* q, int G, const int32_t* uni, const int32_t* count, int64_t M,
                           float scale, float* out, void* ws, cudaStream_t stream)
{
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    AttArgs a{};
    a.k = k;
    a.v = v;
    a.n = n;
    a.sh = sh;
    a.st = st;
    a.M = M;
    a.D = D;
    a.q = q;
    a.uni = uni;
    a.count = count;
    a.scale = scale;
    a.chunks = att_chunks(M);
    const size_t cg = static_cast<size_t>(H) * a.chunks * G;
    char* base = static_cast<char*>(ws);
    a.pm = reinterpret_cast<float*>(base);
    a.pl = reinterpret_cast<float*>(base + up(sizeof(float) * cg));
    a.po = reinterpret_cast<float*>(base + 2 * up(sizeof(float) * cg));
    a.out = out;
    {
        const int64_t esz = kv_dtype == FATHOM_KEYS_BF16 ? 2 : 4;
        auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
        a.fast = D == kFastD && a16(k) && a16(v) && (sh * esz) % 16 == 0 && (st * esz) % 16 == 0;
    }
    if (kv_dtype == FATHOM_KEYS_BF16) return launch_attend_dt<FATHOM_KEYS_BF16>(a, H, G, stream);
    return launch_attend_dt<FATHOM_KEYS_F32>(a, H, G, stream);
}

}  // namespace fathom
