// fathom_scan: variable-depth scores over the bit-plane index.
//
// What it computes (Fathom, sections "方法一" and "方法二"): for every key
// i < n and each of the group's G query heads,
//   score_{g,i} = sum over active (j, t) of q_{g,j} * s_{b,j} * (2 c_t - 2^t + 1) / 2^t,
// where c_t is the key's t-bit prefix code read from the first t plane rows
// of channel j.  The K bytes are read once for all G heads.
//
// Work layout.  A CTA (4 warps) walks `tiles_per_cta` consecutive tiles of
// 16 64-token blocks of one group.  Each warp owns 4 blocks of a tile; a
// lane owns 8 tokens of one block: bit positions l, l+8, l+16, l+24
// (l = lane & 7) of the block's low and of its high 32-bit plane half.
//
// Per tile, the active channels (sorted by depth once per CTA) are staged
// in chunks: their plane words go to shared memory with cp.async, laid out
// [block][slot][64-bit word] so that a lane fetches all planes of a channel
// with one or two 128-bit loads; the coefficients (q_{g,j} 2^-t) * s_{b,j}
// of every (channel, block) are computed once into shared memory as
// duplicated pairs for the packed fp32x2 FMA.
//
// Decoding, per channel and per 32-bit half (four tokens at once):
//   - depth 1: one shift moves each token's sign bit to bit 7 of its own
//     byte, one AND/XOR turns the bytes into 0x3F / 0xBF, and one byte
//     permute per token lays that byte over 0x00800000: +-1.0f exactly.
//   - depth t >= 2: one funnel-shift rotation per plane moves plane p's
//     four bits to bit 7-p of four bytes and one AND/OR merges them, so
//     byte m holds c_t << (8-t); a byte permute drops it into the low
//     mantissa of 1.5 * 2^23 and one packed FMA with exact constants gives
//     the odd integers 2 c_t - 2^t + 1 of two tokens.
//   - then G packed FMAs per token pair add coefficient * value.
// There are no tensor cores: the contraction is a gathered, variable-depth
// GEMV whose operand must be decoded bit by bit first.
//
// Output modes: DENSE writes every score; SAMPLE writes the scores of a
// strided subset of tiles to the candidate buffer's sample area; CANDIDATE
// appends (index, score) of keys whose score reaches the head's threshold
// with warp-aggregated atomics.
#include "common.cuh"

namespace fathom {

namespace {

constexpr int kScanThreads = 128;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kBlocksPerWarp = kScanTileBlocks / kScanWarps;  // 4
constexpr int kChunkCh = 40;        // channels per staging chunk
constexpr int kChunkSlots = 64;     // 64-bit plane words per block per chunk
constexpr int kWordStride = kChunkSlots * 8 + 16;  // bytes per staged block (+16 spreads banks)

enum ScanMode { kDense = 0, kSample = 1, kCandidate = 2 };

struct ScanArgs {
    const uint64_t* planes;
    const uint16_t* scales;
    int64_t nb_stride, n, nb;
    int D;
    const uint16_t* active;
    const int32_t* n_active;
    const float* q;
    float* scores;             // dense [H][G][n]
    CandHeader* hdr;           // [H*G]
    float* sample;             // [H*G][n_sample]
    int32_t* tile_counts;      // [H*G][tiles]
    int2* entries;             // [H*G][cap]
    int64_t cap, tslot, n_sample, tile_stride, tiles;
    int tiles_per_cta;
    int mode;
};

// Slots a channel of depth t takes in a staged block: depth 3 and 4 an
// aligned 32-byte quad, depth 2 an aligned 16-byte pair, depth 1 one word.
// Channels are staged in descending depth, so the alignment holds.
__host__ __device__ constexpr int slots_of(int t) { return t >= 3 ? 4 : t; }

// Coefficient pairs stored per (channel, block): G rounded up to even, so
// every record starts on a 16-byte boundary for the 16-byte stores.
template <int G>
__host__ __device__ constexpr int coef_stride() { return (G + 1) & ~1; }

template <int G>
struct SharedScan {
    __align__(16) unsigned char words[2][kScanTileBlocks * kWordStride];   // double-buffered planes
    __align__(16) uint16_t rawscale[2][kChunkCh * kScanTileBlocks];        // double-buffered fp16 scales
    __align__(16) float2 coef[kChunkCh * kScanTileBlocks * coef_stride<G>()];   // duplicated pairs
    float qs[kMaxD * G];             // q_{g,j} * 2^-t, depth-sorted order
    uint16_t chan[kMaxD];            // depth-sorted entries j | t << 8
    uint8_t slot[kMaxD];             // slot of each sorted channel within its chunk
    int16_t chunk_begin[kMaxD + 1];  // chunk boundaries in sorted order
    int16_t chunk_cnt[kMaxD][4];     // per chunk: channels of depth 4, 3, 2, 1
    int n_chunks;
    float tau[G];
    int direct[G];                    // no threshold sample: every key is kept, at its own index
    int tile_cnt[G];                  // survivors of the current tile per head
};

__device__ __forceinline__ void cp_async8(void* smem, const void* gmem, bool valid)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    const int n = valid ? 8 : 0;   // 0: zero fill, nothing is read
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}

// 16-byte copy of which only the first `bytes` (0..16) are read; the rest is zero-filled.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int bytes)
{
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(bytes) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// Depth-1 values of the four tokens of one 32-bit half: +-1.0f.
__device__ __forceinline__ void values_depth1(uint32_t w, int l, float2& v01, float2& v23)
{
    const uint32_t y = ((w << (7 - l)) & 0x80808080u) ^ 0xBFBFBFBFu;
    v01.x = __uint_as_float(__byte_perm(y, 0x00800000u, 0x0654u));
    v01.y = __uint_as_float(__byte_perm(y, 0x00800000u, 0x1654u));
    v23.x = __uint_as_float(__byte_perm(y, 0x00800000u, 0x2654u));
    v23.y = __uint_as_float(__byte_perm(y, 0x00800000u, 0x3654u));
}

// Depth-T (T >= 2) values of four tokens from T plane halves.
template <int T>
__device__ __forceinline__ void values_depth(const uint32_t (&w)[4], int l, float2& v01, float2& v23)
{
    uint32_t code = 0;
#pragma unroll
    for (int p = 0; p < T; ++p) {
        const uint32_t x = __funnelshift_l(w[p], w[p], (7 - p - l) & 31);
        code |= x & (0x01010101u << (7 - p));
    }
    constexpr float mul = static_cast<float>(1u << T) / 128.0f;                          // 2^(t-7)
    constexpr float sub = 1.5f * static_cast<float>(1u << (16 + T)) + static_cast<float>((1u << T) - 1);
    const float2 m2 = make_float2(mul, mul), s2 = make_float2(-sub, -sub);
    float2 f01, f23;
    f01.x = __uint_as_float(__byte_perm(code, 0x4B400000u, 0x7650u));
    f01.y = __uint_as_float(__byte_perm(code, 0x4B400000u, 0x7651u));
    f23.x = __uint_as_float(__byte_perm(code, 0x4B400000u, 0x7652u));
    f23.y = __uint_as_float(__byte_perm(code, 0x4B400000u, 0x7653u));
    v01 = __ffma2_rn(f01, m2, s2);   // exact odd integers
    v23 = __ffma2_rn(f23, m2, s2);
}

// One channel of depth T for the lane's block: 8 tokens (4 pairs) x G heads.
// wrow: the channel's staged words in the lane's block; cf: its G
// duplicated coefficient pairs for that block.
template <int G, int T>
__device__ __forceinline__ void channel_step(const unsigned char* wrow, const float2* cf, int l, float2 (&acc)[4][G])
{
    uint32_t lo[4] = {0, 0, 0, 0}, hi[4] = {0, 0, 0, 0};
    if (T == 1) {
        const uint2 x = *reinterpret_cast<const uint2*>(wrow);
        lo[0] = x.x; hi[0] = x.y;
    } else {
        const uint4 x = *reinterpret_cast<const uint4*>(wrow);
        lo[0] = x.x; hi[0] = x.y; lo[1] = x.z; hi[1] = x.w;
        if (T >= 3) {
            const uint4 y = *reinterpret_cast<const uint4*>(wrow + 16);
            lo[2] = y.x; hi[2] = y.y; lo[3] = y.z; hi[3] = y.w;
        }
    }
    float2 v[4];
    if (T == 1) {
        values_depth1(lo[0], l, v[0], v[1]);
        values_depth1(hi[0], l, v[2], v[3]);
    } else {
        values_depth<T>(lo, l, v[0], v[1]);
        values_depth<T>(hi, l, v[2], v[3]);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const float2 k2 = cf[g];
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) acc[pr][g] = __ffma2_rn(v[pr], k2, acc[pr][g]);
    }
}

// All channels of one depth class of a chunk.
template <int G, int T>
__device__ __forceinline__ void depth_class(const unsigned char* wrow, const float2* cf, int count, int l,
                                            float2 (&acc)[4][G])
{
    for (int i = 0; i < count; ++i) {
        channel_step<G, T>(wrow, cf, l, acc);
        wrow += slots_of(T) * 8;
        cf += kScanTileBlocks * coef_stride<G>();
    }
}

template <int G>
__global__ void __launch_bounds__(kScanThreads, 4)
scan_kernel(const ScanArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SharedScan<G>& S = *reinterpret_cast<SharedScan<G>*>(smem_raw);

    const int64_t h = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int D = a.D;
    const int na = min(max(a.n_active[h], 0), D);   // trust nothing beyond D entries

    // ---- the group's plan, sorted by depth (4, 3, 2, 1), ascending j within a depth
    if (tid < 32) {
        int base = 0;
        for (int t = 4; t >= 1; --t) {
            for (int i0 = 0; i0 < na; i0 += 32) {
                const int i = i0 + lane;
                int j = 0, tt = 0;
                if (i < na) {
                    const uint16_t e = a.active[h * D + i];
                    j = e & 0xFF;
                    tt = min(e >> 8, kPlanes);
                    if (j >= D) tt = 0;       // malformed entry: read nothing
                }
                const unsigned bal = __ballot_sync(0xffffffffu, tt == t);
                if (tt == t) S.chan[base + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint16_t>(j | (t << 8));
                base += __popc(bal);
            }
        }
        __syncwarp();
        // Chunks of at most kChunkCh channels and kChunkSlots staged words.
        if (lane == 0) {
            int c = 0, k = 0;
            while (c < base) {
                S.chunk_begin[k] = static_cast<int16_t>(c);
                int n4 = 0, n3 = 0, n2 = 0, n1 = 0, slots = 0, ch = 0;
                while (c < base && ch < kChunkCh) {
                    const int t = S.chan[c] >> 8;
                    if (slots + slots_of(t) > kChunkSlots) break;
                    S.slot[c] = static_cast<uint8_t>(slots);
                    slots += slots_of(t);
                    n4 += t == 4; n3 += t == 3; n2 += t == 2; n1 += t == 1;
                    ch++;
                    c++;
                }
                S.chunk_cnt[k][0] = static_cast<int16_t>(n4);
                S.chunk_cnt[k][1] = static_cast<int16_t>(n3);
                S.chunk_cnt[k][2] = static_cast<int16_t>(n2);
                S.chunk_cnt[k][3] = static_cast<int16_t>(n1);
                k++;
            }
            if (k == 0) {   // no active channel: one empty chunk, every score is 0
                S.chunk_begin[0] = 0;
                S.chunk_cnt[0][0] = S.chunk_cnt[0][1] = S.chunk_cnt[0][2] = S.chunk_cnt[0][3] = 0;
                k = 1;
            }
            S.chunk_begin[k] = static_cast<int16_t>(c);
            S.n_chunks = k;
        }
    }
    __syncthreads();
    const int n_chunks = S.n_chunks;
    const int nsorted = S.chunk_begin[n_chunks];
    for (int i = tid; i < nsorted; i += kScanThreads) {
        const int j = S.chan[i] & 0xFF, t = S.chan[i] >> 8;
        const float sc = __uint_as_float(static_cast<uint32_t>(127 - t) << 23);  // 2^-t
#pragma unroll
        for (int g = 0; g < G; ++g) S.qs[i * G + g] = __fmul_rn(a.q[(h * G + g) * D + j], sc);
    }
    if (a.mode == kCandidate && tid < G) {
        S.tau[tid] = a.hdr[h * G + tid].tau;
        S.direct[tid] = a.hdr[h * G + tid].n_sample == 0;
        S.tile_cnt[tid] = 0;
    }
    __syncthreads();   // qs and tau visible to every warp, even with no chunk to stage

    const int l = lane & 7;
    const int blk = warp * kBlocksPerWarp + (lane >> 3);   // the lane's block within a tile

    // Tiles of this CTA that exist.
    int64_t tiles_here = a.tiles_per_cta;
    {
        const int64_t first = static_cast<int64_t>(blockIdx.x) * a.tiles_per_cta;
        const int64_t avail = (a.tiles - 1) / a.tile_stride + 1 - first;   // logical tiles left
        if (avail < tiles_here) tiles_here = avail;
    }
    const int units = static_cast<int>(tiles_here) * n_chunks;

    // Stage unit u = (tile, chunk) into buffer `buf`: plane words (8-byte
    // copies, zero-filled past the last block) and raw fp16 scales.
    auto issue = [&](int u, int buf) {
        const int ti = u / n_chunks, ck = u % n_chunks;
        const int64_t ltile = static_cast<int64_t>(blockIdx.x) * a.tiles_per_cta + ti;
        const int64_t b0 = ltile * a.tile_stride * kScanTileBlocks;
        const int c0 = S.chunk_begin[ck], c1 = S.chunk_begin[ck + 1];
        {
            const int b = tid & 15;
            const int64_t blkg = b0 + b;
            const bool valid = blkg < a.nb;
            for (int c = c0 + (tid >> 4); c < c1; c += kScanThreads / 16) {
                const int j = S.chan[c] & 0xFF, t = S.chan[c] >> 8;
                const uint64_t* src = a.planes + (h * D + j) * kPlanes * a.nb_stride + (valid ? blkg : 0);
                unsigned char* dst = S.words[buf] + b * kWordStride + S.slot[c] * 8;
                for (int p = 0; p < t; ++p) cp_async8(dst + p * 8, src + p * a.nb_stride, valid);
            }
        }
        // Scales: two 16-byte copies (8 blocks each) per channel.
        for (int idx = tid; idx < (c1 - c0) * 2; idx += kScanThreads) {
            const int cl = idx >> 1, part = idx & 1;
            const int j = S.chan[c0 + cl] & 0xFF;
            const int64_t first = b0 + part * 8;
            const int64_t nvalid = a.nb - first;
            const int bytes = nvalid >= 8 ? 16 : (nvalid > 0 ? static_cast<int>(nvalid) * 2 : 0);
            const uint16_t* src = a.scales + (h * D + j) * a.nb_stride + (bytes > 0 ? first : 0);
            cp_async16(S.rawscale[buf] + cl * kScanTileBlocks + part * 8, src, bytes);
        }
        cp_async_commit();
    };

    float2 acc[4][G];
    if (units > 0) issue(0, 0);
    for (int u = 0; u < units; ++u) {
        const int buf = u & 1;
        const int ti = u / n_chunks, ck = u % n_chunks;
        if (u + 1 < units) {
            issue(u + 1, buf ^ 1);
            cp_async_wait<1>();
        } else {
            cp_async_wait<0>();
        }
        __syncthreads();   // unit u's words and scales are in place

        const int c0 = S.chunk_begin[ck], c1 = S.chunk_begin[ck + 1];
        // Coefficients of every (channel, block) as duplicated pairs: each
        // thread writes one 16-byte pair of pairs, consecutive threads
        // consecutive 16 bytes.
        constexpr int kPairs = (G + 1) / 2;
        for (int idx = tid; idx < (c1 - c0) * kScanTileBlocks * kPairs; idx += kScanThreads) {
            const int gp = idx % kPairs, cb = idx / kPairs;
            const int cl = cb / kScanTileBlocks, b = cb % kScanTileBlocks;
            const float s = __half2float(__ushort_as_half(S.rawscale[buf][cl * kScanTileBlocks + b]));
            const float* qsc = S.qs + (c0 + cl) * G;
            float2* dst = S.coef + cb * coef_stride<G>() + 2 * gp;
            const float v0 = __fmul_rn(qsc[2 * gp], s);
            if (2 * gp + 1 < G) {
                const float v1 = __fmul_rn(qsc[2 * gp + 1], s);
                *reinterpret_cast<float4*>(dst) = make_float4(v0, v0, v1, v1);
            } else {
                *dst = make_float2(v0, v0);
            }
        }
        __syncthreads();

        if (ck == 0) {
#pragma unroll
            for (int pr = 0; pr < 4; ++pr)
#pragma unroll
                for (int g = 0; g < G; ++g) acc[pr][g] = make_float2(0.0f, 0.0f);
        }
        {
            const int n4 = S.chunk_cnt[ck][0], n3 = S.chunk_cnt[ck][1], n2 = S.chunk_cnt[ck][2],
                      n1 = S.chunk_cnt[ck][3];
            const unsigned char* wrow = S.words[buf] + blk * kWordStride;   // slots start at 0 per chunk
            constexpr int cs = coef_stride<G>();
            const float2* cf = S.coef + blk * cs;
            depth_class<G, 4>(wrow, cf, n4, l, acc);
            wrow += n4 * 32; cf += n4 * kScanTileBlocks * cs;
            depth_class<G, 3>(wrow, cf, n3, l, acc);
            wrow += n3 * 32; cf += n3 * kScanTileBlocks * cs;
            depth_class<G, 2>(wrow, cf, n2, l, acc);
            wrow += n2 * 16; cf += n2 * kScanTileBlocks * cs;
            depth_class<G, 1>(wrow, cf, n1, l, acc);
        }

        if (ck == n_chunks - 1) {
            // ---- epilogue.  acc[pr] holds tokens half*32 + l + 8*m of the lane's
            // block for (half, m) = (pr >> 1, 2*(pr & 1) + e), e = 0 (.x) or 1 (.y).
            const int64_t ltile = static_cast<int64_t>(blockIdx.x) * a.tiles_per_cta + ti;
            const int64_t b0 = ltile * a.tile_stride * kScanTileBlocks;
            const int64_t tok0 = b0 * kBlockTokens + blk * kBlockTokens + l;
            if (a.mode == kDense) {
#pragma unroll
                for (int pr = 0; pr < 4; ++pr)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int64_t i = tok0 + (pr >> 1) * 32 + 8 * (2 * (pr & 1) + e);
                        if (i < a.n)
#pragma unroll
                            for (int g = 0; g < G; ++g)
                                a.scores[(h * G + g) * a.n + i] = e ? acc[pr][g].y : acc[pr][g].x;
                    }
            } else if (a.mode == kSample) {
                const int64_t lt0 = ltile * kScanTileTokens + blk * kBlockTokens + l;
#pragma unroll
                for (int pr = 0; pr < 4; ++pr)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int off = (pr >> 1) * 32 + 8 * (2 * (pr & 1) + e);
                        const bool in = tok0 + off < a.n;
#pragma unroll
                        for (int g = 0; g < G; ++g)
                            a.sample[(h * G + g) * a.n_sample + lt0 + off] =
                                in ? (e ? acc[pr][g].y : acc[pr][g].x) : -INFINITY;
                    }
            } else {
                // Candidates.  Without a threshold sample every key is kept at
                // its own index.  Otherwise survivors go to this tile's fixed
                // slot range (position from a shared counter, no global
                // atomic); the tile's count is written once all warps are done.
                const int64_t ptile = ltile * a.tile_stride;
#pragma unroll
                for (int pr = 0; pr < 4; ++pr)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int64_t i = tok0 + (pr >> 1) * 32 + 8 * (2 * (pr & 1) + e);
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const float sv = e ? acc[pr][g].y : acc[pr][g].x;
                            if (i < a.n && sv >= S.tau[g]) {
                                const int2 ent = make_int2(static_cast<int>(i), __float_as_int(sv));
                                if (S.direct[g]) {
                                    a.entries[(h * G + g) * a.cap + i] = ent;
                                } else {
                                    const int p = atomicAdd(&S.tile_cnt[g], 1);
                                    if (p < a.tslot) a.entries[(h * G + g) * a.cap + ptile * a.tslot + p] = ent;
                                }
                            }
                        }
                    }
                if (a.tslot > 0) {
                    __syncthreads();
                    if (tid < G) {
                        a.tile_counts[(h * G + tid) * a.tiles + ptile] = S.tile_cnt[tid];
                        S.tile_cnt[tid] = 0;
                    }
                }
            }
        }
        __syncthreads();   // buffers of unit u may be refilled from here on
    }

}

template <int G>
int launch_scan_g(ScanArgs a, int64_t ltiles, unsigned H, cudaStream_t stream)
{
    const size_t smem = sizeof(SharedScan<G>);
    const cudaError_t e = cudaFuncSetAttribute(scan_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_status(e);
    // Several tiles per CTA amortise the per-CTA plan set-up, as long as the
    // grid still fills the GPU several times over.
    int64_t per = ltiles * H / 2400;
    a.tiles_per_cta = static_cast<int>(per < 1 ? 1 : (per > 8 ? 8 : per));
    const unsigned gx = static_cast<unsigned>(ceil_div(ltiles, a.tiles_per_cta));
    scan_kernel<G><<<dim3(gx, H), kScanThreads, smem, stream>>>(a);
    return launch_status();
}

int launch_scan_mode(const ScanArgs& a, int G, int64_t ltiles, unsigned H, cudaStream_t stream)
{
    switch (G) {
        case 1: return launch_scan_g<1>(a, ltiles, H, stream);
        case 2: return launch_scan_g<2>(a, ltiles, H, stream);
        case 3: return launch_scan_g<3>(a, ltiles, H, stream);
        case 4: return launch_scan_g<4>(a, ltiles, H, stream);
        case 5: return launch_scan_g<5>(a, ltiles, H, stream);
        case 6: return launch_scan_g<6>(a, ltiles, H, stream);
        case 7: return launch_scan_g<7>(a, ltiles, H, stream);
        default: return launch_scan_g<8>(a, ltiles, H, stream);
    }
}

}  // namespace

// Defined in topk.cu: per-head threshold selection over the sample.
int launch_tau(const float* sample, CandHeader* hdr, int64_t heads, int64_t n_sample, int64_t m_rank,
               int64_t n_keys, cudaStream_t stream);

CandLayout cand_layout(int64_t H, int G, int64_t n, int k)
{
    CandLayout L{};
    L.heads = H * G;
    L.tiles = ceil_div(n, kScanTileTokens);
    if (n <= 8LL * k || L.tiles < 2) {
        L.cap = n;
        L.tslot = 0;
        L.sample_tiles = 0;
        L.tile_stride = 1;
        L.n_sample = 0;
        L.m_rank = 0;
    } else {
        int64_t S = k / 16;
        S = S < 1 ? 1 : (S > 32 ? 32 : S);
        if (S > L.tiles / 2) S = L.tiles / 2 < 1 ? 1 : L.tiles / 2;
        L.tile_stride = S;
        L.sample_tiles = ceil_div(L.tiles, S);
        L.n_sample = L.sample_tiles * kScanTileTokens;
        // tau is the m-th largest sample score; the sample holds ~1/S of the
        // keys, so about 4k keys reach it.
        int64_t m = ceil_div(4LL * k * L.sample_tiles, L.tiles);
        L.m_rank = m < 1 ? 1 : (m > L.n_sample ? L.n_sample : m);
        // Survivor slots per tile: 8x the expected survivors of a tile.
        const int64_t expect = ceil_div(4LL * k * kScanTileTokens, n);
        int64_t ts = 16;
        while (ts < 8 * expect && ts < kScanTileTokens) ts <<= 1;
        L.tslot = ts;
        L.cap = L.tiles * ts;
    }
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    L.off_hdr = 0;
    L.off_sample = up(sizeof(CandHeader) * L.heads);
    L.off_counts = L.off_sample + up(sizeof(float) * L.heads * L.n_sample);
    L.off_entries = L.off_counts + up(sizeof(int32_t) * L.heads * (L.tslot ? L.tiles : 0));
    L.total = L.off_entries + up(sizeof(int2) * L.heads * L.cap);
    return L;
}

int launch_scan(const uint64_t* planes, const uint16_t* scales, int64_t H, int D, int64_t n,
                int64_t nb_stride, const uint16_t* active, const int32_t* n_active, const float* q,
                int G, int mode, float* scores, void* cand, int k, cudaStream_t stream)
{
    ScanArgs a{};
    a.planes = planes;
    a.scales = scales;
    a.nb_stride = nb_stride;
    a.n = n;
    a.nb = ceil_div(n, kBlockTokens);
    a.D = D;
    a.active = active;
    a.n_active = n_active;
    a.q = q;
    const int64_t tiles = ceil_div(n, kScanTileTokens);
    a.tiles = tiles;
    if (mode == FATHOM_SCAN_DENSE) {
        a.scores = scores;
        a.mode = kDense;
        a.tile_stride = 1;
        return launch_scan_mode(a, G, tiles, static_cast<unsigned>(H), stream);
    }
    const CandLayout L = cand_layout(H, G, n, k);
    char* base = static_cast<char*>(cand);
    a.hdr = reinterpret_cast<CandHeader*>(base + L.off_hdr);
    a.sample = reinterpret_cast<float*>(base + L.off_sample);
    a.tile_counts = reinterpret_cast<int32_t*>(base + L.off_counts);
    a.entries = reinterpret_cast<int2*>(base + L.off_entries);
    a.cap = L.cap;
    a.tslot = L.tslot;
    a.n_sample = L.n_sample;
    if (mode == FATHOM_SCAN_CANDIDATE || mode == FATHOM_SCAN_PREPARE) {
        if (L.sample_tiles > 0) {
            a.mode = kSample;
            a.tile_stride = L.tile_stride;
            int st = launch_scan_mode(a, G, L.sample_tiles, static_cast<unsigned>(H), stream);
            if (st) return st;
        }
        int st = launch_tau(a.sample, a.hdr, L.heads, L.n_sample, L.m_rank, n, stream);
        if (st || mode == FATHOM_SCAN_PREPARE) return st;
    }
    a.mode = kCandidate;
    a.tile_stride = 1;
    return launch_scan_mode(a, G, tiles, static_cast<unsigned>(H), stream);
}

}  // namespace fathom
