// fathom_scan: variable-depth scores over the bit-plane index.
//
// What it computes (Fathom, sections "方法一" and "方法二"): for every key
// i < n and each of the group's G query heads,
//   score_{g,i} = sum over active (j, t) of q_{g,j} * s_{b,j} * (2 c_t - 2^t + 1) / 2^t,
// where c_t is the key's t-bit prefix code read from the first t plane rows
// of channel j.  The K bytes are read once for all G heads.
//
// Work layout.  A CTA (4 warps) scores one tile of 16 consecutive 64-token
// blocks of one group.  Active channels are processed in chunks of 32: the
// chunk's plane rows (sum t words per block) and scale rows are staged in
// shared memory with coalesced loads, then every lane scores four tokens of
// one 32-bit half plane word at once:
//   - token bits sit at positions l, l+8, l+16, l+24 of the half word
//     (l = lane & 7); one funnel-shift rotation per plane moves plane p's
//     four bits to bit 7-p of four different bytes, and one AND/OR merges
//     them, so after t planes byte m holds c_t << (8 - t);
//   - a byte permute drops byte m into the low mantissa bits of 1.5 * 2^23,
//     and one FMA with exact constants turns that float into the odd
//     integer 2 c_t - 2^t + 1;
//   - G FMAs per token add coefficient (q_{g,j} 2^-t) * s_{b,j} times it.
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
constexpr int kChunkCh = 32;                     // active channels per staging chunk
constexpr int kChunkRows = kChunkCh * kPlanes;   // plane rows per chunk (max)
constexpr int kBlocksPerWarp = kScanTileBlocks / kScanWarps;  // 4
constexpr int kSets = kBlocksPerWarp / 2;        // a lane set covers 2 blocks

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
    int2* entries;             // [H*G][cap]
    int64_t cap, n_sample, tile_stride;
    int mode;
};

template <int G>
__global__ void __launch_bounds__(kScanThreads)
scan_kernel(const ScanArgs a)
{
    __shared__ uint16_t act_s[kMaxD];
    __shared__ float qs_s[kMaxD * G];
    __shared__ uint16_t rowsrc_s[kChunkRows];       // (j << 2) | p per staged row
    __shared__ __align__(16) uint64_t words_s[kChunkRows * kScanTileBlocks];
    __shared__ uint16_t scale_s[kChunkCh * kScanTileBlocks];
    __shared__ float tau_s[G];

    const int64_t h = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int D = a.D;
    const int na = min(max(a.n_active[h], 0), D);   // trust nothing beyond D entries
    const int64_t tile = static_cast<int64_t>(blockIdx.x) * a.tile_stride;
    const int64_t b0 = tile * kScanTileBlocks;

    // Plan of the group: active (j, t) and coefficients q_{g,j} * 2^-t.
    for (int i = tid; i < na; i += kScanThreads) {
        uint16_t e = a.active[h * D + i];
        int j = e & 0xFF, t = min(e >> 8, kPlanes);
        if (j >= D) t = 0;                  // malformed entry: read nothing
        if (t == 0) j = 0;
        e = static_cast<uint16_t>(j | (t << 8));
        act_s[i] = e;
        const float sc = __uint_as_float(static_cast<uint32_t>(127 - t) << 23);  // 2^-t
#pragma unroll
        for (int g = 0; g < G; ++g) qs_s[i * G + g] = __fmul_rn(a.q[(h * G + g) * D + j], sc);
    }
    if (a.mode == kCandidate && tid < G) tau_s[tid] = a.hdr[h * G + tid].tau;

    // Lane geometry: which block of the warp's pair, which 32-bit half, and
    // the bit offset l of its four tokens l, l+8, l+16, l+24.
    const int blk_in_pair = lane >> 4;
    const int half = (lane >> 3) & 1;
    const int l = lane & 7;

    float acc[kSets][4][G];
#pragma unroll
    for (int s = 0; s < kSets; ++s)
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
            for (int g = 0; g < G; ++g) acc[s][m][g] = 0.0f;

    __syncthreads();

    const uint32_t* words32 = reinterpret_cast<const uint32_t*>(words_s);
    for (int c0 = 0; c0 < na; c0 += kChunkCh) {
        const int nc = min(kChunkCh, na - c0);
        // Row table of the chunk: staged row r comes from plane (j, p).
        if (tid == 0) {
            int r = 0;
            for (int c = 0; c < nc; ++c) {
                const uint16_t e = act_s[c0 + c];
                const int j = e & 0xFF, t = e >> 8;
                for (int p = 0; p < t; ++p) rowsrc_s[r++] = static_cast<uint16_t>((j << 2) | p);
            }
        }
        int rows = 0;
        for (int c = 0; c < nc; ++c) rows += act_s[c0 + c] >> 8;
        __syncthreads();

        // Stage plane words: row r, block b at words_s[r * 16 + b].
        for (int idx = tid; idx < rows * kScanTileBlocks; idx += kScanThreads) {
            const int r = idx / kScanTileBlocks, b = idx % kScanTileBlocks;
            const int src = rowsrc_s[r];
            const int64_t row = (h * D + (src >> 2)) * kPlanes + (src & 3);
            const int64_t blk = b0 + b;
            words_s[r * kScanTileBlocks + b] = blk < a.nb ? __ldg(a.planes + row * a.nb_stride + blk) : 0ull;
        }
        for (int idx = tid; idx < nc * kScanTileBlocks; idx += kScanThreads) {
            const int c = idx / kScanTileBlocks, b = idx % kScanTileBlocks;
            const int j = act_s[c0 + c] & 0xFF;
            const int64_t blk = b0 + b;
            scale_s[c * kScanTileBlocks + b] = blk < a.nb ? __ldg(a.scales + (h * D + j) * a.nb_stride + blk) : 0;
        }
        __syncthreads();

#pragma unroll
        for (int s = 0; s < kSets; ++s) {
            const int blk = warp * kBlocksPerWarp + s * 2 + blk_in_pair;   // block within tile
            int row = 0;
            for (int c = 0; c < nc; ++c) {
                const int t = act_s[c0 + c] >> 8;
                uint32_t code = 0;
#pragma unroll
                for (int p = 0; p < kPlanes; ++p) {
                    if (p < t) {
                        const uint32_t w = words32[(row + p) * (2 * kScanTileBlocks) + blk * 2 + half];
                        const uint32_t x = __funnelshift_l(w, w, (7 - p - l) & 31);
                        code |= x & (0x01010101u << (7 - p));
                    }
                }
                row += t;
                const float sblk = __half2float(__ushort_as_half(scale_s[c * kScanTileBlocks + blk]));
                const float mul = __uint_as_float(static_cast<uint32_t>(120 + t) << 23);  // 2^(t-7)
                const float sub = 1.5f * __uint_as_float(static_cast<uint32_t>(143 + t) << 23) +
                                  static_cast<float>((1 << t) - 1);                    // 1.5*2^(16+t) + 2^t - 1
                float coef[G];
#pragma unroll
                for (int g = 0; g < G; ++g) coef[g] = __fmul_rn(qs_s[(c0 + c) * G + g], sblk);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float f = __uint_as_float(__byte_perm(code, 0x4B400000u, 0x7650u + m));
                    const float v = __fmaf_rn(f, mul, -sub);      // exact odd integer
#pragma unroll
                    for (int g = 0; g < G; ++g) acc[s][m][g] = __fmaf_rn(coef[g], v, acc[s][m][g]);
                }
            }
        }
        __syncthreads();
    }

    // Epilogue.
    const int64_t tok_tile0 = b0 * kBlockTokens;
#pragma unroll
    for (int s = 0; s < kSets; ++s) {
        const int blk = warp * kBlocksPerWarp + s * 2 + blk_in_pair;
        const int local0 = blk * kBlockTokens + half * 32 + l;      // token within tile, m = 0
        if (a.mode == kDense) {
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int64_t i = tok_tile0 + local0 + 8 * m;
                if (i < a.n)
#pragma unroll
                    for (int g = 0; g < G; ++g) a.scores[(h * G + g) * a.n + i] = acc[s][m][g];
            }
        } else if (a.mode == kSample) {
            const int64_t lt = static_cast<int64_t>(blockIdx.x) * kScanTileTokens;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const int64_t i = tok_tile0 + local0 + 8 * m;
#pragma unroll
                for (int g = 0; g < G; ++g)
                    a.sample[(h * G + g) * a.n_sample + lt + local0 + 8 * m] = (i < a.n) ? acc[s][m][g] : -INFINITY;
            }
        } else {
            bool any = false;
#pragma unroll
            for (int m = 0; m < 4; ++m)
#pragma unroll
                for (int g = 0; g < G; ++g)
                    any |= (tok_tile0 + local0 + 8 * m < a.n) && acc[s][m][g] >= tau_s[g];
            if (__any_sync(0xffffffffu, any)) {
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int64_t i = tok_tile0 + local0 + 8 * m;
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const bool p = (i < a.n) && acc[s][m][g] >= tau_s[g];
                        const unsigned mask = __ballot_sync(0xffffffffu, p);
                        if (mask) {
                            const int leader = __ffs(mask) - 1;
                            int base = 0;
                            if (lane == leader) base = atomicAdd(&a.hdr[h * G + g].count, __popc(mask));
                            base = __shfl_sync(0xffffffffu, base, leader);
                            if (p) {
                                const int64_t pos = base + __popc(mask & ((1u << lane) - 1u));
                                if (pos < a.cap)
                                    a.entries[(h * G + g) * a.cap + pos] =
                                        make_int2(static_cast<int>(i), __float_as_int(acc[s][m][g]));
                            }
                        }
                    }
                }
            }
        }
    }
}

template <int G>
int launch_scan_g(const ScanArgs& a, unsigned tiles, unsigned H, cudaStream_t stream)
{
    scan_kernel<G><<<dim3(tiles, H), kScanThreads, 0, stream>>>(a);
    return launch_status();
}

int launch_scan_mode(const ScanArgs& a, int G, unsigned tiles, unsigned H, cudaStream_t stream)
{
    switch (G) {
        case 1: return launch_scan_g<1>(a, tiles, H, stream);
        case 2: return launch_scan_g<2>(a, tiles, H, stream);
        case 3: return launch_scan_g<3>(a, tiles, H, stream);
        case 4: return launch_scan_g<4>(a, tiles, H, stream);
        case 5: return launch_scan_g<5>(a, tiles, H, stream);
        case 6: return launch_scan_g<6>(a, tiles, H, stream);
        case 7: return launch_scan_g<7>(a, tiles, H, stream);
        default: return launch_scan_g<8>(a, tiles, H, stream);
    }
}

}  // namespace

// Defined in topk.cu: per-head threshold selection over the sample.
int launch_tau(const float* sample, CandHeader* hdr, int64_t heads, int64_t n_sample, int64_t m_rank,
               cudaStream_t stream);

CandLayout cand_layout(int64_t H, int G, int64_t n, int k)
{
    CandLayout L{};
    L.heads = H * G;
    const int64_t tiles = ceil_div(n, kScanTileTokens);
    if (n <= 8LL * k || tiles < 2) {
        L.cap = n;
        L.sample_tiles = 0;
        L.tile_stride = 1;
        L.n_sample = 0;
        L.m_rank = 0;
    } else {
        L.cap = 8LL * k;
        int64_t S = k / 16;
        S = S < 1 ? 1 : (S > 32 ? 32 : S);
        if (S > tiles / 2) S = tiles / 2 < 1 ? 1 : tiles / 2;
        L.tile_stride = S;
        L.sample_tiles = ceil_div(tiles, S);
        L.n_sample = L.sample_tiles * kScanTileTokens;
        // expected survivors ~ 4k: the sample holds ~1/S of the keys
        int64_t m = ceil_div(4LL * k * L.sample_tiles, tiles);
        L.m_rank = m < 1 ? 1 : (m > L.n_sample ? L.n_sample : m);
    }
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    L.off_hdr = 0;
    L.off_sample = up(sizeof(CandHeader) * L.heads);
    L.off_entries = L.off_sample + up(sizeof(float) * L.heads * L.n_sample);
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
    const unsigned tiles = static_cast<unsigned>(ceil_div(n, kScanTileTokens));
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
    a.entries = reinterpret_cast<int2*>(base + L.off_entries);
    a.cap = L.cap;
    a.n_sample = L.n_sample;
    if (mode == FATHOM_SCAN_CANDIDATE || mode == FATHOM_SCAN_PREPARE) {
        if (L.sample_tiles > 0) {
            a.mode = kSample;
            a.tile_stride = L.tile_stride;
            int st = launch_scan_mode(a, G, static_cast<unsigned>(L.sample_tiles), static_cast<unsigned>(H), stream);
            if (st) return st;
        }
        int st = launch_tau(a.sample, a.hdr, L.heads, L.n_sample, L.m_rank, stream);
        if (st || mode == FATHOM_SCAN_PREPARE) return st;
    }
    a.mode = kCandidate;
    a.tile_stride = 1;
    return launch_scan_mode(a, G, tiles, static_cast<unsigned>(H), stream);
}

}  // namespace fathom
