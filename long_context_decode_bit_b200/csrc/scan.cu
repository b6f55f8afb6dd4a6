// fathom_scan: variable-depth scores over the bit-plane index.
//
// What it computes (Fathom, sections "方法一" and "方法二"): for every key
// i < n and each of the group's G query heads,
//   score_{g,i} = sum over active (j, t) of q_{g,j} * s_{b,j} * (2 c_t - 2^t + 1) / 2^t,
// where c_t is the key's t-bit prefix code read from the first t plane rows
// of channel j.  The K bytes are read once for all G heads.
//
// Work layout.  A CTA is one producer warp and kScanTileBlocks / 4 consumer
// warps working on one group.  The CTA walks `tiles_per_cta` tiles of
// kScanTileBlocks 64-token blocks; the group's active channels (sorted by
// depth once per CTA) are split into chunks, and one (tile, chunk) pair is a
// pipeline unit.
//   - The producer streams each unit's plane rows (one 64-bit word per
//     block, 8 * kScanTileBlocks bytes per row) and fp16 scale rows into a
//     2-stage shared-memory ring with 16-byte cp.async copies.  The copies'
//     completion arrives on the stage's "full" mbarrier; each consumer warp
//     arrives on its "empty" mbarrier when done, so a warp waits only for
//     the data it needs, never for the other consumer warps.
//   - Consumer warp w owns blocks 4w..4w+3 of a tile; a lane owns 8 tokens
//     of one block: bit positions l, l+8, l+16, l+24 (l = lane & 7) of the
//     block's low and of its high 32-bit plane half.  Each warp first forms
//     the coefficients (q_{g,j} 2^-t) * s_{b,j} of its own 4 blocks in a
//     warp-private table, then decodes and accumulates.
//
// Decoding, per channel and per 32-bit half (four tokens at once):
//   - depth 1: one shift moves each token's sign bit to bit 7 of its own
//     byte, one AND/XOR turns the bytes into 0x3F / 0xBF, and one byte
//     permute per token lays that byte over 0x00800000: +-1.0f exactly.
//   - depth t >= 2: one funnel-shift rotation per plane moves plane p's
//     four bits to bit 7-p of four bytes and one AND/OR merges them, so
//     byte m holds c_t << (8-t); a byte permute drops it into the low
//     mantissa of 1.5 * 2^23 and one FMA with exact constants gives the odd
//     integer 2 c_t - 2^t + 1.
//   - then packed fp32x2 FMAs over pairs of heads add coefficient * value.
// There are no tensor cores: the contraction is a gathered, variable-depth
// GEMV whose operand must be decoded bit by bit first.
//
// Output modes: DENSE writes every score; SAMPLE writes the scores of a
// strided subset of tiles to the candidate buffer's sample area; CANDIDATE
// keeps keys whose score reaches the head's threshold: at their own index
// when there is no threshold sample, else in this tile's slot range.
#include <cstdlib>
#include <type_traits>

#include "common.cuh"
#include "ring.cuh"

namespace fathom {

namespace {

constexpr int kConsumerWarps = kScanTileBlocks / 4;            // each consumer warp owns 4 blocks
constexpr int kScanThreads = 32 * (kConsumerWarps + 1);         // + one producer warp
constexpr int kBlocksPerWarp = kScanTileBlocks / kConsumerWarps;  // 4
// Two ring stages (one unit in flight while one is consumed) leave room for
// three CTAs per SM, which measured 1.3% faster than three stages at two
// CTAs per SM.
#ifndef FATHOM_SCAN_STAGES
#define FATHOM_SCAN_STAGES 2
#endif
constexpr int kStages = FATHOM_SCAN_STAGES;
constexpr int kChunkCh = 40;        // channels per chunk
constexpr int kChunkRows = 64;      // plane rows per chunk
constexpr int kRowBytes = kScanTileBlocks * 8;   // one plane row of a tile: 128 or 256 B

#ifndef FATHOM_SCAN_TILES_CAP
#define FATHOM_SCAN_TILES_CAP 32
#endif
constexpr int kMaxTilesPerCta = FATHOM_SCAN_TILES_CAP;

// Named barrier among the consumer warps (0 is __syncthreads).
constexpr int kBarConsumers = 1;

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
    int32_t* fault;            // device fault word: set when a ring wait ran out
    int64_t cap_check;         // entries per head the bounds checks allow (cap; less only in a test build)
    bool nib;                  // `planes` is the nibble store, read at 4 bits
#ifdef FATHOM_TEST_HOOKS
    bool withhold;             // test build: withhold one ring arrival (see the producer)
#endif
};

// Heads are handled in pairs for the packed FMA; odd G gets a zero pad.
template <int G>
__host__ __device__ constexpr int head_pairs() { return (G + 1) / 2; }

// Stored pairs per (channel, block): an even count once there are two or
// more, so that every record starts on 16 bytes for the 16-byte loads.
template <int G>
__host__ __device__ constexpr int coef_pairs() { return head_pairs<G>() == 1 ? 1 : (head_pairs<G>() + 1) & ~1; }

template <int G>
struct SharedScan {
    __align__(16) uint64_t words[kStages][kChunkRows * kScanTileBlocks];     // ring: plane rows
    __align__(16) uint16_t rawscale[kStages][kChunkCh * kScanTileBlocks];    // ring: fp16 scale rows
    __align__(16) float2 coef[kConsumerWarps][kChunkCh * kBlocksPerWarp * coef_pairs<G>()];
    float qs[kMaxD * 2 * head_pairs<G>()];   // q_{g,j} * 2^-t, depth-sorted order, zero-padded heads
    uint16_t chan[kMaxD];            // depth-sorted entries j | t << 8
    uint16_t rowsrc[kMaxD * kPlanes];// plane rows in chunk order: j << 2 | p
    int16_t chunk_begin[kMaxD + 1];  // chunk boundaries in sorted order
    int16_t chunk_row0[kMaxD + 1];   // first row of each chunk
    int16_t chunk_cnt[kMaxD][4];     // per chunk: channels of depth 4, 3, 2, 1
    int n_chunks;
    float tau[G];
    int direct[G];                   // no threshold sample: every key is kept, at its own index
    int tile_cnt[kMaxTilesPerCta][G];// survivors per (tile of this CTA, head), written out at the end
    __align__(8) uint64_t full[kStages];   // ring: data of the stage has landed (32 producer lanes)
    __align__(8) uint64_t empty[kStages];  // ring: every consumer warp is done with the stage
};

// Depth-1 values of the four tokens of one 32-bit half: +-1.0f.
__device__ __forceinline__ void values_depth1(uint32_t w, int l, float (&v)[4])
{
    const uint32_t y = ((w << (7 - l)) & 0x80808080u) ^ 0xBFBFBFBFu;
    v[0] = __uint_as_float(__byte_perm(y, 0x00800000u, 0x0654u));
    v[1] = __uint_as_float(__byte_perm(y, 0x00800000u, 0x1654u));
    v[2] = __uint_as_float(__byte_perm(y, 0x00800000u, 0x2654u));
    v[3] = __uint_as_float(__byte_perm(y, 0x00800000u, 0x3654u));
}

// Depth-T (T >= 2) values of four tokens from T plane halves.
template <int T>
__device__ __forceinline__ void values_depth(const uint32_t (&w)[4], int l, float (&v)[4])
{
    uint32_t code = 0;
#pragma unroll
    for (int p = 0; p < T; ++p) {
        const uint32_t x = __funnelshift_l(w[p], w[p], (7 - p - l) & 31);
        code |= x & (0x01010101u << (7 - p));
    }
    constexpr float mul = static_cast<float>(1u << T) / 128.0f;                          // 2^(t-7)
    constexpr float sub = 1.5f * static_cast<float>(1u << (16 + T)) + static_cast<float>((1u << T) - 1);
#pragma unroll
    for (int m = 0; m < 4; ++m)   // exact odd integers
        v[m] = __fmaf_rn(__uint_as_float(__byte_perm(code, 0x4B400000u, 0x7650u + m)), mul, -sub);
}

__device__ __forceinline__ uint2 lds_u2(uint32_t addr)
{
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];\n" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ float2 lds_f2(uint32_t addr)
{
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];\n" : "=f"(v.x), "=f"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ float4 lds_f4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];\n" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr));
    return v;
}

// One channel of depth T for the lane's block: 8 tokens x G heads.
// The whole 4-bit code c in nibble l of `x` as the exact odd integer
// 2c - 15: one rotation moves the nibble to mantissa bits 19..22 of 1.0f,
// giving 1 + c/16, and one FMA with exact constants finishes (32 + 2c - 47).
// Token values of the nibble store (see channel_values).
__device__ __forceinline__ float value_nibble(uint32_t x, int l)
{
    const uint32_t r = __funnelshift_l(x, x, (19 - 4 * l) & 31);
    const float f = __uint_as_float((r & 0x00780000u) | 0x3F800000u);   // 1 + c/16
    return __fmaf_rn(f, 32.0f, -47.0f);
}

// The 8 token values of one channel of depth T for the lane's block.  wrow:
// shared address of the channel's first row at the lane's block column.
// With NIB the rows are the nibble store's four words per block (word w:
// tokens 16w..16w+15, 4 bits each) and T is 4: slot s of the lane (token
// l + 8s, or 32 + l + 8(s - 4)) is nibble l of the 32-bit half s & 1 of
// word s >> 1.
template <int T, bool NIB>
__device__ __forceinline__ void channel_values(uint32_t wrow, int l, float (&v)[8])
{
    uint32_t lo[4] = {0, 0, 0, 0}, hi[4] = {0, 0, 0, 0};
#pragma unroll
    for (int p = 0; p < T; ++p) {
        const uint2 x = lds_u2(wrow + p * kRowBytes);
        lo[p] = x.x;
        hi[p] = x.y;
    }
    if (NIB) {
#pragma unroll
        for (int w = 0; w < 4; ++w) {
            v[2 * w] = value_nibble(lo[w], l);
            v[2 * w + 1] = value_nibble(hi[w], l);
        }
    } else if (T == 1) {
        values_depth1(lo[0], l, *reinterpret_cast<float(*)[4]>(&v[0]));
        values_depth1(hi[0], l, *reinterpret_cast<float(*)[4]>(&v[4]));
    } else {
        values_depth<T>(lo, l, *reinterpret_cast<float(*)[4]>(&v[0]));
        values_depth<T>(hi, l, *reinterpret_cast<float(*)[4]>(&v[4]));
    }
}

// acc += coefficient * value for the 8 tokens x G heads of one channel.  cf:
// shared address of the channel's head-pair coefficients for the block.
template <int G>
__device__ __forceinline__ void channel_macs(const float (&v)[8], uint32_t cf, float2 (&acc)[8][head_pairs<G>()])
{
    constexpr int GP = head_pairs<G>();
    float2 k[GP];
#pragma unroll
    for (int gp = 0; gp + 1 < GP; gp += 2) {
        const float4 k4 = lds_f4(cf + gp * 8);
        k[gp] = make_float2(k4.x, k4.y);
        k[gp + 1] = make_float2(k4.z, k4.w);
    }
    if (GP & 1) k[GP - 1] = lds_f2(cf + (GP - 1) * 8);
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        const float2 vv = make_float2(v[m], v[m]);
#pragma unroll
        for (int gp = 0; gp < GP; ++gp) acc[m][gp] = __ffma2_rn(vv, k[gp], acc[m][gp]);
    }
}

// All channels of depth T in a chunk.
template <int G, int T, bool NIB>
__device__ __forceinline__ void depth_class(uint32_t& wrow, uint32_t& cf, int count, int l,
                                            float2 (&acc)[8][head_pairs<G>()])
{
    constexpr uint32_t kCf = kBlocksPerWarp * coef_pairs<G>() * 8;
    // Two channels per iteration (fewer loop and address instructions:
    // 2.96 -> 2.90 ms at 288 x 1M, G = 4); G >= 5 keeps one, as two would spill.
    constexpr int kUnroll = G <= 4 ? 2 : 1;
#pragma unroll kUnroll
    for (int i = 0; i < count; ++i) {
        float v[8];
        channel_values<T, NIB>(wrow, l, v);
        channel_macs<G>(v, cf, acc);
        wrow += T * kRowBytes;
        cf += kCf;
    }
}

template <int G>
__device__ __forceinline__ float acc_at(const float2 (&acc)[8][head_pairs<G>()], int m, int g)
{
    return (g & 1) ? acc[m][g >> 1].y : acc[m][g >> 1].x;
}

// Resident CTAs per SM the register budget is sized for: three, except
// for G >= 7, whose 64 accumulator registers per thread need the room of two.
#ifndef FATHOM_SCAN_MIN_CTAS
#define FATHOM_SCAN_MIN_CTAS 3
#endif
template <int G>
__host__ __device__ constexpr int scan_min_ctas() { return G >= 7 ? 2 : FATHOM_SCAN_MIN_CTAS; }

template <int G, bool NIB>
__global__ void __launch_bounds__(kScanThreads, scan_min_ctas<G>())
scan_kernel(const ScanArgs a)
{
    extern __shared__ __align__(16) unsigned char smem_raw[];
    SharedScan<G>& S = *reinterpret_cast<SharedScan<G>*>(smem_raw);
    constexpr int GP = head_pairs<G>();

    const int64_t h = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int D = a.D;
    pdl_wait();
    pdl_launch_dependents();
    const int na = min(max(a.n_active[h], 0), D);   // trust nothing beyond D entries

    // ---- the group's plan: one parallel read of the active list, then a
    // sort by depth (4, 3, 2, 1), ascending j within a depth
    for (int i = tid; i < na; i += kScanThreads) {
        const uint16_t e = a.active[h * D + i];
        const int j = e & 0xFF;
        int tt = NIB ? kPlanes : min(e >> 8, kPlanes);   // the nibble store is read whole
        if (j >= D) tt = 0;       // malformed entry: read nothing
        S.rowsrc[i] = static_cast<uint16_t>(j | (tt << 8));   // staging area until the sort is done
    }
    __syncthreads();
    if (warp == 0) {
        int base = 0;
        for (int t = 4; t >= 1; --t) {
            for (int i0 = 0; i0 < na; i0 += 32) {
                const int i = i0 + lane;
                int j = 0, tt = 0;
                if (i < na) {
                    const uint16_t e = S.rowsrc[i];
                    j = e & 0xFF;
                    tt = e >> 8;
                }
                const unsigned bal = __ballot_sync(0xffffffffu, tt == t);
                if (tt == t) S.chan[base + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint16_t>(j | (t << 8));
                base += __popc(bal);
            }
        }
        __syncwarp();   // every lane has read its entries before lane 0 rewrites rowsrc
        // Chunks of at most kChunkCh channels and kChunkRows plane rows, and
        // the row list (j, p) of every chunk in order.
        if (lane == 0) {
            int c = 0, k = 0, row = 0;
            while (c < base) {
                S.chunk_begin[k] = static_cast<int16_t>(c);
                S.chunk_row0[k] = static_cast<int16_t>(row);
                int n4 = 0, n3 = 0, n2 = 0, n1 = 0, rows = 0, ch = 0;
                while (c < base && ch < kChunkCh) {
                    const int j = S.chan[c] & 0xFF, t = S.chan[c] >> 8;
                    if (rows + t > kChunkRows) break;
                    for (int p = 0; p < t; ++p) S.rowsrc[row + rows + p] = static_cast<uint16_t>((j << 2) | p);
                    rows += t;
                    n4 += t == 4; n3 += t == 3; n2 += t == 2; n1 += t == 1;
                    ch++;
                    c++;
                }
                row += rows;
                S.chunk_cnt[k][0] = static_cast<int16_t>(n4);
                S.chunk_cnt[k][1] = static_cast<int16_t>(n3);
                S.chunk_cnt[k][2] = static_cast<int16_t>(n2);
                S.chunk_cnt[k][3] = static_cast<int16_t>(n1);
                k++;
            }
            if (k == 0) {   // no active channel: one empty chunk, every score is 0
                S.chunk_begin[0] = 0;
                S.chunk_row0[0] = 0;
                S.chunk_cnt[0][0] = S.chunk_cnt[0][1] = S.chunk_cnt[0][2] = S.chunk_cnt[0][3] = 0;
                k = 1;
            }
            S.chunk_begin[k] = static_cast<int16_t>(c);
            S.chunk_row0[k] = static_cast<int16_t>(row);
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
        for (int g = 0; g < 2 * GP; ++g)
            S.qs[i * 2 * GP + g] = g < G ? __fmul_rn(a.q[(h * G + g) * D + j], sc) : 0.0f;
    }
    if (a.mode == kCandidate && tid < G) {
        S.tau[tid] = a.hdr[h * G + tid].tau;
        S.direct[tid] = a.hdr[h * G + tid].n_sample == 0;
    }
    for (int i = tid; i < kMaxTilesPerCta * G; i += kScanThreads) (&S.tile_cnt[0][0])[i] = 0;
    if (tid < kStages) {
        mbar_init(static_cast<uint32_t>(__cvta_generic_to_shared(&S.full[tid])), 32);
        mbar_init(static_cast<uint32_t>(__cvta_generic_to_shared(&S.empty[tid])), kConsumerWarps);
    }
    __syncthreads();   // plan, coefficients' q part, thresholds and ring barriers visible to every warp
    const uint32_t full0 = static_cast<uint32_t>(__cvta_generic_to_shared(&S.full[0]));
    const uint32_t empty0 = static_cast<uint32_t>(__cvta_generic_to_shared(&S.empty[0]));

    // Tiles of this CTA that exist.
    int64_t tiles_here = a.tiles_per_cta;
    {
        const int64_t first = static_cast<int64_t>(blockIdx.x) * a.tiles_per_cta;
        const int64_t avail = (a.tiles - 1) / a.tile_stride + 1 - first;   // logical tiles left
        if (avail < tiles_here) tiles_here = avail;
    }
    const int units = static_cast<int>(tiles_here) * n_chunks;

    if (warp == kConsumerWarps) {
        // ================= producer warp =================
        for (int u = 0; u < units; ++u) {
            const int st = u % kStages;
            if (u >= kStages && !__all_sync(0xffffffffu, mbar_wait(empty0 + 8 * st, ((u / kStages) - 1) & 1))) {
                if (lane == 0) atomicOr(a.fault, 1);   // consumers never freed this stage
                break;
            }
            const int ti = u / n_chunks, ck = u % n_chunks;
            const int64_t ltile = static_cast<int64_t>(blockIdx.x) * a.tiles_per_cta + ti;
            const int64_t b0 = ltile * a.tile_stride * kScanTileBlocks;
            const int64_t valid_blocks = a.nb - b0;   // >= 1
            const int r0 = S.chunk_row0[ck], rows = S.chunk_row0[ck + 1] - r0;
            const int c0 = S.chunk_begin[ck], nc = S.chunk_begin[ck + 1] - c0;
            // Plane rows: pieces of 16 B (2 blocks each), kScanTileBlocks / 2 per row.
            constexpr int kRowPieces = kScanTileBlocks / 2;
            for (int idx = lane; idx < rows * kRowPieces; idx += 32) {
                const int r = idx / kRowPieces, part = idx % kRowPieces;
                const int src_rc = S.rowsrc[r0 + r];
                const int64_t row = (h * D + (src_rc >> 2)) * kPlanes + (src_rc & 3);
                const int64_t vb = valid_blocks - 2 * part;
                const int bytes = vb >= 2 ? 16 : (vb == 1 ? 8 : 0);
                const int64_t col = bytes ? b0 + 2 * part : 0;
                if (bounds_ok(row < static_cast<int64_t>(gridDim.y) * D * kPlanes && col + 2 <= a.nb_stride, a.fault))
                    cp_async16(&S.words[st][r * kScanTileBlocks + 2 * part], a.planes + row * a.nb_stride + col, bytes);
            }
            // Scale rows: pieces of 16 B (8 blocks each), kScanTileBlocks / 8 per channel.
            constexpr int kScalePieces = kScanTileBlocks / 8;
            for (int idx = lane; idx < nc * kScalePieces; idx += 32) {
                const int c = idx / kScalePieces, part = idx % kScalePieces;
                const int j = S.chan[c0 + c] & 0xFF;
                const int64_t vb = valid_blocks - 8 * part;
                const int bytes = vb >= 8 ? 16 : (vb > 0 ? static_cast<int>(vb) * 2 : 0);
                const int64_t col = bytes ? b0 + 8 * part : 0;
                if (bounds_ok(j < D && col + 8 <= a.nb_stride, a.fault))
                    cp_async16(&S.rawscale[st][c * kScanTileBlocks + 8 * part], a.scales + (h * D + j) * a.nb_stride + col,
                               bytes);
            }
#ifdef FATHOM_TEST_HOOKS
            // Test build only: lane 0 of the first CTA of head 0 withholds its
            // arrival for the first unit, so that stage never fills, every
            // consumer wait on it runs out, and then this warp's wait for the
            // stage to be freed runs out too.  Its copies still land (the
            // next arrival and the final wait cover them).
            if (a.withhold && u == 0 && lane == 0 && blockIdx.x == 0 && h == 0) continue;
#endif
            cp_async_arrive(full0 + 8 * st);   // this lane's share of unit u
        }
        cp_async_wait_all();
        return;
    }

    // ================= consumer warps =================
    const int l = lane & 7;
    const int bl = lane >> 3;                      // block of the lane within the warp's 4
    const int blk = warp * kBlocksPerWarp + bl;    // block of the lane within the tile
    float2* wcoef = S.coef[warp];

    float2 acc[8][GP];
    for (int u = 0; u < units; ++u) {
        const int st = u % kStages;
        const int ti = u / n_chunks, ck = u % n_chunks;
        if (!__all_sync(0xffffffffu, mbar_wait(full0 + 8 * st, (u / kStages) & 1))) {   // unit u is in stage st
            if (lane == 0) atomicOr(a.fault, 1);
            break;
        }

        const int c0 = S.chunk_begin[ck], nc = S.chunk_begin[ck + 1] - c0;
        // Coefficients of the warp's 4 blocks: (channel, block) -> G/2 head pairs.
        for (int idx = lane; idx < nc * kBlocksPerWarp; idx += 32) {
            const int c = idx >> 2, b = idx & 3;
            const float s = __half2float(__ushort_as_half(S.rawscale[st][c * kScanTileBlocks + warp * kBlocksPerWarp + b]));
            const float* q2 = S.qs + (c0 + c) * 2 * GP;
            float2* dst = wcoef + (c * kBlocksPerWarp + b) * coef_pairs<G>();
#pragma unroll
            for (int gp = 0; gp < GP; ++gp) dst[gp] = make_float2(__fmul_rn(q2[2 * gp], s), __fmul_rn(q2[2 * gp + 1], s));
        }
        __syncwarp();

        if (ck == 0) {
#pragma unroll
            for (int m = 0; m < 8; ++m)
#pragma unroll
                for (int gp = 0; gp < GP; ++gp) acc[m][gp] = make_float2(0.0f, 0.0f);
        }
        {
            const int n4 = S.chunk_cnt[ck][0], n3 = S.chunk_cnt[ck][1], n2 = S.chunk_cnt[ck][2],
                      n1 = S.chunk_cnt[ck][3];
            uint32_t wrow = static_cast<uint32_t>(__cvta_generic_to_shared(&S.words[st][blk]));  // row 0, lane's block
            uint32_t cf = static_cast<uint32_t>(__cvta_generic_to_shared(wcoef + bl * coef_pairs<G>()));
            depth_class<G, 4, NIB>(wrow, cf, n4, l, acc);
            depth_class<G, 3, NIB>(wrow, cf, n3, l, acc);
            depth_class<G, 2, NIB>(wrow, cf, n2, l, acc);
            depth_class<G, 1, NIB>(wrow, cf, n1, l, acc);
        }
        __syncwarp();   // the warp's coefficient table may be rebuilt after this

        if (ck == n_chunks - 1) {
            // ---- epilogue: token m of the lane is blk*64 + (m >> 2)*32 + l + 8*(m & 3).
            const int64_t ltile = static_cast<int64_t>(blockIdx.x) * a.tiles_per_cta + ti;
            const int64_t b0 = ltile * a.tile_stride * kScanTileBlocks;
            const int64_t tok0 = b0 * kBlockTokens + blk * kBlockTokens + l;
            if (a.mode == kDense) {
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int64_t i = tok0 + (m >> 2) * 32 + 8 * (m & 3);
                    if (i < a.n)
#pragma unroll
                        for (int g = 0; g < G; ++g) a.scores[(h * G + g) * a.n + i] = acc_at<G>(acc, m, g);
                }
            } else if (a.mode == kSample) {
                const int64_t lt0 = ltile * kScanTileTokens + blk * kBlockTokens + l;
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int off = (m >> 2) * 32 + 8 * (m & 3);
                    const bool in = tok0 + off < a.n;
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        if (bounds_ok(lt0 + off < a.n_sample, a.fault))
                            a.sample[(h * G + g) * a.n_sample + lt0 + off] = in ? acc_at<G>(acc, m, g) : -INFINITY;
                }
            } else {
                const int64_t ptile = ltile * a.tile_stride;
                const bool whole = (ltile + 1) * kScanTileTokens <= a.n;   // no token of the tile is past n
                int2* const ent_h = a.entries + h * G * a.cap;
                auto keep = [&](int m, int g, float sv) {
                    const int64_t i = tok0 + (m >> 2) * 32 + 8 * (m & 3);
                    if (!whole && i >= a.n) return;
                    const int2 ent = make_int2(static_cast<int>(i), __float_as_int(sv));
                    if (S.direct[g]) {
                        if (bounds_ok(i < a.cap_check, a.fault)) ent_h[g * a.cap + i] = ent;
                    } else {
                        const int p = atomicAdd(&S.tile_cnt[ti][g], 1);
                        if (p < a.tslot && bounds_ok(ptile * a.tslot + p < a.cap_check, a.fault))
                            ent_h[g * a.cap + ptile * a.tslot + p] = ent;
                    }
                };
                // Survivor mask over (head, token): one compare per score and
                // no branch; then one pass per survivor, usually none.  A NaN
                // score counts as reaching tau, as it ranks above every number
                // in the top-k's order (a head of NaN scores then overflows and
                // is rerun densely).  Without a threshold sample every key is
                // kept, so that each key's own slot is written.
                using Mask = typename std::conditional<(G <= 4), uint32_t, unsigned long long>::type;
                Mask mask = 0;
                if (S.direct[0]) {   // the same for every head of a launch: n alone decides it
                    mask = static_cast<Mask>(~static_cast<Mask>(0) >> (8 * sizeof(Mask) - 8 * G));
                } else {
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float tau = S.tau[g];
#pragma unroll
                        for (int m = 0; m < 8; ++m) mask |= static_cast<Mask>(!(acc_at<G>(acc, m, g) < tau)) << (g * 8 + m);
                    }
                }
                while (mask) {
                    const int bit = (G <= 4 ? __ffs(static_cast<uint32_t>(mask)) : __ffsll(static_cast<long long>(mask))) - 1;
                    mask &= mask - 1;
                    const int g = bit >> 3, m = bit & 7;
                    float sv = 0.0f;
#pragma unroll
                    for (int gg = 0; gg < G; ++gg)
#pragma unroll
                        for (int mm = 0; mm < 8; ++mm)
                            if (gg == g && mm == m) sv = acc_at<G>(acc, mm, gg);
                    keep(m, g, sv);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * st);   // stage st may be refilled
    }
    // Survivor counts of every tile of this CTA, once all consumer warps are done.
    if (a.mode == kCandidate && a.tslot > 0) {
        bar_sync<kBarConsumers, 32 * kConsumerWarps>();
        for (int i = tid; i < tiles_here * G; i += 32 * kConsumerWarps) {
            const int ti = i / G, g = i % G;
            const int64_t ptile = (static_cast<int64_t>(blockIdx.x) * a.tiles_per_cta + ti) * a.tile_stride;
            a.tile_counts[(h * G + g) * a.tiles + ptile] = S.tile_cnt[ti][g];
        }
    }
}

template <int G, bool NIB>
int launch_scan_g(ScanArgs a, int64_t ltiles, unsigned H, cudaStream_t stream)
{
    const size_t smem = sizeof(SharedScan<G>);
    int st = ensure_dynamic_smem(reinterpret_cast<const void*>(scan_kernel<G, NIB>), smem);
    if (st) return st;
    // Several tiles per CTA amortise the per-CTA plan set-up: as many as
    // keep the grid at two or more waves of resident CTAs (capped).
#ifndef FATHOM_SCAN_WAVES
#define FATHOM_SCAN_WAVES 2
#endif
    int sms = 0;
    st = device_sm_count(&sms);
    if (st) return st;
    const int64_t slots = static_cast<int64_t>(sms) * scan_min_ctas<G>() * FATHOM_SCAN_WAVES;
    int64_t per = ceil_div(ltiles * static_cast<int64_t>(H), slots);
    per = per < 1 ? 1 : (per > FATHOM_SCAN_TILES_CAP ? FATHOM_SCAN_TILES_CAP : per);
    per = ceil_div(ltiles, ceil_div(ltiles, per));   // the same CTAs per group, their tiles evened out
    a.tiles_per_cta = static_cast<int>(per);
    const unsigned gx = static_cast<unsigned>(ceil_div(ltiles, a.tiles_per_cta));
    return launch_pdl(scan_kernel<G, NIB>, dim3(gx, H), dim3(kScanThreads), smem, stream, a);
}

template <bool NIB>
int launch_scan_layout(const ScanArgs& a, int G, int64_t ltiles, unsigned H, cudaStream_t stream)
{
    switch (G) {
        case 1: return launch_scan_g<1, NIB>(a, ltiles, H, stream);
        case 2: return launch_scan_g<2, NIB>(a, ltiles, H, stream);
        case 3: return launch_scan_g<3, NIB>(a, ltiles, H, stream);
        case 4: return launch_scan_g<4, NIB>(a, ltiles, H, stream);
        case 5: return launch_scan_g<5, NIB>(a, ltiles, H, stream);
        case 6: return launch_scan_g<6, NIB>(a, ltiles, H, stream);
        case 7: return launch_scan_g<7, NIB>(a, ltiles, H, stream);
        default: return launch_scan_g<8, NIB>(a, ltiles, H, stream);
    }
}

int launch_scan_mode(const ScanArgs& a, int G, int64_t ltiles, unsigned H, cudaStream_t stream)
{
    return a.nib ? launch_scan_layout<true>(a, G, ltiles, H, stream) : launch_scan_layout<false>(a, G, ltiles, H, stream);
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
        int64_t S = k / 8;
        S = S < 1 ? 1 : (S > 64 ? 64 : S);
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
                int G, int mode, float* scores, void* cand, int k, bool nib, cudaStream_t stream)
{
    ScanArgs a{};
    a.nib = nib;
#ifdef FATHOM_TEST_HOOKS
    {
        const char* e = getenv("FATHOM_TEST_WITHHOLD_ARRIVAL");
        a.withhold = e != nullptr && e[0] == '1';
    }
#endif
    {
        const int st = device_fault_word(&a.fault);
        if (st) return st;
    }
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
    a.cap_check = L.cap;
#ifdef FATHOM_TEST_HOOKS
    {
        // Test build only: let the bounds checks allow half the entries, so
        // that a test sees a failed check reach the host as FATHOM_ERR_BOUNDS.
        const char* e = getenv("FATHOM_TEST_SHRINK_CAP");
        if (e != nullptr && e[0] == '1') a.cap_check = L.cap / 2;
    }
#endif
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
