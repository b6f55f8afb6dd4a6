// fathom_nibbles_tm_from_planes / fathom_scan_nibbles_tm: the fixed-depth
// comparator scans (byte-accounting section: SparQ-style r-channel reads at
// 4 bits) over a 4-bit key copy stored TOKEN-MAJOR, as a serving stack
// keeps a 4-bit K cache: each token's D codes form one row of D/2 bytes,
// two channels per byte (channel 2c in the low nibble of byte c).  A scan
// that needs r of the D channels still moves whole rows -- D/2 bytes per
// token per KV head, 64 B at D = 128, whatever r is -- which is the cost
// the channel-major stores (the planes and fathom_scan_nibbles) avoid.
//
// Scores are those of fathom_scan_nibbles: every active channel read at 4
// bits, value (c - 7.5) s/8 with the channel's fp16 block scale s.  Modes,
// candidate buffer and threshold are those of fathom_scan, so fathom_topk
// takes either scan's output.
//
// Work layout.  A CTA of 8 warps walks scan tiles (32 blocks of 64 tokens)
// of one group; warp w owns blocks 4w..4w+3 of a tile and lane l tokens
// l and 32 + l of each.  Each warp streams its blocks' 64 rows into its own
// double-buffered shared area with 16-byte cp.async (one block ahead, across
// tile boundaries), rows padded by 16 bytes so that the lanes' 16-byte reads
// of one chunk of their tokens' rows are conflict-free.  A lane reads each
// 16-byte chunk that holds an active channel once per token and takes the
// chunk's channels word by word (the active channels of each 32-bit word
// are a run of ranks).  No wait crosses warps except the tile-boundary
// barriers.
#include "common.cuh"
#include "ring.cuh"

namespace fathom {

namespace {

constexpr int kTmThreads = 256;
constexpr int kTmWarps = kTmThreads / 32;
constexpr int kTmBlocksPerWarp = kScanTileBlocks / kTmWarps;   // 4
constexpr int kTmMaxTilesPerCta = 32;
// Per-tile coefficient table (32 blocks x active channels x G floats): kept
// when active channels x G <= 128 (e.g. 32 channels at G = 4); larger plans
// keep the tile's scales instead and form each coefficient where it is used.
constexpr int kTmCoefFloats = kScanTileBlocks * 128;
static_assert(sizeof(float) * kTmCoefFloats == sizeof(uint16_t) * kMaxD * kScanTileBlocks, "table and scales share");

enum TmMode { kTmDense = 0, kTmSample = 1, kTmCandidate = 2 };

struct TmArgs {
    const uint8_t* store;      // [H][64 * nb_stride][D/2]
    const uint16_t* scales;    // [H][D][nb_stride] fp16 bits
    int64_t nb_stride, n, nb;
    int D;
    const uint16_t* active;
    const int32_t* n_active;
    const float* q;            // [H][G][D]
    float* scores;             // dense [H][G][n]
    CandHeader* hdr;
    float* sample;
    int32_t* tile_counts;
    int2* entries;
    int64_t cap, tslot, n_sample, tile_stride, tiles;
    int tiles_per_cta;
    int mode;
    int32_t* fault;            // device fault word (bounds bit of the debug build)
};

template <int G>
struct SharedTm {
    float qv[kMaxD * 2 * ((G + 1) / 2)];        // q_{g,j} / 16 by active rank, heads padded to pairs
    uint16_t chan[kMaxD];                       // channel of each active rank
    union __align__(16) {
        uint16_t sc[kMaxD * kScanTileBlocks];   // the tile's fp16 scales: [rank][block] (large plans)
        float coef[kTmCoefFloats];              // or its q_{g,j} s_{j,b} / 16: [block][rank][head, pairs padded]
    };
    int wrank[kMaxD / 8 + 1];                   // rank of the first active channel of each 32-bit word
    uint8_t rot[kMaxD];                         // per rank: right rotation putting the code at bits 1..4
    float tau[G];
    int direct[G];
    int tile_cnt[kTmMaxTilesPerCta][G];
};

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory"); }

// 2c - 15 for the 4-bit code c at bits 4s .. 4s + 3 of w, given rot = 4s - 1
// mod 32: the rotation puts 2c at bits 1..4, and 2^23 + 2c - (2^23 + 15) is
// exact.
__device__ __forceinline__ float tm_value(uint32_t w, uint32_t rot)
{
    return __uint_as_float(0x4B000000u | (__funnelshift_r(w, w, rot) & 0x1Eu)) - 8388623.0f;
}

// Shared bytes of one staged row (D/2 bytes + 16 bytes of pad), and of a CTA.
__host__ __device__ inline int tm_pitch(int D) { return D / 2 + 16; }

template <int G>
__host__ __device__ constexpr size_t tm_shared_head() { return (sizeof(SharedTm<G>) + 15) & ~static_cast<size_t>(15); }

template <int G>
size_t tm_smem_bytes(int D)
{
    return tm_shared_head<G>() + static_cast<size_t>(kTmWarps) * 2 * kBlockTokens * tm_pitch(D);
}

// Two CTAs per SM, except for G >= 5, whose 8 G accumulators per thread need
// the registers of one.
template <int G>
__host__ __device__ constexpr int tm_min_ctas() { return G >= 5 ? 1 : 2; }

template <int G>
__global__ void __launch_bounds__(kTmThreads, tm_min_ctas<G>())
scan_tm_kernel(const TmArgs a)
{
    extern __shared__ __align__(16) unsigned char tm_smem[];
    SharedTm<G>& S = *reinterpret_cast<SharedTm<G>*>(tm_smem);
    constexpr int GP = (G + 1) / 2, GQ = 2 * GP;   // head pairs; heads padded to pairs

    const int64_t h = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait();
    pdl_launch_dependents();
    const int D = a.D;
    const int na = min(max(a.n_active[h], 0), D);
    for (int r = tid; r < na; r += kTmThreads) {
        int j = a.active[h * D + r] & 0xFF;
        if (j >= D) j = 0;   // malformed entry: read channel 0 with a zero weight
        const bool ok = (a.active[h * D + r] & 0xFF) < D;
        S.chan[r] = static_cast<uint16_t>(j);
#pragma unroll
        for (int g = 0; g < GQ; ++g) S.qv[r * GQ + g] = (ok && g < G) ? __fmul_rn(a.q[(h * G + g) * D + j], 0.0625f) : 0.0f;
    }
    if (a.mode == kTmCandidate && tid < G) {
        S.tau[tid] = a.hdr[h * G + tid].tau;
        S.direct[tid] = a.hdr[h * G + tid].n_sample == 0;
    }
    for (int i = tid; i < kTmMaxTilesPerCta * G; i += kTmThreads) (&S.tile_cnt[0][0])[i] = 0;
    __syncthreads();   // chan[] complete
    if (warp == 0) {
        // First rank of each 32-bit word of the row (8 channels; the active
        // list is ascending in j, so a word's channels have consecutive ranks).
        const int nw = D / 8;
        int cnt = 0;
        for (int r = 0; r < na; ++r) cnt += (S.chan[r] >> 3) == lane;
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane < nw) S.wrank[lane] = incl - cnt;
        if (lane == 0) S.wrank[nw] = na;
    }
    for (int r = tid; r < na; r += kTmThreads) S.rot[r] = static_cast<uint8_t>((4 * (S.chan[r] & 7) + 31) & 31);
    int64_t tiles_here = a.tiles_per_cta;
    {
        const int64_t first = static_cast<int64_t>(blockIdx.x) * a.tiles_per_cta;
        const int64_t avail = (a.tiles - 1) / a.tile_stride + 1 - first;
        if (avail < tiles_here) tiles_here = avail;
    }
    const uint8_t* st_h = a.store + h * a.nb_stride * kBlockTokens * (D / 2);
    const bool table = na * GQ <= kTmCoefFloats / kScanTileBlocks;

    const int rowb = D / 2, pitch = tm_pitch(D), cpr = D / 32;   // row bytes, staged pitch, 16-byte chunks
    unsigned char* mybuf = tm_smem + tm_shared_head<G>() + static_cast<size_t>(warp) * 2 * kBlockTokens * pitch;
    const int total_u = static_cast<int>(tiles_here) * kTmBlocksPerWarp;
    // Rows of the warp's unit u (tile u / 4, block 4w + u % 4) into buffer u & 1.
    auto issue = [&](int u) {
        if (u < total_u) {
            const int64_t b0u = (static_cast<int64_t>(blockIdx.x) * a.tiles_per_cta + u / kTmBlocksPerWarp) *
                                a.tile_stride * kScanTileBlocks;
            const int bl = warp * kTmBlocksPerWarp + u % kTmBlocksPerWarp;
            if (bl < a.nb - b0u && bounds_ok(b0u + bl < a.nb_stride, a.fault)) {
                const unsigned char* src = st_h + (b0u + bl) * kBlockTokens * rowb;
                unsigned char* dst = mybuf + (u & 1) * kBlockTokens * pitch;
                for (int e = lane; e < kBlockTokens * cpr; e += 32) {
                    const int t = e / cpr, c = e % cpr;
                    cp_async16(dst + t * pitch + c * 16, src + t * rowb + c * 16, 16);
                }
            }
        }
        cp_async_commit();
    };
    issue(0);

    for (int ti = 0; ti < tiles_here; ++ti) {
        const int64_t ltile = static_cast<int64_t>(blockIdx.x) * a.tiles_per_cta + ti;
        const int64_t ptile = ltile * a.tile_stride;
        const int64_t b0 = ptile * kScanTileBlocks;
        const int64_t valid_blocks = a.nb - b0;   // >= 1
        __syncthreads();   // the plan (first tile) is visible; the last tile's scales are no longer read
        if (table) {
            for (int i = tid; i < kScanTileBlocks * na * GQ; i += kTmThreads) {
                const int bl = i / (na * GQ), rg = i % (na * GQ), r = rg / GQ;
                const uint16_t sb = bl < valid_blocks ? a.scales[(h * D + S.chan[r]) * a.nb_stride + b0 + bl] : 0;
                S.coef[i] = __fmul_rn(S.qv[rg], __half2float(__ushort_as_half(sb)));
            }
        } else {
            for (int i = tid; i < na * kScanTileBlocks; i += kTmThreads) {
                const int r = i / kScanTileBlocks, bl = i % kScanTileBlocks;
                S.sc[i] = bl < valid_blocks ? a.scales[(h * D + S.chan[r]) * a.nb_stride + b0 + bl] : 0;
            }
        }
        __syncthreads();

        float2 acc[2 * kTmBlocksPerWarp][GP];   // head pairs, for the packed FMA
#pragma unroll
        for (int m = 0; m < 2 * kTmBlocksPerWarp; ++m)
#pragma unroll
            for (int gp = 0; gp < GP; ++gp) acc[m][gp] = make_float2(0.0f, 0.0f);
        auto acc_g = [&](int m, int g) { return (g & 1) ? acc[m][g >> 1].y : acc[m][g >> 1].x; };
#pragma unroll
        for (int i = 0; i < kTmBlocksPerWarp; ++i) {
            issue(ti * kTmBlocksPerWarp + i + 1);
            cp_async_wait_group<1>();   // this lane's copies of unit ti*4 + i have landed
            __syncwarp();               // and so have the other lanes'
            const int bl = warp * kTmBlocksPerWarp + i;
            if (bl < valid_blocks) {
                const unsigned char* rb = mybuf + (i & 1) * kBlockTokens * pitch;
                const float2* cf = reinterpret_cast<const float2*>(S.coef + bl * na * GQ);
                for (int ck = 0; ck < cpr; ++ck) {
                    if (S.wrank[4 * ck] == S.wrank[4 * ck + 4]) continue;   // no active channel in the chunk
                    const uint4 x0 = *reinterpret_cast<const uint4*>(rb + lane * pitch + ck * 16);
                    const uint4 x1 = *reinterpret_cast<const uint4*>(rb + (32 + lane) * pitch + ck * 16);
                    const uint32_t w0s[4] = {x0.x, x0.y, x0.z, x0.w}, w1s[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
                    for (int wi = 0; wi < 4; ++wi) {   // the chunk's words: channels 8 (4 ck + wi) ..
                        const int r1 = S.wrank[4 * ck + wi + 1];
                        for (int r = S.wrank[4 * ck + wi]; r < r1; ++r) {
                            const uint32_t rt = S.rot[r];
                            const float v0 = tm_value(w0s[wi], rt), v1 = tm_value(w1s[wi], rt);
                            float2 k[GP];
                            if (table) {
#pragma unroll
                                for (int gp = 0; gp < GP; ++gp) k[gp] = cf[r * GP + gp];
                            } else {
                                const float s = __half2float(__ushort_as_half(S.sc[r * kScanTileBlocks + bl]));
#pragma unroll
                                for (int gp = 0; gp < GP; ++gp)
                                    k[gp] = make_float2(__fmul_rn(S.qv[r * GQ + 2 * gp], s),
                                                        __fmul_rn(S.qv[r * GQ + 2 * gp + 1], s));
                            }
                            const float2 vv0 = make_float2(v0, v0), vv1 = make_float2(v1, v1);
#pragma unroll
                            for (int gp = 0; gp < GP; ++gp) {
                                acc[2 * i][gp] = __ffma2_rn(vv0, k[gp], acc[2 * i][gp]);
                                acc[2 * i + 1][gp] = __ffma2_rn(vv1, k[gp], acc[2 * i + 1][gp]);
                            }
                        }
                    }
                }
            }
            __syncwarp();   // the buffer is read before the copy two units on refills it
        }

        // Epilogue: slot m of the lane is token 64 (4w + m/2) + 32 (m & 1) + l of the tile.
        const int64_t tile_tok0 = b0 * kBlockTokens;
        if (a.mode == kTmDense) {
#pragma unroll
            for (int m = 0; m < 2 * kTmBlocksPerWarp; ++m) {
                const int64_t i = tile_tok0 + 64 * (warp * kTmBlocksPerWarp + m / 2) + 32 * (m & 1) + lane;
                if (i < a.n)
#pragma unroll
                    for (int g = 0; g < G; ++g) a.scores[(h * G + g) * a.n + i] = acc_g(m, g);
            }
        } else if (a.mode == kTmSample) {
#pragma unroll
            for (int m = 0; m < 2 * kTmBlocksPerWarp; ++m) {
                const int tl = 64 * (warp * kTmBlocksPerWarp + m / 2) + 32 * (m & 1) + lane;
                const bool in = tile_tok0 + tl < a.n;
#pragma unroll
                for (int g = 0; g < G; ++g)
                    a.sample[(h * G + g) * a.n_sample + ltile * kScanTileTokens + tl] = in ? acc_g(m, g) : -INFINITY;
            }
        } else {
            int2* const ent_h = a.entries + h * G * a.cap;
#pragma unroll
            for (int m = 0; m < 2 * kTmBlocksPerWarp; ++m) {
                const int64_t i = tile_tok0 + 64 * (warp * kTmBlocksPerWarp + m / 2) + 32 * (m & 1) + lane;
                if (i >= a.n) continue;
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float sv = acc_g(m, g);
                    const int2 ent = make_int2(static_cast<int>(i), __float_as_int(sv));
                    if (S.direct[g]) {
                        if (bounds_ok(i < a.cap, a.fault)) ent_h[g * a.cap + i] = ent;
                    } else if (!(sv < S.tau[g])) {   // a NaN score counts as reaching tau
                        const int p = atomicAdd(&S.tile_cnt[ti][g], 1);
                        if (p < a.tslot && bounds_ok(ptile * a.tslot + p < a.cap, a.fault))
                            ent_h[g * a.cap + ptile * a.tslot + p] = ent;
                    }
                }
            }
        }
    }
    cp_async_wait_group<0>();   // nothing of this CTA is in flight when it ends
    if (a.mode == kTmCandidate && a.tslot > 0) {
        __syncthreads();
        for (int i = tid; i < tiles_here * G; i += kTmThreads) {
            const int ti = i / G, g = i % G;
            const int64_t ptile = (static_cast<int64_t>(blockIdx.x) * a.tiles_per_cta + ti) * a.tile_stride;
            a.tile_counts[(h * G + g) * a.tiles + ptile] = S.tile_cnt[ti][g];
        }
    }
}

template <int G>
int launch_tm_g(TmArgs a, int64_t ltiles, unsigned H, cudaStream_t stream)
{
    const size_t smem = tm_smem_bytes<G>(a.D);
    int st = ensure_dynamic_smem(reinterpret_cast<const void*>(scan_tm_kernel<G>), smem);
    if (st) return st;
    int sms = 0;
    st = device_sm_count(&sms);
    if (st) return st;
    const int per_sm = smem <= 110 * 1024 ? tm_min_ctas<G>() : 1;
    const int64_t slots = static_cast<int64_t>(sms) * per_sm * 2;
    int64_t per = ceil_div(ltiles * static_cast<int64_t>(H), slots);
    per = per < 1 ? 1 : (per > kTmMaxTilesPerCta ? kTmMaxTilesPerCta : per);
    per = ceil_div(ltiles, ceil_div(ltiles, per));
    a.tiles_per_cta = static_cast<int>(per);
    const unsigned gx = static_cast<unsigned>(ceil_div(ltiles, a.tiles_per_cta));
    return launch_pdl(scan_tm_kernel<G>, dim3(gx, H), dim3(kTmThreads), smem, stream, a);
}

int launch_tm_mode(const TmArgs& a, int G, int64_t ltiles, unsigned H, cudaStream_t stream)
{
    switch (G) {
        case 1: return launch_tm_g<1>(a, ltiles, H, stream);
        case 2: return launch_tm_g<2>(a, ltiles, H, stream);
        case 3: return launch_tm_g<3>(a, ltiles, H, stream);
        case 4: return launch_tm_g<4>(a, ltiles, H, stream);
        case 5: return launch_tm_g<5>(a, ltiles, H, stream);
        case 6: return launch_tm_g<6>(a, ltiles, H, stream);
        case 7: return launch_tm_g<7>(a, ltiles, H, stream);
        default: return launch_tm_g<8>(a, ltiles, H, stream);
    }
}

// One thread per (group, block, byte column c): the codes of channels 2c and
// 2c + 1 of the block's 64 tokens, from their plane words, into byte c of
// each token's row.
__global__ void tm_from_planes_kernel(const uint64_t* __restrict__ planes, int64_t H, int D, int64_t nb,
                                      int64_t nb_stride, uint8_t* __restrict__ store)
{
    const int half = D / 2;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t >= H * nb * half) return;
    const int c = static_cast<int>(t % half);
    const int64_t b = (t / half) % nb, h = t / (half * nb);
    uint64_t p[2][kPlanes];
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int pl = 0; pl < kPlanes; ++pl) p[e][pl] = planes[((h * D + 2 * c + e) * kPlanes + pl) * nb_stride + b];
    uint8_t* dst = store + (h * nb_stride * kBlockTokens + b * kBlockTokens) * half + c;
    for (int i = 0; i < kBlockTokens; ++i) {
        uint32_t byte = 0;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            uint32_t code = 0;
#pragma unroll
            for (int pl = 0; pl < kPlanes; ++pl) code |= static_cast<uint32_t>((p[e][pl] >> i) & 1ull) << (3 - pl);
            byte |= code << (4 * e);
        }
        dst[static_cast<int64_t>(i) * half] = static_cast<uint8_t>(byte);
    }
}

}  // namespace

// Defined in topk.cu: per-head threshold selection over the sample.
int launch_tau(const float* sample, CandHeader* hdr, int64_t heads, int64_t n_sample, int64_t m_rank,
               int64_t n_keys, cudaStream_t stream);

int launch_tm_from_planes(const uint64_t* planes, int64_t H, int D, int64_t n, int64_t nb_stride, uint8_t* store,
                          cudaStream_t stream)
{
    const int64_t nb = ceil_div(n, kBlockTokens);
    const int64_t total = H * nb * (D / 2);
    tm_from_planes_kernel<<<static_cast<unsigned>(ceil_div(total, 256)), 256, 0, stream>>>(planes, H, D, nb,
                                                                                         nb_stride, store);
    return launch_status();
}

int launch_scan_tm(const uint8_t* store, const uint16_t* scales, int64_t H, int D, int64_t n, int64_t nb_stride,
                   const uint16_t* active, const int32_t* n_active, const float* q, int G, int mode, float* scores,
                   void* cand, int k, cudaStream_t stream)
{
    TmArgs a{};
    {
        const int st = device_fault_word(&a.fault);
        if (st) return st;
    }
    a.store = store;
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
        a.mode = kTmDense;
        a.tile_stride = 1;
        return launch_tm_mode(a, G, tiles, static_cast<unsigned>(H), stream);
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
            a.mode = kTmSample;
            a.tile_stride = L.tile_stride;
            const int st = launch_tm_mode(a, G, L.sample_tiles, static_cast<unsigned>(H), stream);
            if (st) return st;
        }
        const int st = launch_tau(a.sample, a.hdr, L.heads, L.n_sample, L.m_rank, n, stream);
        if (st || mode == FATHOM_SCAN_PREPARE) return st;
    }
    a.mode = kTmCandidate;
    a.tile_stride = 1;
    return launch_tm_mode(a, G, tiles, static_cast<unsigned>(H), stream);
}

}  // namespace fathom
