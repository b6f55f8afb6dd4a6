// fathom_topk: per query head, the k highest-scoring keys (ties to the lower
// index), then the per-group union of the G winner lists (Fathom,
// byte-accounting section, top-k bullet: k winners per query head, the
// union of a KV head's four lists is what gets fetched).
//
// Selection is a three-pass radix select (11 + 11 + 10 bits) over the fp32
// scores mapped to order-preserving uint32 keys, run by one CTA per query
// head; it yields the k-th largest key T and how many keys equal to T are
// taken.  Keys above T are all winners; among keys equal to T the lowest
// indices win (dense scores are scanned in index order; candidate lists are
// unordered, so their ties are sorted by index).  The k winners are sorted
// by (score desc, index asc) for idx, and by index into the group's slice
// of union_idx.  The union merges a group's G index-sorted lists pairwise
// and keeps the first of each run of equal indices: on the candidate path
// the last of the group's G CTAs to finish does it (a per-group counter in
// the candidate header), after a dense top-k a second kernel does.  The same
// select, over per-thread maxima of the sample scores, picks the candidate
// threshold tau.
#include "common.cuh"
#include "select.cuh"

namespace fathom {

namespace {

constexpr int kTopkThreads = 1024;
constexpr int kTopkCandThreads = 512;   // candidate lists are short: smaller CTAs, more of them per SM
constexpr int kMaxTies = 4096;

__device__ __forceinline__ uint64_t composite(uint32_t key, uint32_t idx)
{
    return (static_cast<uint64_t>(key) << 32) | (0xFFFFFFFFu - idx);
}

__host__ __device__ inline int pow2_at_least(int x)
{
    int p = 1;
    while (p < x) p <<= 1;
    return p;
}

// Sort buffer of a top-k CTA: the k winners' 64-bit composites, or up to
// kMaxTies tie indices.
__host__ __device__ inline size_t sort_tmp_bytes(int kpow2)
{
    const size_t a = sizeof(uint64_t) * kpow2, b = sizeof(int32_t) * kMaxTies;
    return a > b ? a : b;
}

// Header of a group's candidate buffer: the threshold, and the counters reset.
__device__ __forceinline__ void write_header(CandHeader* hdr, int64_t hg, float tau, int64_t n_sample, int64_t n_keys)
{
    // Without a sample every key is kept, at its own index (n entries).
    hdr[hg].count = n_sample > 0 ? 0 : static_cast<int32_t>(n_keys);
    hdr[hg].tau = tau;
    hdr[hg].n_sample = static_cast<int32_t>(n_sample);
    hdr[hg].pad = 0;
}

// Threshold for the candidate pass (or -inf without a sample); also resets
// the candidate counters.  Each thread takes the maximum of its share of the
// sample scores, and tau is the m-th largest of those kTopkThreads maxima.
// That is never above the m-th largest sample score (each thread gives at
// most one of the top m), so the pass keeps at least as many keys as the
// exact threshold would.  For m far below the thread count it is close:
// m of the top sample scores land in different threads but for a few
// collisions, and each collision only lowers tau to the next score.  The
// sample is read from global memory once.
__global__ void __launch_bounds__(kTopkThreads)
tau_kernel(const float* __restrict__ sample, CandHeader* __restrict__ hdr, int64_t n_sample, int64_t m_rank,
           int64_t n_keys)
{
    __shared__ uint32_t hist[kRadixBins];
    __shared__ uint32_t tmax[kTopkThreads];
    __shared__ uint32_t sh[2];
    const int64_t hg = blockIdx.x;
    pdl_wait();
    pdl_launch_dependents();
    float tau = -INFINITY;
    if (n_sample > 0) {
        // n_sample is a whole number of 2048-token tiles and the sample
        // 16-byte aligned: float4 reads, several in flight per thread.
        const float4* s4 = reinterpret_cast<const float4*>(sample + hg * n_sample);
        uint32_t mk = 0;   // order key of the thread's maximum (0: none, below every score's key)
#pragma unroll 4
        for (int64_t i = threadIdx.x; i < n_sample / 4; i += blockDim.x) {
            const float4 x = s4[i];
            mk = max(max(mk, order_key(x.x)), max(order_key(x.y), max(order_key(x.z), order_key(x.w))));
        }
        tmax[threadIdx.x] = mk;
        __syncthreads();
        const Select r = block_select([&](int64_t i) { return tmax[i]; }, kTopkThreads, static_cast<int>(m_rank),
                                      hist, sh);
        tau = key_to_float(r.T);
    }
    if (threadIdx.x == 0) write_header(hdr, hg, tau, n_sample, n_keys);
}

// The same with the exact m-th largest sample score (three radix passes
// over the sample), for m beyond a small fraction of the thread count.
__global__ void __launch_bounds__(kTopkThreads)
tau_kernel_large(const float* __restrict__ sample, CandHeader* __restrict__ hdr, int64_t n_sample, int64_t m_rank,
                 int64_t n_keys)
{
    __shared__ uint32_t hist[kRadixBins];
    __shared__ uint32_t sh[2];
    const int64_t hg = blockIdx.x;
    pdl_wait();
    pdl_launch_dependents();
    const float* s = sample + hg * n_sample;
    const Select r = block_select([&](int64_t i) { return order_key(s[i]); }, n_sample, static_cast<int>(m_rank),
                                  hist, sh);
    if (threadIdx.x == 0) write_header(hdr, hg, key_to_float(r.T), n_sample, n_keys);
}

struct TopkArgs {
    const float* scores;        // dense [H*G][n] or null
    CandHeader* hdr;            // candidate mode (hdr[h*G].pad: the head's arrival counter)
    const int32_t* tile_counts; // [H*G][tiles] (with a threshold sample)
    const int2* entries;
    int64_t cap, tiles, tslot;
    int64_t n;
    int G, k, kpow2;
    int gather_cap;             // survivors gathered into shared memory (tile slots)
    int32_t* idx;               // [H*G][k]
    int32_t* union_idx;         // [H][G*k]: group g's winners sorted by index at [g*k, g*k+k), then the union
    int32_t* union_count;       // [H]
    const int32_t* fault;       // device fault word
};

// Sorted, de-duplicated union of a group's G winner lists, each already
// sorted by index, in shared memory (buf0[g*k .. g*k+k)).  The lists are
// merged pairwise (ceil(log2 G) levels, between buf0 and buf1), equal
// indices then sit side by side, and the first of each run is kept.
// dst: the union, padded with -1 to G*k.  Every thread of the CTA must call
// it; buf0 and buf1 hold G*k ints each.
__device__ void merge_union(int32_t* buf0, int32_t* buf1, int G, int k, int32_t* dst, int32_t* union_count_h,
                            int* warp_tot)
{
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nt = blockDim.x;
    const int gk = G * k;
    int32_t* src = buf0;
    int32_t* tmp = buf1;
    for (int L = k; L < gk; L *= 2) {
        merge_level<int32_t, false>(src, tmp, gk, L);
        __syncthreads();
        int32_t* t = src; src = tmp; tmp = t;
    }
    const int32_t* merged = src;
    // Each thread owns a contiguous run of the merged order; keep first occurrences.
    const int per = (gk + nt - 1) / nt;
    const int lo = min(tid * per, gk), hi = min(lo + per, gk);
    int mine = 0;
    for (int i = lo; i < hi; ++i) mine += i == 0 || merged[i] != merged[i - 1];
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < (nt >> 5); ++w) {
        const int v = warp_tot[w];
        before += w < warp ? v : 0;
        total += v;
    }
    int pos = before + incl - mine;
    for (int i = lo; i < hi; ++i)
        if (i == 0 || merged[i] != merged[i - 1]) dst[pos++] = merged[i];
    for (int i = total + tid; i < gk; i += nt) dst[i] = -1;
    if (tid == 0) *union_count_h = total;
}

// Load a head's G sorted lists from union_idx into shared memory (through L2:
// other CTAs wrote them) and check them and the fault word; false if the
// head must report a failure (written here).
__device__ bool load_lists(const TopkArgs& a, int64_t h, int32_t* lists, int* failed)
{
    const int gk = a.G * a.k;
    const int32_t* src = a.union_idx + h * gk;
    if (threadIdx.x == 0) *failed = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < gk; i += blockDim.x) {
        const int32_t x = __ldcg(src + i);
        if (x < 0) *failed = 1;
        lists[i] = x;
    }
    __syncthreads();
    const int32_t faulted = __ldcg(a.fault);   // a scan whose ring wait gave up left void scores
    if (*failed || faulted) {
        for (int i = threadIdx.x; i < gk; i += blockDim.x) a.union_idx[h * gk + i] = -1;
        if (threadIdx.x == 0)
            a.union_count[h] = (faulted & kFaultTimeout) ? FATHOM_ERR_TIMEOUT
                               : (faulted ? FATHOM_ERR_BOUNDS : FATHOM_ERR_OVERFLOW);
        return false;
    }
    return true;
}

// Per query head (h, g): the k winners, in (score desc, index asc) order to
// idx, and sorted by index to the group's slice of union_idx.  A head that
// cannot prove its top-k exact writes -1 to both.  Returns after its writes.
__device__ void topk_head(const TopkArgs& a, unsigned char* smem)
{
    uint64_t* win = reinterpret_cast<uint64_t*>(smem);                        // kpow2
    int32_t* ties = reinterpret_cast<int32_t*>(win + a.kpow2);               // kMaxTies
    uint32_t* hist = reinterpret_cast<uint32_t*>(ties + kMaxTies);           // kRadixBins
    unsigned char* tmp = reinterpret_cast<unsigned char*>(hist + kRadixBins);   // sort buffer (sort_tmp_bytes)
    int2* gathered = reinterpret_cast<int2*>(tmp + sort_tmp_bytes(a.kpow2));     // gather_cap (tile slots)
    __shared__ uint32_t sh[2];
    __shared__ int w_cnt, t_cnt, warp_eq[kTopkThreads / 32], g_cnt, g_bad;

    const int g = blockIdx.x;
    const int64_t h = blockIdx.y;
    const int64_t hg = h * gridDim.x + g;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = a.k;
    int32_t* out = a.idx + hg * k;
    int32_t* sorted_out = a.union_idx + h * a.G * k + g * k;
    auto fail = [&]() {
        for (int r = tid; r < k; r += blockDim.x) { out[r] = -1; sorted_out[r] = -1; }
    };

    int64_t count;
    const int2* ent = nullptr;
    const float* sc = nullptr;
    if (a.scores) {
        count = a.n;
        sc = a.scores + hg * a.n;
    } else if (a.tslot == 0) {
        count = a.hdr[hg].count;            // every key kept at its own index
        ent = a.entries + hg * a.cap;
        if (count < k || count > a.cap) { fail(); return; }
    } else {
        // Gather the non-empty tile slots into shared memory: a warp scan of
        // the tile counts gives each tile its place (one shared atomic per
        // warp), and each thread copies its tile with several loads in flight.
        if (tid == 0) { g_cnt = 0; g_bad = 0; }
        __syncthreads();
        const int32_t* tc = a.tile_counts + hg * a.tiles;
        const int2* src = a.entries + hg * a.cap;
        for (int64_t t0 = 0; t0 < a.tiles; t0 += blockDim.x) {
            const int64_t t = t0 + tid;
            int c = t < a.tiles ? tc[t] : 0;
            if (c > a.tslot) { g_bad = 1; c = 0; }       // slot overflowed: keys were dropped
            c = max(c, 0);
            int incl = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += v;
            }
            int wbase = 0;
            if (lane == 31 && incl > 0) wbase = atomicAdd(&g_cnt, incl);
            wbase = __shfl_sync(kFull, wbase, 31);
            const int base = wbase + incl - c;
            if (c == 0) continue;
            if (base + c > a.gather_cap) { g_bad = 1; continue; }
            const int2* sp = src + t * a.tslot;
            if (!bounds_ok((t + 1) * a.tslot <= a.cap, const_cast<int32_t*>(a.fault))) continue;
            for (int e0 = 0; e0 < c; e0 += 4) {
                int2 x[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (e0 + u < c) x[u] = sp[e0 + u];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if (e0 + u < c) gathered[base + e0 + u] = x[u];
            }
        }
        __syncthreads();
        count = g_cnt;
        if (g_bad || count < k || count > a.gather_cap) { fail(); return; }   // could not prove exactness
        ent = gathered;
    }
    auto key_at = [&](int64_t i) -> uint32_t {
        return sc ? order_key(sc[i]) : order_key(__int_as_float(ent[i].y));
    };
    auto idx_at = [&](int64_t i) -> uint32_t { return sc ? static_cast<uint32_t>(i) : static_cast<uint32_t>(ent[i].x); };

    const Select sel = block_select(key_at, count, k, hist, sh);
    if (tid == 0) { w_cnt = 0; t_cnt = 0; }
    __syncthreads();

    if (sc) {
        // Index-ordered pass: every key above T, and the first take_eq keys equal to T.
        int eq_seen = 0;
        for (int64_t base = 0; base < count; base += blockDim.x) {
            const int64_t i = base + tid;
            uint32_t key = 0;
            if (i < count) key = key_at(i);
            const bool gt = i < count && key > sel.T;
            const bool eq = i < count && key == sel.T;
            if (gt) win[atomicAdd(&w_cnt, 1)] = composite(key, static_cast<uint32_t>(i));
            const unsigned bal = __ballot_sync(kFull, eq);
            if (lane == 0) warp_eq[warp] = __popc(bal);
            __syncthreads();
            int before = 0, total = 0;
            for (int w = 0; w < (kTopkThreads / 32); ++w) {
                if (w < warp) before += warp_eq[w];
                total += warp_eq[w];
            }
            const int rank = eq_seen + before + __popc(bal & ((1u << lane) - 1u));
            if (eq && rank < sel.take_eq) win[atomicAdd(&w_cnt, 1)] = composite(key, static_cast<uint32_t>(i));
            eq_seen += total;
            __syncthreads();
        }
    } else {
        // Keys above T and ties at T, placed with one shared atomic per warp.
        const unsigned below = (1u << lane) - 1u;
        for (int64_t i0 = 0; i0 < count; i0 += blockDim.x) {
            const int64_t i = i0 + tid;
            uint32_t key = 0;
            if (i < count) key = key_at(i);
            const bool gt = i < count && key > sel.T;
            const bool eq = i < count && key == sel.T;
            const unsigned bg = __ballot_sync(kFull, gt), be = __ballot_sync(kFull, eq);
            int wg = 0, we = 0;
            if (lane == 0) {
                if (bg) wg = atomicAdd(&w_cnt, __popc(bg));
                if (be) we = atomicAdd(&t_cnt, __popc(be));
            }
            wg = __shfl_sync(kFull, wg, 0);
            we = __shfl_sync(kFull, we, 0);
            if (gt) win[wg + __popc(bg & below)] = composite(key, idx_at(i));
            if (eq) {
                const int p = we + __popc(be & below);
                if (p < kMaxTies) ties[p] = static_cast<int32_t>(idx_at(i));
            }
        }
        __syncthreads();
        if (t_cnt > kMaxTies) { fail(); return; }
        const int tp = pow2_at_least(t_cnt);
        for (int i = t_cnt + tid; i < tp; i += blockDim.x) ties[i] = INT32_MAX;
        block_sort<int32_t, false>(ties, reinterpret_cast<int32_t*>(tmp), tp);
        const int base = w_cnt;
        for (int r = tid; r < sel.take_eq; r += blockDim.x)
            win[base + r] = composite(sel.T, static_cast<uint32_t>(ties[r]));
    }
    __syncthreads();
    for (int i = k + tid; i < a.kpow2; i += blockDim.x) win[i] = 0;
    block_sort<uint64_t, true>(win, reinterpret_cast<uint64_t*>(tmp), a.kpow2);
    // Score order to idx; the same k indices sorted ascending to the group's
    // slice of union_idx (ties[] is free again and holds kMaxTies >= kpow2).
    for (int r = tid; r < a.kpow2; r += blockDim.x) {
        const int32_t i = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(win[r] & 0xFFFFFFFFu));
        if (r < k) out[r] = i;
        ties[r] = r < k ? i : INT32_MAX;
    }
    block_sort<int32_t, false>(ties, reinterpret_cast<int32_t*>(tmp), a.kpow2);
    for (int r = tid; r < k; r += blockDim.x) sorted_out[r] = ties[r];
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const TopkArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    pdl_wait();
    pdl_launch_dependents();
    topk_head(a, smem);
    if (a.scores) return;   // dense: union_kernel follows
    // Candidate mode: the last of a head's G CTAs to finish builds the head's
    // union from the G sorted slices (fence, then one counter per head; the
    // counter is reset by the threshold pass and again by the last CTA).
    __shared__ int last, failed, warp_tot[kTopkThreads / 32];
    const int64_t h = blockIdx.y;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) last = atomicAdd(&a.hdr[h * a.G].pad, 1) == a.G - 1;
    __syncthreads();
    if (!last) return;
    __threadfence();
    if (threadIdx.x == 0) a.hdr[h * a.G].pad = 0;
    // The head's own top-k is written: its shared memory is free for the union.
    int32_t* lists = reinterpret_cast<int32_t*>(smem);
    int32_t* merged = lists + a.G * a.k;
    if (!load_lists(a, h, lists, &failed)) return;
    merge_union(lists, merged, a.G, a.k, a.union_idx + h * a.G * a.k, a.union_count + h, warp_tot);
}

// The union after a dense top-k (one CTA per group).
__global__ void __launch_bounds__(kTopkThreads)
union_kernel(const TopkArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int failed, warp_tot[kTopkThreads / 32];
    const int64_t h = blockIdx.x;
    pdl_wait();
    pdl_launch_dependents();
    int32_t* lists = reinterpret_cast<int32_t*>(smem);
    int32_t* merged = lists + a.G * a.k;
    if (!load_lists(a, h, lists, &failed)) return;
    merge_union(lists, merged, a.G, a.k, a.union_idx + h * a.G * a.k, a.union_count + h, warp_tot);
}

}  // namespace

int launch_tau(const float* sample, CandHeader* hdr, int64_t heads, int64_t n_sample, int64_t m_rank,
               int64_t n_keys, cudaStream_t stream)
{
    const dim3 grid(static_cast<unsigned>(heads)), block(kTopkThreads);
    if (n_sample > 0 && m_rank * 8 > kTopkThreads)
        return launch_pdl(tau_kernel_large, grid, block, 0, stream, sample, hdr, n_sample, m_rank, n_keys);
    return launch_pdl(tau_kernel, grid, block, 0, stream, sample, hdr, n_sample, m_rank, n_keys);
}

// Survivors one top-k CTA gathers: 8k, twice the ~4k a candidate pass keeps
// (kCandGather at the largest k); more marks the group for the dense rerun.
int gather_cap(int k) { return 8 * k < kCandGather ? 8 * k : kCandGather; }

size_t topk_smem_bytes(int G, int k, bool gather, bool fused_union)
{
    const size_t own = sizeof(uint64_t) * pow2_at_least(k) + sizeof(int32_t) * kMaxTies +
                       sizeof(uint32_t) * kRadixBins + sort_tmp_bytes(pow2_at_least(k)) +
                       (gather ? sizeof(int2) * gather_cap(k) : 0);
    const size_t uni = fused_union ? 2 * sizeof(int32_t) * G * k : 0;   // lists + merged order
    return own > uni ? own : uni;
}

int launch_topk(const float* scores, const void* cand, int64_t H, int G, int64_t n, int k, int32_t* idx,
                int32_t* union_idx, int32_t* union_count, cudaStream_t stream)
{
    TopkArgs a{};
    a.scores = scores;
    a.n = n;
    a.G = G;
    a.k = k;
    a.kpow2 = pow2_at_least(k);
    a.gather_cap = gather_cap(k);
    a.idx = idx;
    a.union_idx = union_idx;
    a.union_count = union_count;
    {
        int32_t* fault = nullptr;
        const int st = device_fault_word(&fault);
        if (st) return st;
        a.fault = fault;
    }
    bool gather = false;
    if (!scores) {
        const CandLayout L = cand_layout(H, G, n, k);
        char* base = static_cast<char*>(const_cast<void*>(cand));
        a.hdr = reinterpret_cast<CandHeader*>(base + L.off_hdr);
        a.tile_counts = reinterpret_cast<const int32_t*>(base + L.off_counts);
        a.entries = reinterpret_cast<const int2*>(base + L.off_entries);
        a.cap = L.cap;
        a.tiles = L.tiles;
        a.tslot = L.tslot;
        gather = L.tslot > 0;
    }
    const size_t smem = topk_smem_bytes(G, k, gather, scores == nullptr);
    int st = ensure_dynamic_smem(reinterpret_cast<const void*>(topk_kernel), smem);
    if (st) return st;
    // The dense path's index-ordered pass counts per warp over kTopkThreads
    // threads; candidate lists take smaller CTAs, and the last CTA of each
    // group builds its union.
    st = launch_pdl(topk_kernel, dim3(G, static_cast<unsigned>(H)), dim3(scores ? kTopkThreads : kTopkCandThreads),
                    smem, stream, a);
    if (st || !scores) return st;
    const size_t usmem = 2 * sizeof(int32_t) * G * k;
    st = ensure_dynamic_smem(reinterpret_cast<const void*>(union_kernel), usmem);
    if (st) return st;
    return launch_pdl(union_kernel, dim3(static_cast<unsigned>(H)), dim3(kTopkThreads), usmem, stream, a);
}

}  // namespace fathom
