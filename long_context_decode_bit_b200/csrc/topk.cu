// fathom_topk: per query head, the k highest-scoring keys (ties to the lower
// index), then the per-group union of the G winner lists (Fathom,
// byte-accounting section, top-k bullet: k winners per query head, the
// union of a KV head's four lists is what gets fetched).
//
// Selection is a three-pass radix select (11 + 11 + 10 bits) over the fp32
// scores mapped to order-preserving uint32 keys, run by one 1024-thread CTA
// per query head; it yields the k-th largest key T and how many keys equal
// to T are taken.  Keys above T are all winners; among keys equal to T the
// lowest indices win (dense scores are scanned in index order; candidate
// lists are unordered, so their ties are sorted by index).  The k winners
// are then sorted by (score desc, index asc) with a shared-memory bitonic
// sort on 64-bit composite keys.  The same select, over per-thread maxima
// of the sample scores, picks the candidate threshold tau.
#include "common.cuh"

namespace fathom {

namespace {

constexpr int kTopkThreads = 1024;
constexpr int kTopkCandThreads = 512;   // candidate lists are short: smaller CTAs, more of them per SM
constexpr int kRadixBins = 2048;
constexpr int kMaxTies = 4096;
constexpr unsigned kFull = 0xffffffffu;

struct Select {
    uint32_t T;     // k-th largest key
    int take_eq;    // keys equal to T that belong to the top k (>= 1)
};

// k-th largest of key_at(0 .. count-1), 1 <= kk <= count.  All threads of the
// CTA must call it.  hist: kRadixBins words of shared memory; sh: 2 ints.
template <class KeyAt>
__device__ Select block_select(KeyAt key_at, int64_t count, int kk, uint32_t* hist, uint32_t* sh)
{
    uint32_t prefix = 0, mask = 0;
#pragma unroll
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int width = pass == 2 ? 10 : 11;
        const uint32_t dmask = (1u << width) - 1u;
        const int nbins = 1 << width;
        for (int b = threadIdx.x; b < nbins; b += blockDim.x) hist[b] = 0;
        __syncthreads();
        for (int64_t i = threadIdx.x; i < count; i += blockDim.x) {
            const uint32_t key = key_at(i);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            // Lane L owns bins [top - per, top), top = nbins - per*L: lane 0
            // has the highest digits.  Find the digit holding the kk-th key.
            const int lane = threadIdx.x, per = nbins / 32, top = nbins - per * lane;
            uint32_t lsum = 0;
            for (int b = top - 1; b >= top - per; --b) lsum += hist[b];
            uint32_t incl = lsum;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t v = __shfl_up_sync(kFull, incl, o);
                if (lane >= o) incl += v;
            }
            const uint32_t excl = incl - lsum;
            const unsigned bal = __ballot_sync(kFull, excl < static_cast<uint32_t>(kk) &&
                                                          static_cast<uint32_t>(kk) <= incl);
            if (lane == __ffs(bal) - 1) {
                uint32_t c = excl;
                for (int b = top - 1; b >= top - per; --b) {
                    if (c + hist[b] >= static_cast<uint32_t>(kk)) { sh[0] = b; sh[1] = c; break; }
                    c += hist[b];
                }
            }
        }
        __syncthreads();
        kk -= static_cast<int>(sh[1]);
        prefix |= sh[0] << shift;
        mask |= dmask << shift;
        __syncthreads();
    }
    return Select{prefix, kk};
}

// In-place bitonic sort of n (a power of two) elements in shared memory.
template <typename T, bool kDescending>
__device__ void bitonic_sort(T* v, int n)
{
    for (int size = 2; size <= n; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int i = threadIdx.x; i < (n >> 1); i += blockDim.x) {
                const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
                const bool up = (lo & size) == 0;
                const T x = v[lo], y = v[hi];
                const bool sw = kDescending ? (up ? (x < y) : (x > y)) : (up ? (x > y) : (x < y));
                if (sw) { v[lo] = y; v[hi] = x; }
            }
        }
    }
    __syncthreads();
}

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
    float tau = -INFINITY;
    if (n_sample > 0) {
        const float* s = sample + hg * n_sample;
        uint32_t mk = 0;   // order key of the thread's maximum (0: none, below every score's key)
        for (int64_t i = threadIdx.x; i < n_sample; i += blockDim.x) mk = max(mk, order_key(s[i]));
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
    const float* s = sample + hg * n_sample;
    const Select r = block_select([&](int64_t i) { return order_key(s[i]); }, n_sample, static_cast<int>(m_rank),
                                  hist, sh);
    if (threadIdx.x == 0) write_header(hdr, hg, key_to_float(r.T), n_sample, n_keys);
}

struct TopkArgs {
    const float* scores;        // dense [H*G][n] or null
    const CandHeader* hdr;      // candidate mode
    const int32_t* tile_counts; // [H*G][tiles] (with a threshold sample)
    const int2* entries;
    int64_t cap, tiles, tslot;
    int64_t n;
    int k, kpow2;
    int gather_cap;             // survivors gathered into shared memory (tile slots)
    int32_t* idx;               // [H*G][k]
};

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const TopkArgs a)
{
    extern __shared__ __align__(16) unsigned char smem[];
    uint64_t* win = reinterpret_cast<uint64_t*>(smem);                        // kpow2
    int32_t* ties = reinterpret_cast<int32_t*>(win + a.kpow2);               // kMaxTies
    uint32_t* hist = reinterpret_cast<uint32_t*>(ties + kMaxTies);           // kRadixBins
    int2* gathered = reinterpret_cast<int2*>(hist + kRadixBins);             // gather_cap (tile slots)
    __shared__ uint32_t sh[2];
    __shared__ int w_cnt, t_cnt, warp_eq[kTopkThreads / 32], g_cnt, g_bad;

    const int64_t hg = static_cast<int64_t>(blockIdx.y) * gridDim.x + blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int k = a.k;
    int32_t* out = a.idx + hg * k;

    int64_t count;
    const int2* ent = nullptr;
    const float* sc = nullptr;
    if (a.scores) {
        count = a.n;
        sc = a.scores + hg * a.n;
    } else if (a.tslot == 0) {
        count = a.hdr[hg].count;            // every key kept at its own index
        ent = a.entries + hg * a.cap;
        if (count < k || count > a.cap) {
            for (int r = tid; r < k; r += blockDim.x) out[r] = -1;
            return;
        }
    } else {
        // Gather the non-empty tile slots into shared memory.
        if (tid == 0) { g_cnt = 0; g_bad = 0; }
        __syncthreads();
        const int32_t* tc = a.tile_counts + hg * a.tiles;
        const int2* src = a.entries + hg * a.cap;
        for (int64_t t = tid; t < a.tiles; t += blockDim.x) {
            const int c = tc[t];
            if (c <= 0) continue;
            if (c > a.tslot) { g_bad = 1; continue; }       // slot overflowed: keys were dropped
            const int base = atomicAdd(&g_cnt, c);
            if (base + c > a.gather_cap) { g_bad = 1; continue; }
            for (int e = 0; e < c; ++e) gathered[base + e] = src[t * a.tslot + e];
        }
        __syncthreads();
        count = g_cnt;
        if (g_bad || count < k || count > a.gather_cap) {   // could not prove exactness
            for (int r = tid; r < k; r += blockDim.x) out[r] = -1;
            return;
        }
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
        for (int64_t i = tid; i < count; i += blockDim.x) {
            const uint32_t key = key_at(i);
            if (key > sel.T) win[atomicAdd(&w_cnt, 1)] = composite(key, idx_at(i));
            else if (key == sel.T) {
                const int p = atomicAdd(&t_cnt, 1);
                if (p < kMaxTies) ties[p] = static_cast<int32_t>(idx_at(i));
            }
        }
        __syncthreads();
        if (t_cnt > kMaxTies) {
            for (int r = tid; r < k; r += blockDim.x) out[r] = -1;
            return;
        }
        const int tp = pow2_at_least(t_cnt);
        for (int i = t_cnt + tid; i < tp; i += blockDim.x) ties[i] = INT32_MAX;
        bitonic_sort<int32_t, false>(ties, tp);
        const int base = w_cnt;
        for (int r = tid; r < sel.take_eq; r += blockDim.x)
            win[base + r] = composite(sel.T, static_cast<uint32_t>(ties[r]));
    }
    __syncthreads();
    for (int i = k + tid; i < a.kpow2; i += blockDim.x) win[i] = 0;
    bitonic_sort<uint64_t, true>(win, a.kpow2);
    for (int r = tid; r < k; r += blockDim.x)
        out[r] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(win[r] & 0xFFFFFFFFu));
}

// Sorted, de-duplicated union of a group's G winner lists.
__global__ void __launch_bounds__(kTopkThreads)
union_kernel(const int32_t* __restrict__ idx, int G, int k, int upow2, int32_t* __restrict__ union_idx,
             int32_t* __restrict__ union_count, const int32_t* __restrict__ fault)
{
    extern __shared__ __align__(16) unsigned char smem[];
    int32_t* v = reinterpret_cast<int32_t*>(smem);
    __shared__ int warp_tot[kTopkThreads / 32], failed;
    const int64_t h = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gk = G * k;
    const int32_t* src = idx + h * gk;
    int32_t* dst = union_idx + h * gk;
    if (tid == 0) failed = 0;
    __syncthreads();
    for (int i = tid; i < upow2; i += blockDim.x) {
        const int32_t x = i < gk ? src[i] : INT32_MAX;
        if (x < 0) failed = 1;
        v[i] = x;
    }
    __syncthreads();
    const int32_t faulted = *fault;   // a scan whose ring wait gave up left void scores
    if (failed || faulted) {
        for (int i = tid; i < gk; i += blockDim.x) dst[i] = -1;
        if (tid == 0) union_count[h] = faulted ? FATHOM_ERR_TIMEOUT : FATHOM_ERR_OVERFLOW;
        return;
    }
    bitonic_sort<int32_t, false>(v, upow2);
    // Each thread owns a contiguous run; keep first occurrences.
    const int per = upow2 / blockDim.x > 0 ? upow2 / blockDim.x : 1;
    const int lo = tid * per;
    int mine = 0;
    for (int i = lo; i < lo + per && i < upow2; ++i)
        mine += (v[i] != INT32_MAX) && (i == 0 || v[i] != v[i - 1]);
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < (kTopkThreads / 32); ++w) {
        if (w < warp) before += warp_tot[w];
        total += warp_tot[w];
    }
    int pos = before + incl - mine;
    for (int i = lo; i < lo + per && i < upow2; ++i)
        if ((v[i] != INT32_MAX) && (i == 0 || v[i] != v[i - 1])) dst[pos++] = v[i];
    for (int i = total + tid; i < gk; i += blockDim.x) dst[i] = -1;
    if (tid == 0) union_count[h] = total;
}

}  // namespace

int launch_tau(const float* sample, CandHeader* hdr, int64_t heads, int64_t n_sample, int64_t m_rank,
               int64_t n_keys, cudaStream_t stream)
{
    if (n_sample > 0 && m_rank * 8 > kTopkThreads)
        tau_kernel_large<<<static_cast<unsigned>(heads), kTopkThreads, 0, stream>>>(sample, hdr, n_sample, m_rank,
                                                                                  n_keys);
    else
        tau_kernel<<<static_cast<unsigned>(heads), kTopkThreads, 0, stream>>>(sample, hdr, n_sample, m_rank, n_keys);
    return launch_status();
}

// Survivors one top-k CTA gathers: 8k, twice the ~4k a candidate pass keeps
// (kCandGather at the largest k); more marks the group for the dense rerun.
int gather_cap(int k) { return 8 * k < kCandGather ? 8 * k : kCandGather; }

size_t topk_smem_bytes(int k, bool gather)
{
    return sizeof(uint64_t) * pow2_at_least(k) + sizeof(int32_t) * kMaxTies + sizeof(uint32_t) * kRadixBins +
           (gather ? sizeof(int2) * gather_cap(k) : 0);
}

int launch_topk(const float* scores, const void* cand, int64_t H, int G, int64_t n, int k, int32_t* idx,
                int32_t* union_idx, int32_t* union_count, cudaStream_t stream)
{
    TopkArgs a{};
    a.scores = scores;
    a.n = n;
    a.k = k;
    a.kpow2 = pow2_at_least(k);
    a.gather_cap = gather_cap(k);
    a.idx = idx;
    bool gather = false;
    if (!scores) {
        const CandLayout L = cand_layout(H, G, n, k);
        const char* base = static_cast<const char*>(cand);
        a.hdr = reinterpret_cast<const CandHeader*>(base + L.off_hdr);
        a.tile_counts = reinterpret_cast<const int32_t*>(base + L.off_counts);
        a.entries = reinterpret_cast<const int2*>(base + L.off_entries);
        a.cap = L.cap;
        a.tiles = L.tiles;
        a.tslot = L.tslot;
        gather = L.tslot > 0;
    }
    const size_t smem = topk_smem_bytes(k, gather);
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_status(e);
    // The dense path's index-ordered pass counts per warp over kTopkThreads
    // threads; candidate lists take smaller CTAs.
    topk_kernel<<<dim3(G, static_cast<unsigned>(H)), scores ? kTopkThreads : kTopkCandThreads, smem, stream>>>(a);
    int st = launch_status();
    if (st) return st;
    int32_t* fault = nullptr;
    st = device_fault_word(&fault);
    if (st) return st;
    const int upow2 = pow2_at_least(G * k);
    const size_t usmem = sizeof(int32_t) * upow2;
    e = cudaFuncSetAttribute(union_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(usmem));
    if (e != cudaSuccess) return cuda_status(e);
    union_kernel<<<static_cast<unsigned>(H), kTopkThreads, usmem, stream>>>(idx, G, k, upow2, union_idx,
                                                                          union_count, fault);
    return launch_status();
}

}  // namespace fathom
