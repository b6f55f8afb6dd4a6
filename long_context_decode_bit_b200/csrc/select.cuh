// Block-wide selection and sorting in shared memory and registers, shared
// by the top-k, the candidate threshold and the read plan: a radix select
// of the k-th largest 32-bit key, and sorts (warp bitonic runs merged
// pairwise, or a plain bitonic network for small arrays).
#pragma once

#include <type_traits>

#include "common.cuh"

namespace fathom {
namespace {

constexpr int kRadixBins = 2048;
constexpr unsigned kFull = 0xffffffffu;

struct Select {
    uint32_t T;     // k-th largest key
    int take_eq;    // keys equal to T that belong to the top k (>= 1)
};

// k-th largest of key_at(0 .. count-1), 1 <= kk <= count.  All threads of the
// CTA must call it (blockDim.x a multiple of 32, at most 1024).  hist:
// kRadixBins words of shared memory; sh: 2 ints.  Each pass histograms one
// digit of the keys that match the digits chosen so far; the digit holding
// the kk-th largest key is found by a block-wide scan over the bins from the
// top (each thread sums its own run of bins, then a warp scan and one pass
// over the warp totals), so no thread walks the whole histogram.
template <class KeyAt>
__device__ Select block_select(KeyAt key_at, int64_t count, int kk, uint32_t* hist, uint32_t* sh)
{
    __shared__ uint32_t wsum[32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t prefix = 0, mask = 0;
#pragma unroll
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int width = pass == 2 ? 10 : 11;
        const uint32_t dmask = (1u << width) - 1u;
        const int nbins = 1 << width;
        for (int b = tid; b < nbins; b += blockDim.x) hist[b] = 0;
        __syncthreads();
        for (int64_t i = tid; i < count; i += blockDim.x) {
            const uint32_t key = key_at(i);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
        }
        __syncthreads();
        // Thread t owns bins [top - per, top), top = nbins - per * t: thread 0
        // has the highest digits.
        const int per = nbins / static_cast<int>(blockDim.x), top = nbins - per * tid;
        uint32_t lsum = 0;
        for (int b = top - 1; b >= top - per; --b) lsum += hist[b];
        uint32_t incl = lsum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t v = __shfl_up_sync(kFull, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        uint32_t excl = incl - lsum;
        for (int w = 0; w < warp; ++w) excl += wsum[w];
        if (excl < static_cast<uint32_t>(kk) && static_cast<uint32_t>(kk) <= excl + lsum) {   // exactly one thread
            uint32_t c = excl;
            for (int b = top - 1; b >= top - per; --b) {
                if (c + hist[b] >= static_cast<uint32_t>(kk)) { sh[0] = b; sh[1] = c; break; }
                c += hist[b];
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

// One level of a pairwise merge sort: the sorted runs of src (length L each,
// the last possibly shorter; m elements in all) are merged two by two into
// runs of 2L in dst, in ascending (or, kDescending, descending) order.  Each
// thread makes a contiguous stretch of the output: it finds where its first
// element comes from with one binary search along the merge path, then
// walks both runs.  On equal values the first run's entry goes first.
template <typename T, bool kDescending>
__device__ void merge_level(const T* src, T* dst, int m, int L)
{
    auto before = [](const T& x, const T& y) { return kDescending ? (y < x) : (x < y); };
    const int nt = blockDim.x;
    const int per = (m + nt - 1) / nt;
    const int p0 = threadIdx.x * per, p1 = min(p0 + per, m);
    int pair = -1, i = 0, j = 0, na = 0, nb = 0;
    const T* A = src;
    const T* B = src;
    for (int p = p0; p < p1; ++p) {
        if (p / (2 * L) != pair) {   // first output of this thread in a new pair of runs
            pair = p / (2 * L);
            const int a0 = pair * 2 * L;
            na = min(L, m - a0);
            nb = max(0, min(L, m - a0 - na));
            A = src + a0;
            B = A + na;
            const int d = p - a0;    // outputs of this pair before p
            int lo = max(0, d - nb), hi = min(d, na);
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (!before(B[d - mid - 1], A[mid])) lo = mid + 1; else hi = mid;
            }
            i = lo;
            j = d - lo;
        }
        const bool take_a = i < na && (j >= nb || !before(B[j], A[i]));
        dst[p] = take_a ? A[i++] : B[j++];
    }
}

// Sort n elements of shared memory s in place (ascending, or descending),
// which any thread of the CTA may have written just before the call.  Runs
// of 32 are sorted in registers by one warp each (a bitonic network over
// shuffles), then merged pairwise level by level between s and tmp (n
// elements of shared memory).  n a multiple of 32; smaller n take the plain
// shared-memory network.  Every thread of the CTA must call it.
template <typename T, bool kDescending>
__device__ void block_sort(T* s, T* tmp, int n)
{
    if (n < 32 || (n & 31)) { bitonic_sort<T, kDescending>(s, n); return; }
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    __syncthreads();
    for (int c = warp; c < (n >> 5); c += nw) {
        T v = s[c * 32 + lane];
#pragma unroll
        for (int size = 2; size <= 32; size <<= 1)
#pragma unroll
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                const T o = __shfl_xor_sync(kFull, v, stride);
                const bool asc = ((lane & size) == 0) != kDescending;
                const bool keep_min = ((lane & stride) == 0) == asc;
                v = keep_min ? (o < v ? o : v) : (o > v ? o : v);
            }
        s[c * 32 + lane] = v;
    }
    __syncthreads();
    T* src = s;
    T* dst = tmp;
    for (int L = 32; L < n; L *= 2) {
        merge_level<T, kDescending>(src, dst, n, L);
        __syncthreads();
        T* t = src; src = dst; dst = t;
    }
    if (src != s) {
        for (int i = threadIdx.x; i < n; i += blockDim.x) s[i] = src[i];
        __syncthreads();
    }
}

}  // namespace
}  // namespace fathom
