// fathom_plan / fathom_plan_fixed: the per-group read plan.
//
// Reverse water-filling (Fathom, section "方法二"): the (t+1)-th plane of
// channel j is worth the item w_j * 4^-t; the water level theta* is the
// smallest theta whose item count above it fits the budget, and each
// channel's depth is its number of items above theta*.  One CTA plans one
// group, one thread per channel.  Items are compared through an integer key
// that orders them exactly and grows like log2 of the item: the fp32
// exponent and fraction of w, with the exponent extended below the
// subnormal range and lowered by 2t for the factor 4^-t.  The level is the
// (B+1)-th largest item key, found by a radix select over the 4 D keys.
#include "common.cuh"
#include "select.cuh"

namespace fathom {

namespace {

// Exact, order-preserving key of the positive value w * 4^-t (w a positive
// finite fp32).  key = (extended biased exponent) * 2^23 + fraction.
__device__ __forceinline__ int32_t item_key(float w, int t)
{
    const uint32_t u = __float_as_uint(w);
    int e = static_cast<int>((u >> 23) & 0xFF);
    uint32_t f = u & 0x7FFFFFu;
    if (e == 0) {                      // subnormal: normalise the fraction
        const int msb = 31 - __clz(f);  // 0..22
        e = msb - 22;                   // extended exponent, <= 0
        f = (f << (23 - msb)) & 0x7FFFFFu;
    }
    return (e - 2 * t) * (1 << 23) + static_cast<int32_t>(f);
}

__device__ __forceinline__ float key_value(int32_t key)
{
    const int e = key >> 23;  // arithmetic shift: floor division
    const uint32_t f = static_cast<uint32_t>(key) & 0x7FFFFFu;
    if (e >= 1) return __uint_as_float(static_cast<uint32_t>(key));
    return ldexpf(1.0f + static_cast<float>(f) * 0x1p-23f, e - 127);
}

// Compact (j, t) pairs with t > 0 into ascending-j active entries.
__device__ __forceinline__ void write_active(int j, int t, int D, int64_t h, uint16_t* active,
                                             int32_t* n_active, int* warp_cnt)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const unsigned bal = __ballot_sync(0xffffffffu, t > 0);
    if (lane == 0) warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int base = 0, total = 0;
    for (int w = 0; w < nwarps; ++w) {
        if (w < warp) base += warp_cnt[w];
        total += warp_cnt[w];
    }
    const int pos = base + __popc(bal & ((1u << lane) - 1u));
    uint16_t* act = active + h * D;
    if (t > 0) act[pos] = static_cast<uint16_t>(j | (t << 8));
    if (j >= total) act[j] = 0;   // positions past n_active, exactly once each
    if (j == 0) n_active[h] = total;
}

__global__ void plan_kernel(const float* __restrict__ sigma2, const float* __restrict__ q, int G, int D,
                            const int32_t* __restrict__ budget_bits, int32_t budget_flat,
                            uint8_t* __restrict__ depth, uint16_t* __restrict__ active,
                            int32_t* __restrict__ n_active, float* __restrict__ theta)
{
    __shared__ int warp_cnt[kMaxD / 32];
    __shared__ int32_t key0[kMaxD];
    const int64_t h = blockIdx.x;
    const int j = threadIdx.x;   // blockDim.x == D
    pdl_wait();
    pdl_launch_dependents();

    // Importance in the plan's fixed single-precision order (no FMA).
    const float* qh = q + h * G * D + j;
    float acc = __fmul_rn(qh[0], qh[0]);
    for (int g = 1; g < G; ++g) acc = __fadd_rn(acc, __fmul_rn(qh[g * D], qh[g * D]));
    const float w = __fmul_rn(sigma2[h * D + j], acc);
    const bool pos = w > 0.0f;   // NaN and non-positive importance never read

    int B = budget_bits ? budget_bits[h] : budget_flat;
    B = min(max(B, 0), 4 * D);

    const int32_t k0 = pos ? item_key(w, 0) : 0;
    const int npos = __syncthreads_count(pos);

    int32_t kstar;          // items with key > kstar are read
    bool all_positive = false;
    if (npos == 0 || 4 * npos <= B) {
        all_positive = true;
        kstar = 0;
    } else {
        // kstar is the (B+1)-th largest item key: the smallest level with at
        // most B items above it.  Item t of channel j has the key
        // k0_j - t * 2^24 (the exponent lowered by 2t); a block radix select
        // over the 4 D items finds it in three passes.  Channels that read
        // nothing give the key 0, below every real item, and as 4 npos > B
        // they never reach rank B + 1.
        __shared__ uint32_t hist[kRadixBins];
        __shared__ uint32_t sh[2];
        key0[j] = pos ? k0 : INT32_MIN;   // INT32_MIN: no items (every real key is far above it)
        __syncthreads();
        auto key_at = [&](int64_t i) -> uint32_t {
            const int32_t c = key0[i >> 2];
            if (c == INT32_MIN) return 0u;
            return static_cast<uint32_t>(c - static_cast<int32_t>(i & 3) * (1 << 24)) ^ 0x80000000u;
        };
        const Select r = block_select(key_at, 4LL * D, B + 1, hist, sh);
        kstar = static_cast<int32_t>(r.T ^ 0x80000000u);
    }

    int t = 0;
    if (pos) {
        if (all_positive) t = 4;
        else
            for (int r = 0; r < 4; ++r) t += item_key(w, r) > kstar;
    }
    depth[h * D + j] = static_cast<uint8_t>(t);
    if (theta && j == 0) theta[h] = all_positive ? 0.0f : key_value(kstar);
    write_active(j, t, D, h, active, n_active, warp_cnt);
}

__global__ void plan_fixed_kernel(const float* __restrict__ q, int G, int D, int r, int bits,
                                  uint8_t* __restrict__ depth, uint16_t* __restrict__ active,
                                  int32_t* __restrict__ n_active)
{
    __shared__ float a_s[kMaxD];
    __shared__ int warp_cnt[kMaxD / 32];
    const int64_t h = blockIdx.x;
    const int j = threadIdx.x;
    const float* qh = q + h * G * D + j;
    float a = fabsf(qh[0]);
    for (int g = 1; g < G; ++g) a = __fadd_rn(a, fabsf(qh[g * D]));
    a_s[j] = a;
    __syncthreads();
    int rank = 0;
    for (int i = 0; i < D; ++i) {
        const float b = a_s[i];
        rank += (b > a) || (b == a && i < j);
    }
    const int t = rank < r ? bits : 0;
    depth[h * D + j] = static_cast<uint8_t>(t);
    write_active(j, t, D, h, active, n_active, warp_cnt);
}

// Per-layer budgets, step 1 (one CTA per group, one thread per channel):
// the group's items w_j 4^-t (w in the plan's fp32 order; 0 for a channel
// whose w is not positive) sorted in descending order into items[h][4D],
// and w itself (0 when not positive) into wout[h][D].
__global__ void layer_items_kernel(const float* __restrict__ sigma2, const float* __restrict__ q, int G, int D,
                                   int npow2, double* __restrict__ items, float* __restrict__ wout)
{
    __shared__ double it[4 * kMaxD];
    const int64_t h = blockIdx.x;
    const int j = threadIdx.x;   // blockDim.x == D
    const float* qh = q + h * G * D + j;
    float acc = __fmul_rn(qh[0], qh[0]);
    for (int g = 1; g < G; ++g) acc = __fadd_rn(acc, __fmul_rn(qh[g * D], qh[g * D]));
    const float w = __fmul_rn(sigma2[h * D + j], acc);
    const bool pos = w > 0.0f;
    wout[h * D + j] = pos ? w : 0.0f;
    for (int t = 0; t < 4; ++t) it[4 * j + t] = pos ? ldexp(static_cast<double>(w), -2 * t) : 0.0;
    for (int i = 4 * D + j; i < npow2; i += D) it[i] = -1.0;   // below every item
    // bitonic sort, descending
    for (int size = 2; size <= npow2; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int i = j; i < (npow2 >> 1); i += D) {
                const int lo = 2 * i - (i & (stride - 1)), hi = lo + stride;
                const bool up = (lo & size) == 0;
                const double x = it[lo], y = it[hi];
                if (up ? (x < y) : (x > y)) { it[lo] = y; it[hi] = x; }
            }
        }
    }
    __syncthreads();
    for (int i = j; i < 4 * D; i += D) items[h * 4 * D + i] = it[i];
}

// Per-layer budgets, step 2 (one warp): the greedy.  Layer l (groups
// l*P .. l*P+P-1) has the next gain g_l(b) = 0.75 * (sum_h items[h][b-1]) / N_l,
// N_l = sum over its groups and channels of w; each step gives one bit to
// the layer with the largest next gain, ties to the lower layer.  Sums run
// in double in the order h ascending, then j ascending.
__global__ void layer_greedy_kernel(const double* __restrict__ items, const float* __restrict__ w, int64_t H, int D,
                                    int layers, int64_t T, int32_t* __restrict__ budget)
{
    extern __shared__ __align__(8) unsigned char lsm[];
    double* N = reinterpret_cast<double*>(lsm);
    double* gain = N + layers;
    int* ptr = reinterpret_cast<int*>(gain + layers);
    const int lane = threadIdx.x;
    const int64_t P = H / layers;
    const int NI = 4 * D;
    auto next_gain = [&](int l, int b) -> double {   // gain of the layer's (b+1)-th bit
        double S = 0.0;
        for (int64_t h = l * P; h < (l + 1) * P; ++h) S += items[h * NI + b];
        return N[l] > 0.0 ? 0.75 * S / N[l] : 0.0;
    };
    for (int l = lane; l < layers; l += 32) {
        double n = 0.0;
        for (int64_t h = l * P; h < (l + 1) * P; ++h)
            for (int j = 0; j < D; ++j) n += static_cast<double>(w[h * D + j]);
        N[l] = n;
        ptr[l] = 0;
        gain[l] = next_gain(l, 0);
    }
    __syncwarp();
    for (int64_t step = 0; step < T; ++step) {
        double bg = -1.0;
        int bl = INT32_MAX;
        for (int l = lane; l < layers; l += 32) {
            if (ptr[l] >= NI) continue;
            if (gain[l] > bg) { bg = gain[l]; bl = l; }   // ascending l: the first maximum wins
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const double og = __shfl_xor_sync(0xffffffffu, bg, o);
            const int ol = __shfl_xor_sync(0xffffffffu, bl, o);
            if (og > bg || (og == bg && ol < bl)) { bg = og; bl = ol; }
        }
        if (bl == INT32_MAX) break;   // every layer full (T was capped before the launch)
        if ((bl & 31) == lane) {
            const int b = ++ptr[bl];
            gain[bl] = b < NI ? next_gain(bl, b) : 0.0;
        }
        __syncwarp();
    }
    for (int64_t h = lane; h < H; h += 32) budget[h] = ptr[h / P];
}

}  // namespace

size_t layer_budgets_workspace_bytes(int64_t H, int D)
{
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    return up(sizeof(double) * H * 4 * D) + up(sizeof(float) * H * D);
}

int launch_layer_budgets(const float* sigma2, const float* q, int64_t H, int G, int D, int layers, int64_t total_bits,
                         int32_t* budget, void* ws, cudaStream_t stream)
{
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    double* items = static_cast<double*>(ws);
    float* w = reinterpret_cast<float*>(static_cast<char*>(ws) + up(sizeof(double) * H * 4 * D));
    int npow2 = 1;
    while (npow2 < 4 * D) npow2 <<= 1;
    layer_items_kernel<<<static_cast<unsigned>(H), D, 0, stream>>>(sigma2, q, G, D, npow2, items, w);
    int st = launch_status();
    if (st) return st;
    int64_t T = total_bits < 0 ? 0 : total_bits;
    if (T > static_cast<int64_t>(layers) * 4 * D) T = static_cast<int64_t>(layers) * 4 * D;
    const size_t smem = sizeof(double) * 2 * layers + sizeof(int) * layers;
    layer_greedy_kernel<<<1, 32, smem, stream>>>(items, w, H, D, layers, T, budget);
    return launch_status();
}

int launch_plan(const float* sigma2, const float* q, int64_t H, int G, int D, const int32_t* budget_bits,
                int32_t budget_flat, uint8_t* depth, uint16_t* active, int32_t* n_active, float* theta,
                cudaStream_t stream)
{
    return launch_pdl(plan_kernel, dim3(static_cast<unsigned>(H)), dim3(D), 0, stream, sigma2, q, G, D, budget_bits,
                      budget_flat, depth, active, n_active, theta);
}

int launch_plan_fixed(const float* q, int64_t H, int G, int D, int r, int bits, uint8_t* depth, uint16_t* active,
                      int32_t* n_active, cudaStream_t stream)
{
    plan_fixed_kernel<<<static_cast<unsigned>(H), D, 0, stream>>>(q, G, D, r, bits, depth, active, n_active);
    return launch_status();
}

}  // namespace fathom
