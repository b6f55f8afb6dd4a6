// Shared device helpers and launch plumbing for the Fathom kernels.
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "fathom.h"

namespace fathom {

constexpr int kBlockTokens = 64;   // tokens per scale block (one plane word)
constexpr int kPlanes = 4;         // 4-bit codes
constexpr int kMaxD = 256;
constexpr int kMaxG = 8;
constexpr int kMaxK = 4096;
constexpr int kMaxCandK = 1024;      // largest k of the candidate path
constexpr int kCandGather = 8 * kMaxCandK;   // survivors a top-k CTA gathers per head
constexpr int kMaxUnion = 16384;

// Record a CUDA error for fathom_last_cuda_error() and map it to a status.
int cuda_status(cudaError_t e);

// Launch-error check after a <<<>>> launch.
inline int launch_status() { return cuda_status(cudaGetLastError()); }

// Device address of this device's fault word (set when a bounded device
// wait gave up; see fault.cu).
int device_fault_word(int32_t** out);

// Programmatic dependent launch for the kernels of a decode step (plan,
// scans, threshold, top-k, union): each is launched so that the next one's
// CTAs can become resident while it finishes.  A kernel calls pdl_wait()
// before it reads anything an earlier kernel wrote, and lets its successor
// launch (pdl_launch_dependents) only after that wait; so when any kernel's
// wait returns, every kernel before it in the stream has completed and its
// writes are visible.  Without the launch attribute both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...));
}

// Device fault word bits: 1 = a bounded wait gave up; 2 = a bounds check of
// the debug build failed.
constexpr int32_t kFaultTimeout = 1;
constexpr int32_t kFaultBounds = 2;

// Debug build (FATHOM_DEBUG_BOUNDS): `ok` guards a memory access; a false
// check sets the fault word's bounds bit and the caller skips the access.
// Release builds compile the check away.
__device__ __forceinline__ bool bounds_ok(bool ok, int32_t* fault)
{
#ifdef FATHOM_DEBUG_BOUNDS
    if (!ok) atomicOr(fault, kFaultBounds);
    return ok;
#else
    (void)ok;
    (void)fault;
    return true;
#endif
}

// SM count of the current device (queried once per device; launch.cu).
int device_sm_count(int* sms);

// Raise `func`'s dynamic shared memory limit on the current device to at
// least `bytes`; the driver is called only the first time (or for a larger
// size).  launch.cu.
int ensure_dynamic_smem(const void* func, size_t bytes);

// ---------------------------------------------------------------------
// Order-preserving map from fp32 to uint32: larger float -> larger key.
// -0 is folded onto +0 so that the two compare equal, as fp32 values do.
// ---------------------------------------------------------------------
__device__ __forceinline__ uint32_t order_key(float f)
{
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float key_to_float(uint32_t k)
{
    uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
    return __uint_as_float(u);
}

// ---------------------------------------------------------------------
// Candidate buffer of a CANDIDATE scan, per (group, head):
//   header (count, tau, sample size);
//   sample scores (only when a threshold is sampled);
//   survivors: without a sample, every key at its own index (n entries);
//   with a sample, a fixed slot of `tslot` entries per scan tile, plus one
//   count per tile (a count above tslot marks an overflowed slot).
// ---------------------------------------------------------------------
struct CandHeader {
    int32_t count;   // without a sample: n; with one: unused (tile counts hold the totals)
    float tau;       // threshold the main pass used
    int32_t n_sample;
    int32_t pad;
};

struct CandLayout {
    int64_t heads;        // H * G
    int64_t tiles;        // scan tiles of n
    int64_t tslot;        // survivor slots per (tile, head); 0 without a sample
    int64_t cap;          // entries per head: n (no sample) or tiles * tslot
    int64_t sample_tiles; // tiles in the sample (0: tau = -inf, every key kept)
    int64_t tile_stride;  // sample takes every tile_stride-th tile
    int64_t n_sample;     // sample tokens per head (sample_tiles * tile tokens)
    int64_t m_rank;       // tau = m_rank-th largest sample score
    size_t off_hdr, off_sample, off_counts, off_entries, total;
};

#ifndef FATHOM_SCAN_TILE_BLOCKS
#define FATHOM_SCAN_TILE_BLOCKS 32
#endif
constexpr int kScanTileBlocks = FATHOM_SCAN_TILE_BLOCKS;   // 64-token blocks per scan tile (16 or 32)
static_assert(kScanTileBlocks == 16 || kScanTileBlocks == 32, "scan tiles hold 16 or 32 blocks");
constexpr int kScanTileTokens = kScanTileBlocks * kBlockTokens;

CandLayout cand_layout(int64_t H, int G, int64_t n, int k);

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

}  // namespace fathom
