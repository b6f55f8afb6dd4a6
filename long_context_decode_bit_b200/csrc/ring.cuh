// Shared-memory staging ring of the scan kernels: cp.async copies whose
// completion arrives on an mbarrier, and bounded mbarrier waits.
//
// Every wait polls `mbarrier.try_wait.parity` (each poll suspends the thread
// for at most about a microsecond) up to kSpinLimit times; a wait that runs
// out returns false and the caller marks the device fault word and leaves its
// loop, so a kernel never spins for ever.
#pragma once

#include <stdint.h>

namespace fathom {

#ifndef FATHOM_SPIN_LIMIT
#define FATHOM_SPIN_LIMIT (1 << 22)
#endif
constexpr int kSpinLimit = FATHOM_SPIN_LIMIT;

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Named barriers with compile-time ids (a run-time id reserves all 16).
template <int ID, int COUNT>
__device__ __forceinline__ void bar_sync()
{
    asm volatile("bar.sync %0, %1;\n" ::"n"(ID), "n"(COUNT) : "memory");
}

__device__ __forceinline__ void mbar_init(uint32_t bar, int count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("{\n .reg .b64 st;\n mbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(bar) : "memory");
}

// One arrival on `bar` once every cp.async this thread has issued so far has landed.
__device__ __forceinline__ void cp_async_arrive(uint32_t bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" ::"r"(bar) : "memory");
}

// Wait for the phase of `bar` with the given parity to complete; false if
// the poll limit ran out first.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    for (int it = 0; it < kSpinLimit; ++it) {
        uint32_t ok;
        asm volatile("{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
                     : "=r"(ok) : "r"(bar), "r"(parity), "n"(1000) : "memory");
        if (ok) return true;
    }
    return false;
}

// 16-byte copy of which only the first `bytes` (0..16) are read; the rest is zero-filled.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_addr(smem)), "l"(gmem), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;\n" ::: "memory"); }

}  // namespace fathom
