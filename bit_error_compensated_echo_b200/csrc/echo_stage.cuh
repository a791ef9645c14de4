// echo_stage.cuh -- staging a block's tiles in shared memory with bulk copies
// (the untiled cp.async.bulk of sm_90+, global -> this block's shared
// memory, completing on an mbarrier), and waits that give up after a time
// limit instead of spinning forever.
//
// Only the plain global -> shared form is used: never a multicast form and
// never another GPU's memory.  Source and destination are 16-byte aligned
// and sizes are multiples of 16 bytes; each caller states why.
#pragma once

#include <stdint.h>

namespace echo {

// A wait that has not completed after this long is abandoned: the kernel
// sets kDevErrWaitTimeout in the library's device error word
// (echo_device_error, read and cleared by the host through
// echo_device_error_get) and winds down without computing.
constexpr unsigned long long kWaitLimitNs = 1000000000ull;   // 1 s
constexpr int kDevErrWaitTimeout = 1;

// The device error word of this library on each device (one per context
// that loads the kernels).  Only kernels set bits in it; the host reads it
// (device_error_read).  Being a static in a header, it is one variable only
// because a single translation unit -- echo_launch.cu, the one that
// instantiates the kernels and holds device_error_read -- includes this
// file; another unit that included it would set a copy the host never reads.
static __device__ int echo_device_error;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

// make an initialized barrier visible to the bulk-copy (async) proxy
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// one arrival that also announces the bytes the phase still waits for
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// try_wait may suspend the thread for a while inside the instruction, so a
// loop around it is not a busy poll
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase of the given parity to complete, at most kWaitLimitNs;
// on timeout set the error word and return false.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_ns() - t0 > kWaitLimitNs) {
            atomicOr(&echo_device_error, kDevErrWaitTimeout);
            return false;
        }
    }
    return true;
}

// bulk copy of `bytes` from global src to this block's shared dst,
// completing on bar (both 16-byte aligned, bytes a multiple of 16)
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                              uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

}  // namespace echo
