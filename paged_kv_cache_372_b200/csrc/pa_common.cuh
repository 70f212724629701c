// Device helpers shared by the kernels of libpa_b200: mbarrier and bulk-copy
// (TMA) wrappers in inline PTX for sm_100a, element conversions, and the
// per-device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

// Acquire fence at GPU scope.
__device__ __forceinline__ void fence_acquire_gpu() { asm volatile("fence.acquire.gpu;" ::: "memory"); }

// Atomic add at GPU scope with release semantics; returns the old value.
__device__ __forceinline__ int atomic_add_release_gpu(int *addr, int v) {
    int old;
    asm volatile("atom.release.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(addr), "r"(v) : "memory");
    return old;
}

// Counts one finished partition of a partitioned result and reports whether
// it was the last of `total`. The warp's lanes have stored their partial
// results; the warp barrier orders those stores before the counting lane's
// atomic, whose release semantics publish them at GPU scope (happens-before
// is transitive through the barrier). The lane that completes the count
// takes an acquire fence after its atomic, and the second warp barrier
// extends that to the other lanes, which then read every partition's
// partials: the release / acquire pattern of the PTX memory model. (Measured
// against a full acquire-release fence before a relaxed atomic: 2-3% faster
// on the calls that merge in the attention kernel.)
__device__ __forceinline__ bool count_partition(int *counter, int total, bool counting_lane) {
    __syncwarp();
    bool last = false;
    if (counting_lane) {
        last = atomic_add_release_gpu(counter, 1) == total - 1;
        if (last) fence_acquire_gpu();
    }
    __syncwarp();
    return last;
}


constexpr unsigned FULL_MASK = 0xffffffffu;

// Per-device error word. Kernels OR PA_DEVERR_* bits into it instead of
// faulting on a bad index; pa_device_errors() reads and clears it.
__device__ unsigned int g_device_errors;

__device__ __forceinline__ void raise_error(unsigned bits) { atomicOr(&g_device_errors, bits); }

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's generic-proxy shared-memory accesses before later
// async-proxy (TMA) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

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

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits for the phase with the given parity to complete, for at most
// limit_ns nanoseconds. Returns false if the limit ran out.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_timer_ns() - t0 > limit_ns) return false;
    }
}

// ---- bulk copy global -> this CTA's shared memory (TMA, no tensor map) -------
// dst and src 16-byte aligned, bytes a multiple of 16. Completion is counted
// on the mbarrier as transaction bytes.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar,
                                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// ---- 16-bit element types ---------------------------------------------------
template <typename T>
struct Elem;

// fp16: IEEE binary16, converted with the hardware cvt instructions.
template <>
struct Elem<__half> {
    static __device__ __forceinline__ float2 pair(uint32_t w) {
        return __half22float2(*reinterpret_cast<const __half2 *>(&w));
    }
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __half2 h = __floats2half2_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
};

// bf16: the upper 16 bits of an IEEE binary32, so widening is a shift/mask.
// Element 0 of a 32-bit word is its low half (little-endian storage).
template <>
struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float2 pair(uint32_t w) {
        return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
    }
    static __device__ __forceinline__ uint32_t pack(float a, float b) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
        return *reinterpret_cast<uint32_t *>(&h);
    }
};

template <typename T>
__device__ __forceinline__ void unpack8(const uint4 &raw, float (&f)[8]) {
    const float2 a = Elem<T>::pair(raw.x), b = Elem<T>::pair(raw.y);
    const float2 c = Elem<T>::pair(raw.z), d = Elem<T>::pair(raw.w);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

}  // namespace pa
