// Device-side helpers shared by the libccq kernels (sm_100a): error word, mbarriers with bounded
// waits, TMA (cp.async.bulk.tensor) loads, and small bit utilities.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ccq {

// ------------------------------------------------------------------------------------------------
// Device error word: the first 16 bytes of every MoE workspace.  Kernels OR a code into word 0
// and record the first offending index in word 1; nothing traps.
// ------------------------------------------------------------------------------------------------
enum : uint32_t {
    DEV_ERR_BAD_EXPERT = 1u,   // expert id outside [0, E)
    DEV_ERR_DUP_EXPERT = 2u,   // the same expert twice within one token
    DEV_ERR_TIMEOUT = 4u,      // a bounded wait gave up
};

__device__ __forceinline__ void record_error(uint32_t *err, uint32_t code, uint32_t where) {
    if (err) {
        uint32_t old = atomicOr(err, code);
        if (old == 0u) atomicExch(err + 1, where);
    }
}

// Time limit for every mbarrier wait (ns of %globaltimer): a healthy pipeline waits microseconds.
// On expiry the waiter records DEV_ERR_TIMEOUT and returns false; callers then stop waiting.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Programmatic dependent launch.  pdl_wait: block until the grids this one depends on have
// completed and their memory is visible (a no-op when the launch carries no such dependency).
// pdl_trigger: let the next grid in the stream, if launched with programmatic serialization, be
// scheduled now (it still waits in its own pdl_wait before touching this grid's results).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile(
        "{\n\t.reg .b64 st;\n\t"
        "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
        "r"(bytes)
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that may suspend the thread for up to `ns` nanoseconds while the phase is incomplete
// (it resumes as soon as the phase completes), so a waiting warp does not take issue slots from
// the warps that compute.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint64_t *bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Bounded wait on phase `parity`; returns false (and records a timeout) if it does not complete
// within limit_ns.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t *err,
                                          uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        for (int i = 0; i < 8; ++i)
            if (mbar_try_wait_suspend(bar, parity, 20000u)) return true;
        if (global_ns() - t0 > limit_ns) break;
    }
    record_error(err, DEV_ERR_TIMEOUT, 0xFFFFFFFFu);
    return false;
}

__device__ __forceinline__ int ld_acquire_gpu(const int *ptr) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

// Bounded wait until *ctr >= need (another CTA's release); false (and a recorded timeout) after
// limit_ns.
__device__ __forceinline__ bool wait_counter(const int *ctr, int need, uint32_t *err,
                                             uint64_t limit_ns = kWaitLimitNs) {
    if (ld_acquire_gpu(ctr) >= need) return true;
    const uint64_t t0 = global_ns();
    for (;;) {
        __nanosleep(200);
        if (ld_acquire_gpu(ctr) >= need) return true;
        if (global_ns() - t0 > limit_ns) break;
    }
    record_error(err, DEV_ERR_TIMEOUT, 0xFFFFFFFEu);
    return false;
}

// 2D / 3D tiled TMA loads into shared memory, completing on an mbarrier (no multicast).
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int32_t x,
                                            int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int32_t x,
                                            int32_t y, int32_t z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// BF16 bit patterns <-> float.
__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) { return __uint_as_float(uint32_t(b) << 16); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float f) {
    return static_cast<uint16_t>(pack_bf16x2(f, 0.0f) & 0xFFFFu);
}

}  // namespace ccq
