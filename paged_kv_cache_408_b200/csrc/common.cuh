// common.cuh -- small sm_100a device helpers shared by the libpa kernels:
// mbarriers, 1-D bulk async copies (the TMA engine's untiled form), packed
// fp32x2 FMA, bf16 / fp8 unpacking and the base-2 exponential.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pa.h"

#define PA_DEVICE __device__ __forceinline__

namespace pa {

// ------------------------------------------------------------------ mbarrier
PA_DEVICE uint32_t smem_addr(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

PA_DEVICE void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

PA_DEVICE void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

// Arrive on `bar` and add `bytes` to the transaction count it waits for.
PA_DEVICE void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

PA_DEVICE void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

PA_DEVICE bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

PA_DEVICE uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded waits.  Every wait of a launch shares ONE deadline, taken once per
// thread right after the launch's dependency wait (wait_deadline()), so a
// lost transaction ends the whole launch about kWaitBudgetNs after it
// started, however many waits remain.  Callers stop issuing waits after the
// first failure (they evaluate `ok && mbar_wait(...)`), record
// PA_DEVERR_TIMEOUT, then drain what they have in flight with
// drain_deadline(): a short fresh budget for the copies and MMAs already
// issued, so that no asynchronous write lands after the CTA has exited.
constexpr uint64_t kWaitBudgetNs = 2000000000ull;   // 2 s per launch
constexpr uint64_t kDrainBudgetNs = 20000000ull;    // 20 ms for the drain after a failure

PA_DEVICE uint64_t wait_deadline() { return global_ns() + kWaitBudgetNs; }
PA_DEVICE uint64_t drain_deadline() { return global_ns() + kDrainBudgetNs; }

// Wait for phase `parity` of `bar` to complete, until `deadline` (ns of
// %globaltimer); false if the deadline passed first.
PA_DEVICE bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t deadline) {
    while (!mbar_try_wait(bar, parity))
        if (global_ns() > deadline) return false;
    return true;
}

// ------------------------------------------- programmatic dependent launch
// Every libpa kernel is launched as a programmatic dependent of the kernel
// before it on the stream (launch_pdl below).  Its CTAs may then be
// scheduled while that kernel drains, which hides the launch latency;
// pdl_wait(), placed before the kernel's first global memory access, returns
// once the preceding grid has completed with all its memory operations
// visible, so the ordering is that of a plain launch whatever that kernel
// is.  pdl_trigger() lets the next kernel be scheduled.  Both are no-ops
// when there is no programmatic dependency.
PA_DEVICE void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
PA_DEVICE void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
    return e != cudaSuccess ? e : cudaGetLastError();
}

// ------------------------------------------------------- 1-D bulk async copy
// Global -> shared copy of `bytes` (multiple of 16, both addresses 16-byte
// aligned) completing on `bar` as a transaction.  No multicast.
PA_DEVICE void bulk_g2s(void *dst_smem, const void *src_gmem, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// Fetch the 128-byte line holding p into L2 (no register result, no wait).
PA_DEVICE void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// Named barrier `id` (1..15) over `nthreads` threads (a multiple of 32).
PA_DEVICE void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Arrive on named barrier `id` without waiting for it (the other threads of
// the count wait with named_bar_sync).  A thread must not arrive on the same
// barrier again before that phase completes.
PA_DEVICE void named_bar_arrive(int id, int nthreads) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ----------------------------------------------------------------- arithmetic
// Packed fp32x2 fused multiply-add (sm_100): d = a * b + c, lane-wise, RN.
PA_DEVICE float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;"
        : "=l"(reinterpret_cast<unsigned long long &>(d))
        : "l"(reinterpret_cast<unsigned long long &>(a)), "l"(reinterpret_cast<unsigned long long &>(b)),
          "l"(reinterpret_cast<unsigned long long &>(c)));
    return d;
}

PA_DEVICE float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("mul.rn.f32x2 %0, %1, %2;"
        : "=l"(reinterpret_cast<unsigned long long &>(d))
        : "l"(reinterpret_cast<unsigned long long &>(a)), "l"(reinterpret_cast<unsigned long long &>(b)));
    return d;
}

PA_DEVICE float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("add.rn.f32x2 %0, %1, %2;"
        : "=l"(reinterpret_cast<unsigned long long &>(d))
        : "l"(reinterpret_cast<unsigned long long &>(a)), "l"(reinterpret_cast<unsigned long long &>(b)));
    return d;
}

// Three-input maximum (sm_100).
PA_DEVICE float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x with the hardware approximation (MUFU.EX2), flushing denormal results.
PA_DEVICE float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log2(x) with the hardware approximation (MUFU.LG2).
PA_DEVICE float lg2(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two bf16 packed in one 32-bit word -> (low element, high element) as fp32.
// bf16 is the upper half of a binary32, so widening is a shift / mask.
PA_DEVICE float2 bf16x2_to_float2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Two E4M3 codes packed in 16 bits (low byte first) -> fp32 pair.
PA_DEVICE float2 e4m3x2_to_float2(uint16_t w) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w), __NV_E4M3);
    return __half22float2(*reinterpret_cast<__half2 *>(&h));
}

// Two E4M3 codes (low byte first) -> f16x2 (low element first), exact:
// every E4M3 value is an f16 normal number or zero.
PA_DEVICE uint32_t e4m3x2_to_h2(uint32_t w16) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w16 & 0xffffu), __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// Device status word (PA_DEVERR_* bits).
PA_DEVICE void flag_error(unsigned *err, unsigned bits) {
    if (err) atomicOr(err, bits);
}

}  // namespace pa
