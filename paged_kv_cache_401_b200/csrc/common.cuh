// Device helpers shared by the paged-KV kernels (sm_100a): mbarrier and bulk
// async copies (the TMA engine's 1-D form), bounded waits, element decoders.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "paged_kv.h"

namespace pkv {

constexpr int kBlockTokens = 16;  // tokens per paged block (the pages' default of 16)

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Make barrier initialisation visible to the async (bulk-copy) proxy.
__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// One poll of an mbarrier phase.  A thread whose phase is not complete may be
// suspended until it completes or a time limit passes: the hardware's own limit
// (SUSPEND_NS = 0), else SUSPEND_NS nanoseconds.
template <uint32_t SUSPEND_NS = 0>
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    if constexpr (SUSPEND_NS == 0) {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_addr(bar)), "r"(parity)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(smem_addr(bar)), "r"(parity), "n"(SUSPEND_NS)
            : "memory");
    }
    return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// A wait on staged data never spins forever: it gives up after ~2 s of wall
// time (or 2^30 polls) and reports false; the caller records KV_DEVERR_TIMEOUT.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

template <uint32_t SUSPEND_NS = 0>
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait<SUSPEND_NS>(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0; it < (1u << 30); ++it) {
        if (mbar_try_wait<SUSPEND_NS>(bar, parity)) return true;
        if ((it & 63u) == 63u && globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
    return false;
}

// ---- bulk async copy global -> shared (no multicast) ------------------------
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                              uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// ---- programmatic dependent launch -------------------------------------------
// Every kernel of the library waits for the grid before it in the stream to
// finish (and its writes to be visible) before touching global memory.  The
// short kernels then let the next grid start launching at once, so its launch
// and prologue overlap their tail; the persistent decode kernel does not (its
// dependents start as it exits).  Without the launch attribute both
// instructions are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- error word --------------------------------------------------------------
__device__ __forceinline__ void report(int32_t* dev_error, int32_t bits) {
    if (dev_error != nullptr) atomicOr(dev_error, bits);
}

// ---- element decoders ----------------------------------------------------------
// Two bf16 packed in a 32-bit word -> two fp32 (exact: bf16 is the top half of fp32).
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// Two E4M3 codes packed in 16 bits -> two fp32 (exact: E4M3 -> f16 -> f32).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t w16) {
    uint32_t h2;
    asm("{\n\t.reg .b16 lo;\n\tcvt.u16.u32 lo, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}"
        : "=r"(h2)
        : "r"(w16));
    const __half2 h = *reinterpret_cast<const __half2*>(&h2);
    return __half22float2(h);
}

// Two signed 8-bit codes (low 16 bits of w16, low byte first) -> two floats,
// exact.  Each code c is flipped to the biased byte c + 128, placed in the
// mantissa of 2^23 (bit pattern 0x4B0000xx = 2^23 + c + 128) and the bias
// subtracted.
__device__ __forceinline__ float2 i8x2_to_float2(uint32_t w16) {
    const uint32_t u = w16 ^ 0x8080u;
    const float bias = 8388608.0f + 128.0f;
    return make_float2(__uint_as_float(__byte_perm(u, 0x4B000000u, 0x7650)) - bias,
                       __uint_as_float(__byte_perm(u, 0x4B000000u, 0x7651)) - bias);
}

// Two fp32 -> two E4M3 codes (round to nearest even, finite overflow saturates
// to +-448), low byte = first argument.
__device__ __forceinline__ uint32_t float2_to_e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

}  // namespace pkv
