// Shared device helpers for the liblsa kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lsa {

constexpr int kStatusBadIndex = 1;   // mirrors LSA_DEV_BAD_INDEX
constexpr int kStatusTimeout = 2;    // mirrors LSA_DEV_TIMEOUT

// Bound of the waits that drain asynchronous copies or MMAs already issued
// before a CTA gives up after a timeout: those always complete, so this bound
// is only a last resort and does not follow the (debug-settable) wait limit.
constexpr long long kDrainNs = 4000000000ll;   // 4 s

// ---------------------------------------------------------------- bf16 bits
// A 32-bit word holding two bf16 values: element 2k in the low half, 2k+1 in
// the high half (little-endian). bf16 -> fp32 is exact: the bf16 bits are the
// high 16 bits of the fp32 value.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// fp32 -> bf16 bits, round to nearest even (via the CUDA intrinsic).
__device__ __forceinline__ uint16_t f2bf(float x) {
    __nv_bfloat16_raw r = __nv_bfloat16_raw(__float2bfloat16_rn(x));
    return r.x;
}

// ---------------------------------------------------------------- order keys
// Monotone map fp32 -> uint32: a < b (as reals) <=> key(a) < key(b);
// -0.0 and +0.0 map to the same key; NaN maps to 0, below every number
// (the key of -inf is 0x007fffff), and NaN is treated as "not a candidate".
__device__ __forceinline__ uint32_t score_key(float x) {
    if (x != x) return 0u;
    x = x + 0.0f;                             // -0.0 -> +0.0
    uint32_t u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Order key -> the smallest float with that key (keys of NaN patterns -> -inf),
// so that s >= key_floor(k) <=> score_key(s) >= k for every non-NaN s.
__device__ __forceinline__ float key_floor(uint32_t k) {
    if (k & 0x80000000u) return __uint_as_float(k & 0x7FFFFFFFu);
    if (k <= 0x007FFFFFu) return -__int_as_float(0x7f800000);
    return __uint_as_float(~k);
}

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

// Non-blocking probe of phase `parity`.
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Potentially blocking probe: the hardware may suspend the thread for a
// system-dependent time before it returns false.
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bounded wait on phase `parity`: gives up after `limit_ns` nanoseconds of
// device time (0: after the first failed probe) or as soon as *abort becomes
// non-zero (abort may be null). Returns false if the phase did not complete.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, long long limit_ns,
                                                  const volatile int* abort = nullptr) {
    if (mbar_test(bar, parity)) return true;
    if (limit_ns <= 0) return false;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (abort && *abort) return false;
        if ((long long)(globaltimer_ns() - t0) > limit_ns) return false;
    }
}

// 1-D bulk copy global -> shared through the TMA unit, completing on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// L2 eviction-priority policies for cache-hinted accesses.
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// bulk_g2s with an L2 cache hint (e.g. evict_first for a read-once stream).
__device__ __forceinline__ void bulk_g2s_hint(void* smem_dst, const void* gmem_src, uint32_t bytes, uint64_t* bar,
                                              uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
            smem_addr(smem_dst)),
        "l"(gmem_src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// fp32 store with an L2 cache hint (e.g. evict_last for data re-read soon).
__device__ __forceinline__ void st_hint(float* p, float v, uint64_t policy) {
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(p), "f"(v), "l"(policy) : "memory");
}

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue now / wait until every prerequisite grid has completed and its
// memory is visible (a no-op without a programmatic dependency).
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// 16-byte cp.async global -> shared; src_bytes = 0 zero-fills the destination.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(smem_dst)), "l"(gmem_src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Streaming 16-byte global load that does not allocate in L1.
__device__ __forceinline__ uint4 ldg_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void set_status(unsigned* status, unsigned bits) {
    if (status) atomicOr(status, bits);
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

}  // namespace lsa
