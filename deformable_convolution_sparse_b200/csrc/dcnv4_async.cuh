// Asynchronous-copy primitives of the sm_100a kernels: mbarriers, bulk copies,
// TMA tensor loads, bounded waits and the device status bits they report
// through. Shared by the forward ring kernel and the predictor.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace dcnv4 {

// Bits of the device status word (dcnv4_device_status()).
constexpr unsigned kStatusCopyTimeout = 1u;     // a copy wait gave up in a kernel
constexpr unsigned kStatusSelftestTimeout = 2u; // the self-test wait gave up (expected)

constexpr uint64_t kCopyWaitLimitNs = 1000000000ull;  // 1 s

// n / d for 0 <= n < 2^31 by multiply-high and shift (Granlund & Montgomery,
// "Division by invariant integers using multiplication", 1994).
struct FastDiv {
    unsigned d, mul, shift;
};

inline FastDiv make_fastdiv(unsigned d) {
    FastDiv f{d, 0u, 0u};
    unsigned s = 0;
    while ((1ull << s) < d) ++s;
    f.shift = s;
    f.mul = static_cast<unsigned>(((1ull << 32) * ((1ull << s) - d)) / d + 1ull);
    if (d == 1) f.mul = 0u;  // q = (0 + n) >> 0
    return f;
}

__device__ __forceinline__ unsigned fdiv(unsigned n, const FastDiv& f) {
    return (__umulhi(n, f.mul) + n) >> f.shift;
}

__device__ __forceinline__ unsigned smem_addr(const void* p) {
    return static_cast<unsigned>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, unsigned bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar))
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Waits for phase `parity` of `bar`, giving up after `limit_ns` nanoseconds.
// The global timer (a slow special-register read) is read only once the first
// try has failed: a phase that has already completed costs one try_wait.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (unsigned i = 1;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255u) == 0u && global_ns() - t0 > limit_ns) return false;
    }
}
// global -> shared bulk copy of `bytes` (multiple of 16; both addresses 16-byte
// aligned) with its byte count posted on `bar` first. No cluster multicast.
__device__ __forceinline__ void bulk_g2s_counted(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
    mbar_expect_tx(bar, bytes);
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}
// One TMA tile load from a 5-D tensor map (no multicast); out-of-range
// elements are written as zeros. The caller posts the byte count.
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, int c3, int c4,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, "
        "%6}], [%7];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(smem_dst)), "l"(gsrc) : "memory");
}
// one arrival on `bar` once every cp.async this thread issued before has landed
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

}  // namespace dcnv4
