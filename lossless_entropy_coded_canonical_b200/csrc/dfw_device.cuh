// dfw_device.cuh -- device helpers shared by the decode kernels (one
// translation unit: included by dfw_decode.cu only).
#pragma once

#include <cuda_runtime.h>

#include "dfw_internal.h"

namespace dfw {
namespace {

constexpr uint32_t ESC_BAD = 0x40000000u;

// The checks build (DFW_CHECKS): check(ok, site) records a failed range check
// (status bit and the first failing site) and returns whether the access may
// go ahead; in the ordinary build it is the constant true and costs nothing.
#ifdef DFW_CHECKS
__device__ __noinline__ void check_failed(uint32_t site) {
    atomicOr(&g_status, ST_CHECK);
    atomicCAS(&g_check_site, 0u, site);
}
__device__ __forceinline__ bool check(bool ok, uint32_t site) {
    if (!ok) check_failed(site);
    return ok;
}
#else
__device__ __forceinline__ constexpr bool check(bool, uint32_t) { return true; }
#endif
constexpr unsigned long long WAIT_LIMIT_NS = 2000000000ull;  // 2 s, far above any copy

// --------------------------------------------------------------- PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's earlier generic accesses to shared memory (made
// visible to it by a barrier) before its later bulk-copy writes.
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory; 16-byte aligned addresses
// and a size that is a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// 1-D bulk copy this CTA's shared memory -> global, tracked in a bulk group.
__device__ __forceinline__ void bulk_store(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until this thread's bulk stores have read their shared memory.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// Waits until this thread's bulk stores have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0u;
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits for a phase of an mbarrier with a time and iteration limit; false if
// it gave up.
__device__ __noinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (uint32_t it = 0; it < (1u << 24); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > WAIT_LIMIT_NS) break;
    }
    return false;
}

// Waits for a phase of an mbarrier: one inline try (the copy has usually
// landed by now), the bounded loop only if that fails.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    return mbar_try_wait(bar, parity) || mbar_wait_bounded(bar, parity);
}

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

// Shared-memory accesses by 32-bit shared-window address.
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
    return v;
}
// A 16-bit shared load only where p holds (0 elsewhere), without a branch.
__device__ __forceinline__ uint32_t lds16_if(bool p, uint32_t a) {
    uint32_t v = 0;
    asm volatile(
        "{\n\t.reg .pred q;\n\t.reg .b16 h;\n\t"
        "setp.ne.u32 q, %1, 0;\n\t"
        "mov.b16 h, 0;\n\t"
        "@q ld.shared.u16 h, [%2];\n\t"
        "cvt.u32.u16 %0, h;\n\t}"
        : "+r"(v)
        : "r"((uint32_t)p), "r"(a)
        : "memory");
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t v) {
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

// 32-byte streaming store (sm_100 256-bit vector store): one whole L2 sector
// per thread; the address must be 32-byte aligned.
__device__ __forceinline__ void stg256_cs(void *p, uint4 a, uint4 b) {
    asm volatile("st.global.cs.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y),
                 "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
}

// 32-byte read-only load (sm_100 256-bit vector load); 32-byte aligned address.
__device__ __forceinline__ void ldg256_nc(const void *p, uint4 &a, uint4 &b) {
    asm volatile("ld.global.nc.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w)
                 : "l"(p));
}

// acc + w.lo * x.lo, then + w.hi * x.hi: two bf16 pairs, fp32 accumulation
// (the product of two bf16 values is exact in the fused multiply-add).
__device__ __forceinline__ float fma2_bf16(uint32_t w, uint32_t x, float acc) {
    asm("{\n\t.reg .b16 wl, wh, xl, xh;\n\t"
        "mov.b32 {wl, wh}, %1;\n\t"
        "mov.b32 {xl, xh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, wl, xl, %0;\n\t"
        "fma.rn.f32.bf16 %0, wh, xh, %0;\n\t}"
        : "+f"(acc)
        : "r"(w), "r"(x));
    return acc;
}

// --------------------------------------------------------------- decoding

// A codeword longer than the fast table's key: walk the byte-keyed hierarchy
// (global memory, read-only path).  x holds the 32 stream bits from the
// codeword's first bit.  Returns a hierarchy leaf (symbol, total length), or
// on a corrupt table ESC_BAD with length 1.
__device__ __noinline__ uint32_t resolve_escape(uint32_t x, const uint32_t *__restrict__ g_hier,
                                                uint32_t n_tables) {
    uint32_t e = __ldg(g_hier + (x >> 24));
#pragma unroll 1
    for (int level = 1; level < 4 && (e & LUT_PTR); ++level) {
        const uint32_t child = e & LUT_CHILD_MASK;
        if (child >= n_tables) break;
        e = __ldg(g_hier + child * 256u + ((x >> (24 - 8 * level)) & 0xFFu));
        if (!(e & LUT_PTR)) {
            const uint32_t l = (e >> LUT_LEN_SHIFT) & 63u;
            if (l > 8u * level && l <= 8u * level + 8u) return e;
            break;
        }
    }
    return ESC_BAD | (1u << LUT_LEN_SHIFT);  // length 1 keeps the walk finite
}

// Exponent symbols are kept rotated right by one bit, r = (e >> 1) | (e << 7)
// (mod 256): bits 6..0 of r are the bf16 pattern's high byte below the sign,
// bit 7 of r is the top bit of its low byte.  The fast table stores its
// symbols this way; a symbol from the byte-keyed hierarchy is rotated here.
// Only the low byte of e is used (a hierarchy leaf carries its length above).
__device__ __forceinline__ uint32_t rot_sym(uint32_t e) { return ((e & 0xFFu) >> 1) | ((e & 1u) << 7); }

// Four (rotated exponent, raw byte) pairs -> four bf16 patterns in two words.
__device__ __forceinline__ void join4(uint32_t R, uint32_t M, uint32_t &w0, uint32_t &w1) {
    const uint32_t hi = (M & 0x80808080u) | (R & 0x7F7F7F7Fu);  // sign | exp[7:1]
    const uint32_t lo = (R & 0x80808080u) | (M & 0x7F7F7F7Fu);  // exp[0] | mant
    w0 = __byte_perm(lo, hi, 0x5140);
    w1 = __byte_perm(lo, hi, 0x7362);
}

__device__ __forceinline__ uint16_t join1(uint32_t r, uint32_t m) {
    return (uint16_t)((((m & 0x80u) | (r & 0x7Fu)) << 8) | (r & 0x80u) | (m & 0x7Fu));
}

// One distinct exponent: every weight is (sym, raw byte).
__global__ void fill_single(const uint8_t *__restrict__ mant, uint32_t sym, uint64_t n,
                            uint16_t *__restrict__ out) {
    const uint32_t E = rot_sym(sym) * 0x01010101u;
    const uint64_t nfull = n >> 3;
    for (uint64_t c = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; c < nfull;
         c += (uint64_t)gridDim.x * blockDim.x) {
        const uint2 m = __ldcs(reinterpret_cast<const uint2 *>(mant + (c << 3)));
        uint4 r;
        join4(E, m.x, r.x, r.y);
        join4(E, m.y, r.z, r.w);
        __stcs(reinterpret_cast<uint4 *>(out + (c << 3)), r);
    }
    if (blockIdx.x == 0 && threadIdx.x < (n & 7)) {
        const uint64_t j = (nfull << 3) + threadIdx.x;
        out[j] = join1(rot_sym(sym), mant[j]);
    }
}

}  // namespace
}  // namespace dfw
