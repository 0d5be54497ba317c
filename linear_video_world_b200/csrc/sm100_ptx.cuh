// Inline-PTX wrappers shared by the sm_100a kernels: shared-memory addresses, mbarriers
// (with a bounded wait), TMA tile loads and bulk copies, async-proxy fences, and the
// 128-byte-swizzle address map of [rows][128] bf16 tiles staged as two [rows][64] halves.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace hlta {
namespace ptx {

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity)
{
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

// Bounded wait on an mbarrier phase: gives up after `limit` SM cycles (default 2^32, about two
// seconds), or at once when another role of the CTA already gave up (*abort_flag != 0); an
// expiry sets *abort_flag and ORs `code` into the device error word.
__device__ __noinline__ inline bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                              unsigned int *err, unsigned int code,
                                              long long limit = 1LL << 32)
{
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try(bar, parity)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) {
            *abort_flag = 1;
            atomicOr(err, code);
            return false;
        }
    }
}

// 2-D tiled TMA load (box of the tensor map) into shared memory, completing on `bar`
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(bar)
        : "memory");
}

// Contiguous bulk copy global -> shared (both 16-byte aligned, size a multiple of 16)
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// Byte offset of element (r, c) of a [rows][128] bf16 tile staged as two 128B-swizzled
// [rows][64] halves (the layout a SWIZZLE_128B TMA box of 64 columns writes): the 16-byte
// chunk index inside a 128-byte row is XORed with the row index mod 8.
__device__ __forceinline__ uint32_t sw128_off(int r, int c, int rows)
{
    return (uint32_t)(((c >> 6) * rows * 128) + (r << 7) + ((((c >> 3) & 7) ^ (r & 7)) << 4) +
                      ((c & 7) << 1));
}

}  // namespace ptx
}  // namespace hlta
