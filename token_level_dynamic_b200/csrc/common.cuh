// common.cuh -- device-side helpers shared by the libwide kernels (sm_100a).
//
// Inline-PTX wrappers for mbarriers, TMA tensor copies and timers, the
// bounded wait every spin in this library goes through, and small numeric
// helpers.  Nothing here is specific to one kernel.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "wide.h"

namespace wide {

// A bounded wait gives up after this many nanoseconds of %globaltimer.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void set_status(int32_t *status, int bits)
{
    if (status)
        atomicOr(status, bits);
}

// ------------------------------------------------------------- mbarriers

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// As mbar_try_wait, but the thread may be suspended (not spinning, so it
// takes no issue slots from other warps) until the phase completes or
// kSuspendNs elapse.
constexpr uint32_t kSuspendNs = 1000000;   // 1 ms
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendNs)
        : "memory");
    return ok != 0;
}

// Waits for the phase with the given parity to complete.  Returns false if
// it has not completed after kWaitLimitNs (the caller then reports
// WIDE_DEV_TIMEOUT and winds down instead of waiting for ever).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = globaltimer();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity))
            return true;
        if (globaltimer() - t0 > kWaitLimitNs)
            return false;
    }
}

// ------------------------------------------------------------ TMA copies
// Tile-mode tensor copies global -> shared completing on an mbarrier; each
// CTA loads its own tiles from this GPU's memory.

__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, int32_t x,
                                            int32_t y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, int32_t x,
                                            int32_t y, int32_t z, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(void *smem_dst, const CUtensorMap *map, int32_t x,
                                            int32_t y, int32_t z, int32_t w, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar))
        : "memory");
}

// Untiled bulk copy of `bytes` contiguous bytes global -> shared, completing
// on an mbarrier.  Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes,
                                          uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------- cp.async
// 16-byte global -> shared copy that bypasses L1.
__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void *gsrc)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_dst), "l"(gsrc)
                 : "memory");
}
// As cp_async16, but copies src_bytes (0 or 16) bytes and fills the rest of
// the 16 with zeros: with 0, nothing is read from global memory (src must
// still be a valid address) and the destination is zeroed.
__device__ __forceinline__ void cp_async16_zfill(uint32_t smem_dst, const void *gsrc,
                                                 uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_dst), "l"(gsrc),
                 "r"(src_bytes)
                 : "memory");
}
// Arrive on the mbarrier once every cp.async this thread issued so far has
// completed; the barrier's expected count already includes this arrive.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void cp_async_wait_all()
{
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// Byte offset of 16-byte chunk j of row r in a tile of 128-byte rows written
// by TMA with CU_TENSOR_MAP_SWIZZLE_128B (tile base 1024-byte aligned).
__device__ __forceinline__ uint32_t swz128(uint32_t r, uint32_t j)
{
    return r * 128u + (((j ^ r) & 7u) << 4);
}

// Element (t, col) of a [T][ld] fp32 activation stored with token pairs
// interleaved: row t/2 holds, for every column, the values of tokens t and
// t+1 side by side, so a packed fp32x2 FMA can take two tokens at once.
__host__ __device__ __forceinline__ size_t il2(int t, size_t col, size_t ld)
{
    return (size_t)(t >> 1) * 2 * ld + col * 2 + (size_t)(t & 1);
}

// ------------------------------------------------------------- numerics

// Word i (0..3, a compile-time index after unrolling) of a 16-byte chunk.
__device__ __forceinline__ uint32_t word(const uint4 v, int i)
{
    return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

// The bf16 in the low / high half of w as fp32 (byte permutes: exact).
__device__ __forceinline__ float bf_lo(uint32_t w) { return __uint_as_float(__byte_perm(w, 0u, 0x1044)); }
__device__ __forceinline__ float bf_hi(uint32_t w) { return __uint_as_float(__byte_perm(w, 0u, 0x3244)); }
// ... in both halves of a register pair (the weight operand of a token
// pair), each half written by its own byte permute
__device__ __forceinline__ float2 dup_lo(uint32_t w)
{
    uint32_t a, b;
    asm("prmt.b32 %0, %2, 0, 0x1044;\n\tprmt.b32 %1, %2, 0, 0x1044;" : "=r"(a), "=r"(b) : "r"(w));
    return make_float2(__uint_as_float(a), __uint_as_float(b));
}
__device__ __forceinline__ float2 dup_hi(uint32_t w)
{
    uint32_t a, b;
    asm("prmt.b32 %0, %2, 0, 0x3244;\n\tprmt.b32 %1, %2, 0, 0x3244;" : "=r"(a), "=r"(b) : "r"(w));
    return make_float2(__uint_as_float(a), __uint_as_float(b));
}


// Widens 8 bf16 values (one 16-byte chunk) to fp32 exactly.
__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&f)[8])
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(float v) { return v; }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v)
{
    return __float2bfloat16_rn(v);
}

// SiLU(a) = a * sigmoid(a).  Written as a / (1 + e^-a) with CUDA's expf.
__device__ __forceinline__ float silu_f32(float a) { return a / (1.0f + expf(-a)); }

}  // namespace wide
