// Tensor-memory-accelerator (TMA) copies and mbarrier waits shared by the
// kernels: tiled bulk loads global -> shared (completion counted on an
// mbarrier), tiled bulk stores shared -> global (bulk groups), and host-side
// tensor-map encoding through the driver entry point.  No multicast form is
// used anywhere.  Every wait is bounded in time.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace slstm {

SLSTM_DEVINL uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

SLSTM_DEVINL void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async proxy (TMA).
SLSTM_DEVINL void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

SLSTM_DEVINL void mbar_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

SLSTM_DEVINL bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n"
        " .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0u;
}

// Wait for the phase of `bar` with the given parity to complete; false when
// the time bound passes first.
SLSTM_DEVINL bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns = 1000000000ull)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer_ns() - t0 > limit_ns) return false;
    return true;
}

SLSTM_DEVINL void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

SLSTM_DEVINL void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1, int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
        "[%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

SLSTM_DEVINL void tma_load_4d(void *dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1, int c2, int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], "
        "[%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// Contiguous bulk copy global -> shared; size, src and dst multiples of 16 bytes.
SLSTM_DEVINL void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Store a box from shared memory; elements outside the tensor are not
// written.  The caller makes its shared-memory writes visible first
// (tma_store_fence by every writing thread, then a barrier or __syncwarp).
SLSTM_DEVINL void tma_store_3d(const CUtensorMap *map, const void *src, int c0, int c1, int c2)
{
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}

SLSTM_DEVINL void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

SLSTM_DEVINL void tma_store_2d(const CUtensorMap *map, const void *src, int c0, int c1)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1)
                 : "memory");
}

// The source shared memory of all but the most recent committed bulk store
// group may be reused.
SLSTM_DEVINL void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// At most three of this thread's bulk store groups still read shared memory.
SLSTM_DEVINL void bulk_wait_read_3() { asm volatile("cp.async.bulk.wait_group.read 3;" ::: "memory"); }

SLSTM_DEVINL void tma_store_fence() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
SLSTM_DEVINL void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// The source shared memory of every committed bulk store may be reused.
SLSTM_DEVINL void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Every committed bulk store has completed.
SLSTM_DEVINL void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Host: the driver's cuTensorMapEncodeTiled, or null.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();

// Host: fp32 tensor of dims (n0 contiguous, n1, n2) with row strides ld1 and
// ld2 elements, box (b0, b1, 1), no swizzle, zero fill out of bounds.  False
// when the driver refuses (alignment: base and strides multiples of 16 bytes).
bool make_map_f32_3d(CUtensorMap *map, const void *base, uint64_t n0, uint64_t n1, uint64_t n2, uint64_t ld1,
                     uint64_t ld2, uint32_t b0, uint32_t b1);

// Host: fp32 tensor of dims (n0 contiguous, n1, n2, n3) with row strides ld1,
// ld2, ld3 elements, box (b0, 1, b2, 1), no swizzle, zero fill out of bounds.
bool make_map_f32_4d(CUtensorMap *map, const void *base, uint64_t n0, uint64_t n1, uint64_t n2, uint64_t n3,
                     uint64_t ld1, uint64_t ld2, uint64_t ld3, uint32_t b0, uint32_t b2);

}  // namespace slstm
