// 5th-generation tensor-core (tcgen05) primitives for sm_100a, as inline PTX:
// tensor-memory allocation, the bf16 MMA with its fp32 accumulator in tensor
// memory, commit to an mbarrier, tensor-memory loads, and the shared-memory
// matrix descriptors of 128-byte-swizzled K-major tiles.  Plus 4D tensor-copy
// loads and waits that give up when another role of the CTA has given up.
// Every MMA here is the one-CTA form (cta_group::1); no load is broadcast to a
// cluster.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "tma.cuh"

namespace tok {

// ---------------------------------------------------------------------------
// Tensor memory.  alloc / relinquish / dealloc are executed by one whole warp.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Order tensor-core operations against thread synchronization (barriers, mbarrier waits).
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---------------------------------------------------------------------------
// MMA: D[tmem] (+)= A[smem] x B[smem]^T, bf16 operands, fp32 accumulator, issued
// by one thread.  accumulate == 0 overwrites D.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile("{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
                 " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
                 "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// One arrive on the mbarrier once every tensor-core operation this thread issued
// before has completed (its shared-memory operands may then be overwritten).
__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// Instruction descriptor of kind::f16: bf16 A and B (both K-major), fp32 D, M x N.
// Fields: D format bits [4,6) = 1 (f32); A format [7,10) = 1 (bf16); B format
// [10,13) = 1 (bf16); transposes (bits 15, 16) = 0 (K-major); N >> 3 in [17,23);
// M >> 4 in [24,29).
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory descriptor of a K-major tile with 128-byte rows (64 bf16 of K per
// row) in the 128-byte swizzle: rows 128 bytes apart, groups of 8 rows 1024 bytes
// apart (stride field), 16-byte chunk c of row r stored at chunk c ^ (r % 8), tile
// base on a 1024-byte boundary.  Fields: start address >> 4 in [0,14); leading
// offset (unused by swizzled K-major tiles, 1) in [16,30); stride offset 1024 >> 4
// in [32,46); descriptor version 1 in [46,48); base offset 0; layout 2 (128-byte
// swizzle) in [61,64).  The K steps of 16 elements inside the 128-byte row advance
// the start address by 32 bytes (add 2).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Byte offset of element k (0..63) of row r in a 128-byte-swizzled K-major tile.
__host__ __device__ constexpr uint32_t sw128_offset(uint32_t r, uint32_t k)
{
    return r * 128u + ((((k >> 3) ^ r) & 7u) << 4) + (k & 7u) * 2u;
}

// 32 lanes x 32 consecutive 32-bit columns of tensor memory into 32 registers per
// thread (thread i gets lane base + i).  Complete with tmem_wait_ld().
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                 "%13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
                 "[%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
                   "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
                   "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
                   "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Tensor copies and barriers.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                            uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];"
                 ::"r"(dst), "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Wait for phase `parity` of the barrier.  Gives up (false) after kWaitPolls polls,
// raising the CTA's abort flag, or as soon as another role has raised it; every role
// then leaves its loop, so no thread of the CTA waits for work that will not come.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int *abort)
{
    for (uint32_t i = 0; i < kWaitPolls; ++i) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((i & 31u) == 31u && *abort)
            return false;
    }
    *abort = 1;
    return false;
}

// Host: a tiled tensor map in the 128-byte swizzle (bf16; innermost box 64 elements
// = 128 bytes), zero fill out of bounds.  dims / box innermost first; strides are the
// byte strides of dims 1..rank-1.  False if the driver rejects it.
bool encode_tensor_map_sw128(CUtensorMap *map, int rank, const void *base, const uint64_t *dims,
                             const uint64_t *strides_bytes, const uint32_t *box);

} // namespace tok
