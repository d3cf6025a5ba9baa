// Shared helpers of the sm_100a kernels behind tok.h: argument checks that run on
// the host, and the global-memory load/store forms the kernels use.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tok.h"

namespace tok {

// ---------------------------------------------------------------------------
// Host-side argument checks.
// ---------------------------------------------------------------------------

// a * b into *out; false on overflow or a negative factor.
inline bool mul_ok(int64_t a, int64_t b, int64_t *out)
{
    if (a < 0 || b < 0)
        return false;
    return !__builtin_mul_overflow(a, b, out);
}

inline bool prod_ok(std::initializer_list<int64_t> f, int64_t *out)
{
    int64_t p = 1;
    for (int64_t v : f)
        if (!mul_ok(p, v, &p))
            return false;
    *out = p;
    return true;
}

inline bool overlaps(const void *a, int64_t abytes, const void *b, int64_t bbytes)
{
    const uintptr_t a0 = (uintptr_t)a, b0 = (uintptr_t)b;
    return a0 < b0 + (uintptr_t)bbytes && b0 < a0 + (uintptr_t)abytes;
}

inline bool aligned(const void *p, uintptr_t n) { return ((uintptr_t)p % n) == 0; }

// Records the CUDA error of a failed launch for tok_last_cuda_error().
tok_status launch_status();

// ---------------------------------------------------------------------------
// Device-side memory access.  ld_stream_* bypass L1 allocation (used by the
// FSQ register kernels, where they measured faster).  Outputs use plain stores
// (the next kernel of a pipeline may find the tail of them in L2).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint4 ld_stream_u4(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ uint2 ld_stream_u2(const void *p)
{
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
    return r;
}

__device__ __forceinline__ uint32_t ld_stream_u1(const void *p)
{
    uint32_t r;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(r) : "l"(p));
    return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Round two floats to bf16 (nearest even) and pack them, `lo` at the lower address.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&p);
}

// N consecutive elements of type T <-> floats.  VEC: p is aligned to
// min(16, N * sizeof(T)) bytes and the widest vector form is used (plain
// cached loads: measured faster than L1::no_allocate for these kernels);
// otherwise element-wise accesses.
template <typename T, int N, bool VEC> struct Row;

template <int N, bool VEC> struct Row<float, N, VEC> {
    static __device__ __forceinline__ void load(const float *p, float *v)
    {
        if constexpr (VEC && N % 4 == 0) {
#pragma unroll
            for (int k = 0; k < N / 4; ++k) {
                const uint4 r = *reinterpret_cast<const uint4 *>(p + 4 * k);
                v[4 * k + 0] = __uint_as_float(r.x);
                v[4 * k + 1] = __uint_as_float(r.y);
                v[4 * k + 2] = __uint_as_float(r.z);
                v[4 * k + 3] = __uint_as_float(r.w);
            }
        } else if constexpr (VEC && N == 2) {
            const uint2 r = *reinterpret_cast<const uint2 *>(p);
            v[0] = __uint_as_float(r.x);
            v[1] = __uint_as_float(r.y);
        } else {
#pragma unroll
            for (int k = 0; k < N; ++k)
                v[k] = __uint_as_float(ld_stream_u1(p + k));
        }
    }
    static __device__ __forceinline__ void store(float *p, const float *v)
    {
        if constexpr (VEC && N % 4 == 0) {
#pragma unroll
            for (int k = 0; k < N / 4; ++k)
                *reinterpret_cast<float4 *>(p + 4 * k) = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
        } else if constexpr (VEC && N == 2) {
            *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
        } else {
#pragma unroll
            for (int k = 0; k < N; ++k)
                p[k] = v[k];
        }
    }
};

template <int N, bool VEC> struct Row<__nv_bfloat16, N, VEC> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float *v)
    {
        if constexpr (VEC && N % 8 == 0) {
#pragma unroll
            for (int k = 0; k < N / 8; ++k) {
                const uint4 r = *reinterpret_cast<const uint4 *>(p + 8 * k);
                v[8 * k + 0] = bf16_lo(r.x);
                v[8 * k + 1] = bf16_hi(r.x);
                v[8 * k + 2] = bf16_lo(r.y);
                v[8 * k + 3] = bf16_hi(r.y);
                v[8 * k + 4] = bf16_lo(r.z);
                v[8 * k + 5] = bf16_hi(r.z);
                v[8 * k + 6] = bf16_lo(r.w);
                v[8 * k + 7] = bf16_hi(r.w);
            }
        } else if constexpr (VEC && N == 4) {
            const uint2 r = *reinterpret_cast<const uint2 *>(p);
            v[0] = bf16_lo(r.x);
            v[1] = bf16_hi(r.x);
            v[2] = bf16_lo(r.y);
            v[3] = bf16_hi(r.y);
        } else if constexpr (VEC && N == 2) {
            const uint32_t r = *reinterpret_cast<const uint32_t *>(p);
            v[0] = bf16_lo(r);
            v[1] = bf16_hi(r);
        } else {
            const unsigned short *q = reinterpret_cast<const unsigned short *>(p);
#pragma unroll
            for (int k = 0; k < N; ++k)
                v[k] = __uint_as_float(((uint32_t)__ldg(q + k)) << 16);
        }
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float *v)
    {
        if constexpr (VEC && N % 8 == 0) {
#pragma unroll
            for (int k = 0; k < N / 8; ++k)
                *reinterpret_cast<uint4 *>(p + 8 * k) =
                    make_uint4(pack_bf16x2(v[8 * k + 0], v[8 * k + 1]), pack_bf16x2(v[8 * k + 2], v[8 * k + 3]),
                               pack_bf16x2(v[8 * k + 4], v[8 * k + 5]), pack_bf16x2(v[8 * k + 6], v[8 * k + 7]));
        } else if constexpr (VEC && N == 4) {
            *reinterpret_cast<uint2 *>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
        } else if constexpr (VEC && N == 2) {
            *reinterpret_cast<uint32_t *>(p) = pack_bf16x2(v[0], v[1]);
        } else {
#pragma unroll
            for (int k = 0; k < N; ++k)
                p[k] = __float2bfloat16_rn(v[k]);
        }
    }
};

} // namespace tok
