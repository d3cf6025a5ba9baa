// FSQ backward for sm_100a: the straight-through gradient of the fused encode and
// the gradient of the fused decode.
//
// Source: "NVIDIA Cosmos Tokenizer 完全指南", section 7.2: the bound uses tanh and
// round_ste keeps a straight-through gradient, i.e. the rounding passes the
// gradient unchanged, so with the bound of the published FSQ method
//   d zhat_i / d z_i = half_i * sech^2(z_i + shift_i) / floor(L_i / 2).
// Encode backward, per token (z the same fp32 chain as the forward):
//   t_i = g_i * slope_i(z_i);  grad_u[c] = sum_i w[i][c] t_i;  grad_w[i][c] = sum_tokens t_i u_c.
// Decode backward, per token (zhat from the index; invalid indices count as zero):
//   grad_codes_i = sum_c w[i][c] g_c;  grad_w[i][c] = sum_tokens zhat_i g_c.
//
// sech^2(x) is evaluated as 4a / (1 + a)^2 with a = exp(-2|x|) = 2^(-2 log2(e) |x|):
// accurate where tanh saturates, unlike 1 - tanh^2.  Both paths round the same
// sequence of fp32 operations, so they give the same t bit for bit.
//
// Reduction of grad_w: tokens are cut into fixed blocks of kTokensPerCta (the
// partition does not depend on the device), each thread accumulates its tokens
// in registers in order, a shuffle tree and shared memory reduce a CTA's
// threads in a fixed order into one row of the caller's workspace
// [blocks][6C], and a second kernel sums the rows in double in a fixed order
// (strided per thread, then a pairwise tree).  The result is therefore the same
// on every run and every B200.
//
// Memory: encode backward reads u (4C B), g (24 B) and writes grad_u (4C B)
// per token; decode backward reads the index (4 B) and g (4C B) and writes
// grad_codes (24 B).  Both are HBM-bound.
//
// Main path (C = 16, S % 4 == 0, 16-byte-aligned tensors): single-warp CTAs,
// each owning a fixed run of kTilesPerRow = 8 tiles of 128 tokens (tile order:
// batch row, then position).  A two-stage ring of TMA loads brings a tile's
// inputs into shared memory while the previous tile is computed; each lane owns
// 4 consecutive tokens, reads them with 16-byte shared loads, computes with
// packed f32x2 operations and writes with 16-byte global stores.  The grad_w
// accumulators stay in registers across the CTA's tiles and are reduced by a
// shuffle butterfly into the CTA's workspace row.  Other shapes take the
// register kernels (2048 tokens per CTA, 128 threads).
//
// The workspace holds one row of 6C sums per CTA, partial[row * 6C + k] with
// k = i*C + c (a CTA writes its row as a contiguous block, the cheapest pattern
// for the row kernel).  The summing kernel (one CTA per entry) is launched as a
// programmatic dependent of the row kernel, so its launch is prepared while the
// row kernel runs; it waits for the row kernel's completion before reading.
// (Measured: letting the row kernel release it early, a grouped summing kernel
// with 16-byte loads, and entry-major or sector-grouped workspace layouts were
// all slower.)
#include <cmath>
#include <cstring>
#include <mutex>

#include "tma.cuh"
#include "tok_common.cuh"
#include "tok_internal.h"

namespace tok {
namespace {

constexpr int kThreads = 128;
constexpr int kTokensPerCta = 2048; // 16 tokens per thread
constexpr int kMaxC = 16;           // channel count held in registers

// Main path: tiles of 128 tokens, kTilesPerRow tiles per CTA (one workspace row).
constexpr int kTileTokens = 128;
constexpr int kTilesPerRow = 8;
constexpr int kStages = 2;

// Barrier waits that ran out in this file's kernels (read by tok_check_device).
static __device__ unsigned int g_bwd_wait_timeouts;

struct SlopeConsts {
    float shift[6];  // atanh(off / half)
    float scale4[6]; // 4 * half / floor(L / 2)
};

SlopeConsts slope_consts()
{
    static const int L[6] = {8, 8, 8, 5, 5, 5};
    SlopeConsts k{};
    for (int i = 0; i < 6; ++i) {
        const double half = (L[i] - 1) * (1.0 + 1e-3) / 2.0;
        const double off = (L[i] % 2 == 0) ? 0.5 : 0.0;
        k.shift[i] = (float)std::atanh(off / half);
        k.scale4[i] = (float)(4.0 * half / (double)(L[i] / 2));
    }
    return k;
}

// 2^x and 1/x from the hardware approximations (relative error about 2^-22).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp_approx(float x)
{
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

constexpr float kMinus2Log2e = -2.88539008f; // -2 log2(e): e^{-2|x|} = 2^(kMinus2Log2e |x|)

// t = g * slope(z) with slope = scale4 * a / (1 + a)^2, a = e^{-2|z + shift|} in (0, 1]:
// the denominator lies in [1, 4], so the approximate reciprocal is accurate there; the
// rounding of the exponent's argument costs about |x| * 2^-24 relative, which matters
// only where the slope itself is negligible.  Relative accuracy about 1e-6.
__device__ __forceinline__ float ste_grad(float z, float g, float shift, float scale4)
{
    const float x = z + shift;
    const float a = ex2_approx(kMinus2Log2e * fabsf(x));
    const float d = a + 1.0f;
    const float r = rcp_approx(d * d);
    return g * ((a * r) * scale4);
}

// The same for two tokens, in packed f32x2 operations with the same roundings.
__device__ __forceinline__ float2 ste_grad2(float2 z, float2 g, float2 shift, float2 scale4)
{
    const float2 x = __fadd2_rn(z, shift);
    const float2 a = make_float2(ex2_approx(kMinus2Log2e * fabsf(x.x)), ex2_approx(kMinus2Log2e * fabsf(x.y)));
    const float2 d = __fadd2_rn(a, make_float2(1.0f, 1.0f));
    const float2 dd = __fmul2_rn(d, d);
    const float2 r = make_float2(rcp_approx(dd.x), rcp_approx(dd.y));
    return __fmul2_rn(g, __fmul2_rn(__fmul2_rn(a, r), scale4));
}

// Reduces the per-thread accumulators acc[i * kMaxC + c] over the CTA in a fixed
// order and writes the CTA's row of 6*C sums, partial[row * 6C + i * C + c].  All indices into
// acc are compile-time constants, so it stays in registers.
__device__ __forceinline__ void reduce_rows(const float (&acc)[6 * kMaxC], int C, float *red, float *partial)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int q = 0; q < 6 * kMaxC; ++q) {
        const int i = q / kMaxC, c = q % kMaxC;
        if (c >= C)
            continue;
        float v = acc[q];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
            v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
        if (lane == 0)
            red[warp * 6 * kMaxC + i * C + c] = v;
    }
    __syncthreads();
    for (int k = threadIdx.x; k < 6 * C; k += kThreads) {
        float s = 0.0f;
        for (int w = 0; w < kThreads / 32; ++w)
            s += red[w * 6 * kMaxC + k];
        partial[(int64_t)blockIdx.x * 6 * C + k] = s;
    }
}

__global__ void __launch_bounds__(kThreads)
    fsq_encode_bwd_kernel(const float *__restrict__ u, const float *__restrict__ w, const float *__restrict__ g,
                          float *__restrict__ gu, float *__restrict__ partial, int64_t B, int C, int64_t S,
                          SlopeConsts k)
{
    __shared__ float ws[6 * kMaxC];
    __shared__ float red[(kThreads / 32) * 6 * kMaxC];
    for (int i = threadIdx.x; i < 6 * C; i += kThreads)
        ws[i] = w[i];
    __syncthreads();

    float acc[6 * kMaxC];
#pragma unroll
    for (int q = 0; q < 6 * kMaxC; ++q)
        acc[q] = 0.0f;
    const int64_t N = B * S, n0 = (int64_t)blockIdx.x * kTokensPerCta;
    for (int j = 0; j < kTokensPerCta / kThreads; ++j) {
        const int64_t n = n0 + (int64_t)j * kThreads + threadIdx.x;
        if (n >= N)
            break;
        const int64_t b = n / S, s = n - b * S;
        const float *ub = u + b * C * S + s;
        float uc[kMaxC];
#pragma unroll
        for (int c = 0; c < kMaxC; ++c)
            uc[c] = c < C ? ub[(int64_t)c * S] : 0.0f;
        float t[6];
#pragma unroll
        for (int i = 0; i < 6; ++i) {
            float z = 0.0f;
#pragma unroll
            for (int c = 0; c < kMaxC; ++c)
                if (c < C)
                    z = fmaf(ws[i * C + c], uc[c], z);
            t[i] = ste_grad(z, g[(b * 6 + i) * S + s], k.shift[i], k.scale4[i]);
        }
#pragma unroll
        for (int c = 0; c < kMaxC; ++c) {
            if (c >= C)
                break;
            float acc_u = 0.0f;
#pragma unroll
            for (int i = 0; i < 6; ++i) {
                acc_u = fmaf(ws[i * C + c], t[i], acc_u);
                acc[i * kMaxC + c] = fmaf(t[i], uc[c], acc[i * kMaxC + c]);
            }
            gu[(b * C + c) * S + s] = acc_u;
        }
    }
    reduce_rows(acc, C, red, partial);
}

__global__ void __launch_bounds__(kThreads)
    fsq_decode_bwd_kernel(const int32_t *__restrict__ idx, const float *__restrict__ w, const float *__restrict__ g,
                          float *__restrict__ gcodes, float *__restrict__ partial, int64_t B, int C, int64_t S)
{
    __shared__ float ws[6 * kMaxC];
    __shared__ float red[(kThreads / 32) * 6 * kMaxC];
    for (int i = threadIdx.x; i < 6 * C; i += kThreads)
        ws[i] = w[i];
    __syncthreads();

    float acc[6 * kMaxC];
#pragma unroll
    for (int q = 0; q < 6 * kMaxC; ++q)
        acc[q] = 0.0f;
    const int64_t N = B * S, n0 = (int64_t)blockIdx.x * kTokensPerCta;
    for (int j = 0; j < kTokensPerCta / kThreads; ++j) {
        const int64_t n = n0 + (int64_t)j * kThreads + threadIdx.x;
        if (n >= N)
            break;
        const int64_t b = n / S, s = n - b * S;
        const int32_t id = idx[n];
        const bool valid = (uint32_t)id < (uint32_t)TOK_FSQ_CODEBOOK;
        uint32_t r = valid ? (uint32_t)id : 0u;
        int d[6];
        d[0] = r % 8u; r /= 8u;
        d[1] = r % 8u; r /= 8u;
        d[2] = r % 8u; r /= 8u;
        d[3] = r % 5u; r /= 5u;
        d[4] = r % 5u; r /= 5u;
        d[5] = (int)r;
        float zh[6];
#pragma unroll
        for (int i = 0; i < 6; ++i) {
            const int hw = i < 3 ? 4 : 2;
            zh[i] = valid ? (float)(d[i] - hw) * (i < 3 ? 0.25f : 0.5f) : 0.0f;
        }
        const float *gb = g + b * C * S + s;
        float gc[kMaxC];
#pragma unroll
        for (int c = 0; c < kMaxC; ++c)
            gc[c] = c < C ? gb[(int64_t)c * S] : 0.0f;
#pragma unroll
        for (int i = 0; i < 6; ++i) {
            float a = 0.0f;
#pragma unroll
            for (int c = 0; c < kMaxC; ++c)
                if (c < C) {
                    a = fmaf(ws[i * C + c], gc[c], a);
                    acc[i * kMaxC + c] = fmaf(zh[i], gc[c], acc[i * kMaxC + c]);
                }
            gcodes[(b * 6 + i) * S + s] = valid ? a : 0.0f;
        }
    }
    reduce_rows(acc, C, red, partial);
}

// grad_w[k] = sum over the rows of partial, in double, in a fixed order: one CTA
// per entry k; thread t sums rows t, t + 512, ... in order, each warp then sums its
// 32 threads by a shuffle butterfly, and one warp sums the 16 warp totals the same
// way.  Launched as a programmatic dependent of the row kernel: it waits for that
// grid's completion (and the visibility of its writes) before it reads.
constexpr int kSumThreads = 512;

__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    return v;
}

__global__ void __launch_bounds__(kSumThreads)
    fsq_bwd_sum_rows_kernel(const float *__restrict__ partial, int64_t rows, int K, float *__restrict__ out)
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    __shared__ double warps[kSumThreads / 32];
    const int t = threadIdx.x, k = blockIdx.x;
    double s = 0.0;
#pragma unroll 8
    for (int64_t r = t; r < rows; r += kSumThreads)
        s += (double)partial[r * K + k];
    s = warp_sum(s);
    if ((t & 31) == 0)
        warps[t >> 5] = s;
    __syncthreads();
    if (t < 32) {
        double v = t < kSumThreads / 32 ? warps[t] : 0.0;
        v = warp_sum(v);
        if (t == 0)
            out[k] = (float)v;
    }
}

// Launches the sum of `rows` rows of K entries into out[K] on `stream` as a
// programmatic dependent of the preceding kernel.
cudaError_t launch_sum_rows(const float *partial, int64_t rows, int K, float *out, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)K);
    cfg.blockDim = dim3(kSumThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fsq_bwd_sum_rows_kernel, partial, rows, K, out);
}

// ---------------------------------------------------------------------------
// Main path.
// ---------------------------------------------------------------------------

// grad_w on the main path.  A pair of lanes (2p, 2p + 1) covers the pair's 8 tokens
// 8p .. 8p + 7 of the tile; lane 2p + h accumulates the channels c = 8h .. 8h + 7, so
// a lane holds 48 sums, as f32x2 pairs acc2[ip][cc] = (acc[2ip][8h + cc], acc[2ip + 1][8h + cc]).
constexpr int kHalfC = 8;

// Sums acc2 over the 16 lanes of the same half (xor butterfly over lane bits 1..4:
// every lane ends with the same sums in the same order) and writes entry
// k = i * 16 + 8h + cc of this CTA's row to partial[row * 96 + k], three per lane.
__device__ __forceinline__ void warp_row_half(const float2 (&acc2)[3][kHalfC], float *partial)
{
    const int lane = threadIdx.x & 31, h = lane & 1;
#pragma unroll
    for (int q = 0; q < 6 * kHalfC; ++q) {
        const int i = q / kHalfC, cc = q % kHalfC;
        float v = (i & 1) ? acc2[i >> 1][cc].y : acc2[i >> 1][cc].x;
#pragma unroll
        for (int off = 16; off > 1; off >>= 1)
            v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
        if ((q & 15) == (lane >> 1))
            partial[(int64_t)blockIdx.x * 6 * kMaxC + i * 16 + kHalfC * h + cc] = v;
    }
}

// Shared tables after the stages: the weights with each entry twice,
// wd[c * 12 + 2i + e] = w[i][c] (e = 0, 1), so three 16-byte loads give a channel's six
// weights as (w, w) pairs for the packed FMAs; then kd[i] = (shift, shift, scale4, scale4).
constexpr int kTableBytes = 16 * 12 * 4 + 6 * 16;

__device__ __forceinline__ void stage_weights(const float *__restrict__ w, float *wd)
{
    for (int q = threadIdx.x; q < 16 * 12; q += 32) {
        const int c = q / 12, i = (q % 12) >> 1;
        wd[q] = w[i * 16 + c];
    }
}

__device__ __forceinline__ void stage_slopes(const SlopeConsts &k, float *wd)
{
    float4 *kd = reinterpret_cast<float4 *>(wd + 16 * 12);
#pragma unroll
    for (int i = 0; i < 6; ++i) // constant indices keep the parameter in the constant bank
        if (threadIdx.x == i)
            kd[i] = make_float4(k.shift[i], k.shift[i], k.scale4[i], k.scale4[i]);
}

__device__ __forceinline__ void wpairs_of(const float *wd, int c, float2 (&wp)[6])
{
    const float4 a = *reinterpret_cast<const float4 *>(wd + c * 12);
    const float4 b = *reinterpret_cast<const float4 *>(wd + c * 12 + 4);
    const float4 e = *reinterpret_cast<const float4 *>(wd + c * 12 + 8);
    wp[0] = make_float2(a.x, a.y), wp[1] = make_float2(a.z, a.w), wp[2] = make_float2(b.x, b.y);
    wp[3] = make_float2(b.z, b.w), wp[4] = make_float2(e.x, e.y), wp[5] = make_float2(e.z, e.w);
}

// Normalized codes of an index as channel pairs (zh0, zh1), (zh2, zh3), (zh4, zh5);
// an invalid index gives zeros.
__device__ __forceinline__ void zhat_pairs(int32_t id, float2 (&zp)[3])
{
    const bool valid = (uint32_t)id < (uint32_t)TOK_FSQ_CODEBOOK;
    uint32_t r = valid ? (uint32_t)id : 0u;
    const int d0 = r % 8u; r /= 8u;
    const int d1 = r % 8u; r /= 8u;
    const int d2 = r % 8u; r /= 8u;
    const int d3 = r % 5u; r /= 5u;
    const int d4 = r % 5u; r /= 5u;
    const int d5 = (int)r;
    const float v = valid ? 1.0f : 0.0f;
    zp[0] = make_float2(v * ((float)(d0 - 4) * 0.25f), v * ((float)(d1 - 4) * 0.25f));
    zp[1] = make_float2(v * ((float)(d2 - 4) * 0.25f), v * ((float)(d3 - 2) * 0.5f));
    zp[2] = make_float2(v * ((float)(d4 - 2) * 0.5f), v * ((float)(d5 - 2) * 0.5f));
}

// Ring bookkeeping shared by both kernels: tile j of the CTA sits in stage j % STAGES
// and completes phase (j / STAGES) & 1 of that stage's barrier.
template <int STAGES> __device__ __forceinline__ uint32_t ring_parity(int j) { return (uint32_t)((j / STAGES) & 1); }

// After a wait ran out at tile j: let the loads still in flight land (each wait bounded
// again) so that no copy targets shared memory of an exited CTA, then count it.
template <int STAGES>
__device__ __forceinline__ void ring_drain(const uint64_t *bars, int j, int count)
{
    if ((threadIdx.x & 31) == 0) {
        for (int r = j; r < count && r < j + STAGES; ++r)
            mbar_wait(smem_addr(bars + r % STAGES), ring_parity<STAGES>(r));
        atomicAdd(&g_bwd_wait_timeouts, 1u);
    }
    __syncwarp();
}

// Encode backward, C = 16.  Stage layout: u tile [16][128] then g tile [6][128] (fp32).
// Once every lane has read its g, each lane writes t = g * slope(z) of its four tokens
// over the g tile as channel pairs, tp[ip][m] = (t[2ip][m], t[2ip + 1][m]), which the
// lane pair then reads back for grad_w.
template <int TPR, int STAGES>
__global__ void __launch_bounds__(32)
    fsq_encode_bwd_tma_kernel(const __grid_constant__ CUtensorMap umap, const __grid_constant__ CUtensorMap gmap,
                              const float *__restrict__ w, float *__restrict__ gu, float *__restrict__ partial,
                              int64_t S, FastDiv ntx, uint32_t ntiles, SlopeConsts k)
{
    constexpr int U_BYTES = 16 * kTileTokens * 4, STAGE = U_BYTES + 6 * kTileTokens * 4;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + STAGES * STAGE);
    float *wd = reinterpret_cast<float *>(smem_raw + STAGES * STAGE + 16 * STAGES); // 16-byte aligned
    const float4 *kd = reinterpret_cast<const float4 *>(wd + 16 * 12);
    const int lane = threadIdx.x, h = lane & 1;
    const uint32_t first = blockIdx.x * (uint32_t)TPR;
    const int count = (int)min((uint32_t)TPR, ntiles - first);

    auto issue = [&](int j) {
        const uint32_t n = first + j, b = ntx.div(n), tx = n - b * ntx.d;
        const uint32_t bar = smem_addr(bars + j % STAGES), dst = smem_addr(smem_raw + (j % STAGES) * STAGE);
        mbar_expect_tx(bar, STAGE);
        tma_load_3d(dst, &umap, (int)(tx * kTileTokens), 0, (int)b, bar);
        tma_load_3d(dst + U_BYTES, &gmap, (int)(tx * kTileTokens), 0, (int)b, bar);
    };
    if (lane == 0) {
        for (int s = 0; s < STAGES; ++s)
            mbar_init(smem_addr(bars + s), 1);
        fence_barrier_init();
        for (int j = 0; j < count && j < STAGES; ++j)
            issue(j);
    }
    stage_weights(w, wd);
    stage_slopes(k, wd);
    __syncwarp();

    float2 acc2[3][kHalfC];
#pragma unroll
    for (int ip = 0; ip < 3; ++ip)
#pragma unroll
        for (int cc = 0; cc < kHalfC; ++cc)
            acc2[ip][cc] = make_float2(0.0f, 0.0f);

    int j = 0;
    for (; j < count; ++j) {
        const bool ok = mbar_wait(smem_addr(bars + j % STAGES), ring_parity<STAGES>(j));
        if (__any_sync(0xFFFFFFFFu, !ok))
            break;
        const uint32_t n = first + j, b = ntx.div(n), tx = n - b * ntx.d;
        const float *tu = reinterpret_cast<const float *>(smem_raw + (j % STAGES) * STAGE);
        float *tg = reinterpret_cast<float *>(smem_raw + (j % STAGES) * STAGE + U_BYTES);

        {
            // z_i of the lane's tokens (0,1) and (2,3): the fp32 chain over c from 0.
            float2 z[6][2];
#pragma unroll
            for (int i = 0; i < 6; ++i)
                z[i][0] = z[i][1] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float4 q = *reinterpret_cast<const float4 *>(tu + c * kTileTokens + 4 * lane);
                float2 wp[6];
                wpairs_of(wd, c, wp);
#pragma unroll
                for (int i = 0; i < 6; ++i) {
                    z[i][0] = __ffma2_rn(wp[i], make_float2(q.x, q.y), z[i][0]);
                    z[i][1] = __ffma2_rn(wp[i], make_float2(q.z, q.w), z[i][1]);
                }
            }
            // t_i = g_i * slope_i(z_i).
            float2 t2[6][2];
#pragma unroll
            for (int i = 0; i < 6; ++i) {
                const float4 gq = *reinterpret_cast<const float4 *>(tg + i * kTileTokens + 4 * lane);
                const float4 kq = kd[i];
                const float2 shift = make_float2(kq.x, kq.y), scale4 = make_float2(kq.z, kq.w);
                t2[i][0] = ste_grad2(z[i][0], make_float2(gq.x, gq.y), shift, scale4);
                t2[i][1] = ste_grad2(z[i][1], make_float2(gq.z, gq.w), shift, scale4);
            }
            __syncwarp(); // every lane has read its g: the tile may now hold t
#pragma unroll
            for (int ip = 0; ip < 3; ++ip) {
                float4 *dst = reinterpret_cast<float4 *>(tg + (ip * kTileTokens + 4 * lane) * 2);
                dst[0] = make_float4(t2[2 * ip][0].x, t2[2 * ip + 1][0].x, t2[2 * ip][0].y, t2[2 * ip + 1][0].y);
                dst[1] = make_float4(t2[2 * ip][1].x, t2[2 * ip + 1][1].x, t2[2 * ip][1].y, t2[2 * ip + 1][1].y);
            }
            // grad_u = sum_i w[i][c] t_i, the chain over i from 0, for the lane's tokens.
            const int64_t t0 = (int64_t)tx * kTileTokens + 4 * lane;
            if (t0 < S) { // S % 4 == 0: a lane's four tokens are all in range or all out
                float *gub = gu + (int64_t)b * 16 * S + t0;
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    float2 wp[6];
                    wpairs_of(wd, c, wp);
                    float2 o0 = make_float2(0.0f, 0.0f), o1 = o0;
#pragma unroll
                    for (int i = 0; i < 6; ++i) {
                        o0 = __ffma2_rn(wp[i], t2[i][0], o0);
                        o1 = __ffma2_rn(wp[i], t2[i][1], o1);
                    }
                    *reinterpret_cast<float4 *>(gub) = make_float4(o0.x, o0.y, o1.x, o1.y);
                    gub += S;
                }
            }
        }
        __syncwarp(); // t of the partner lane is in shared memory
        // grad_w: the pair's 8 tokens in increasing order, channels 8h .. 8h + 7.
#pragma unroll
        for (int g2 = 0; g2 < 2; ++g2) {
            const int col = 4 * ((lane & ~1) + g2);
            float2 tp[3][4];
#pragma unroll
            for (int ip = 0; ip < 3; ++ip) {
                const float4 *src = reinterpret_cast<const float4 *>(tg + (ip * kTileTokens + col) * 2);
                const float4 a = src[0], e = src[1];
                tp[ip][0] = make_float2(a.x, a.y), tp[ip][1] = make_float2(a.z, a.w);
                tp[ip][2] = make_float2(e.x, e.y), tp[ip][3] = make_float2(e.z, e.w);
            }
#pragma unroll
            for (int cc = 0; cc < kHalfC; ++cc) {
                const float4 q = *reinterpret_cast<const float4 *>(tu + (kHalfC * h + cc) * kTileTokens + col);
                const float uq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float2 ub = make_float2(uq[m], uq[m]);
#pragma unroll
                    for (int ip = 0; ip < 3; ++ip)
                        acc2[ip][cc] = __ffma2_rn(tp[ip][m], ub, acc2[ip][cc]);
                }
            }
        }
        __syncwarp(); // every lane has read this stage
        if (lane == 0 && j + STAGES < count) {
            fence_proxy_async_smem();
            issue(j + STAGES);
        }
    }
    if (j < count)
        ring_drain<STAGES>(bars, j, count);
    warp_row_half(acc2, partial);
}

// Decode backward, C = 16.  Stage layout: g tile [16][128] (fp32) then the 128 indices.
template <int TPR, int STAGES>
__global__ void __launch_bounds__(32)
    fsq_decode_bwd_tma_kernel(const __grid_constant__ CUtensorMap gmap, const __grid_constant__ CUtensorMap imap,
                              const float *__restrict__ w, float *__restrict__ gcodes, float *__restrict__ partial,
                              int64_t S, FastDiv ntx, uint32_t ntiles)
{
    constexpr int G_BYTES = 16 * kTileTokens * 4, STAGE = G_BYTES + kTileTokens * 4;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + STAGES * STAGE);
    float *wd = reinterpret_cast<float *>(smem_raw + STAGES * STAGE + 16 * STAGES); // 16-byte aligned
    const int lane = threadIdx.x, h = lane & 1;
    const uint32_t first = blockIdx.x * (uint32_t)TPR;
    const int count = (int)min((uint32_t)TPR, ntiles - first);

    auto issue = [&](int j) {
        const uint32_t n = first + j, b = ntx.div(n), tx = n - b * ntx.d;
        const uint32_t bar = smem_addr(bars + j % STAGES), dst = smem_addr(smem_raw + (j % STAGES) * STAGE);
        mbar_expect_tx(bar, STAGE);
        tma_load_3d(dst, &gmap, (int)(tx * kTileTokens), 0, (int)b, bar);
        tma_load_2d(dst + G_BYTES, &imap, (int)(tx * kTileTokens), (int)b, bar);
    };
    if (lane == 0) {
        for (int s = 0; s < STAGES; ++s)
            mbar_init(smem_addr(bars + s), 1);
        fence_barrier_init();
        for (int j = 0; j < count && j < STAGES; ++j)
            issue(j);
    }
    stage_weights(w, wd);
    __syncwarp();

    float2 acc2[3][kHalfC];
#pragma unroll
    for (int ip = 0; ip < 3; ++ip)
#pragma unroll
        for (int cc = 0; cc < kHalfC; ++cc)
            acc2[ip][cc] = make_float2(0.0f, 0.0f);

    int j = 0;
    for (; j < count; ++j) {
        const bool ok = mbar_wait(smem_addr(bars + j % STAGES), ring_parity<STAGES>(j));
        if (__any_sync(0xFFFFFFFFu, !ok))
            break;
        const uint32_t n = first + j, b = ntx.div(n), tx = n - b * ntx.d;
        const float *tgl = reinterpret_cast<const float *>(smem_raw + (j % STAGES) * STAGE);
        const int32_t *tid = reinterpret_cast<const int32_t *>(smem_raw + (j % STAGES) * STAGE + G_BYTES);

        // grad_codes = sum_c w[i][c] g_c, the chain over c from 0, for the lane's tokens.
        const int64_t t0 = (int64_t)tx * kTileTokens + 4 * lane;
        if (t0 < S) {
            const int4 iq = *reinterpret_cast<const int4 *>(tid + 4 * lane);
            const bool v0 = (uint32_t)iq.x < (uint32_t)TOK_FSQ_CODEBOOK, v1 = (uint32_t)iq.y < (uint32_t)TOK_FSQ_CODEBOOK;
            const bool v2 = (uint32_t)iq.z < (uint32_t)TOK_FSQ_CODEBOOK, v3 = (uint32_t)iq.w < (uint32_t)TOK_FSQ_CODEBOOK;
            float2 gc2[6][2];
#pragma unroll
            for (int i = 0; i < 6; ++i)
                gc2[i][0] = gc2[i][1] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float4 q = *reinterpret_cast<const float4 *>(tgl + c * kTileTokens + 4 * lane);
                float2 wp[6];
                wpairs_of(wd, c, wp);
#pragma unroll
                for (int i = 0; i < 6; ++i) {
                    gc2[i][0] = __ffma2_rn(wp[i], make_float2(q.x, q.y), gc2[i][0]);
                    gc2[i][1] = __ffma2_rn(wp[i], make_float2(q.z, q.w), gc2[i][1]);
                }
            }
            float *gcb = gcodes + (int64_t)b * 6 * S + t0;
#pragma unroll
            for (int i = 0; i < 6; ++i)
                *reinterpret_cast<float4 *>(gcb + (int64_t)i * S) =
                    make_float4(v0 ? gc2[i][0].x : 0.0f, v1 ? gc2[i][0].y : 0.0f, v2 ? gc2[i][1].x : 0.0f,
                                v3 ? gc2[i][1].y : 0.0f);
        }
        // grad_w: the pair's 8 tokens in increasing order, channels 8h .. 8h + 7.
#pragma unroll
        for (int g2 = 0; g2 < 2; ++g2) {
            const int col = 4 * ((lane & ~1) + g2);
            const int4 iq = *reinterpret_cast<const int4 *>(tid + col);
            float2 zp[4][3];
            zhat_pairs(iq.x, zp[0]);
            zhat_pairs(iq.y, zp[1]);
            zhat_pairs(iq.z, zp[2]);
            zhat_pairs(iq.w, zp[3]);
#pragma unroll
            for (int cc = 0; cc < kHalfC; ++cc) {
                const float4 q = *reinterpret_cast<const float4 *>(tgl + (kHalfC * h + cc) * kTileTokens + col);
                const float gq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float2 gb = make_float2(gq[m], gq[m]);
#pragma unroll
                    for (int ip = 0; ip < 3; ++ip)
                        acc2[ip][cc] = __ffma2_rn(zp[m][ip], gb, acc2[ip][cc]);
                }
            }
        }
        __syncwarp(); // every lane has read this stage
        if (lane == 0 && j + STAGES < count) {
            fence_proxy_async_smem();
            issue(j + STAGES);
        }
    }
    if (j < count)
        ring_drain<STAGES>(bars, j, count);
    warp_row_half(acc2, partial);
}

// Shared memory: the stages (multiples of 128 bytes), one 16-byte slot per stage for
// its barrier, then the tables.
template <int STAGES> constexpr int enc_smem() { return STAGES * (22 * kTileTokens * 4 + 16) + kTableBytes; }
template <int STAGES> constexpr int dec_smem() { return STAGES * (17 * kTileTokens * 4 + 16) + kTableBytes; }

// Tiles of the main path: B * ceil(S / 128).
int64_t tma_tiles(int64_t B, int64_t S) { return B * ((S + kTileTokens - 1) / kTileTokens); }

// The main path takes C = 16 with S % 4 == 0 (TMA needs rows of a multiple of 16
// bytes) and 16-byte-aligned tensors.
bool bwd_tma_eligible(int64_t B, int64_t C, int64_t S, const void *a, const void *b, const void *c)
{
    return C == 16 && S % 4 == 0 && S < ((int64_t)1 << 31) && B < ((int64_t)1 << 31) &&
           tma_tiles(B, S) < ((int64_t)1 << 31) && aligned(a, 16) && aligned(b, 16) && aligned(c, 16) &&
           sm_count() > 0;
}

// Launches the main-path encode backward; false if a tensor map was refused (then
// nothing ran and the register kernel is used).
template <int TPR, int STAGES>
bool launch_encode_bwd_tma(const float *u, const float *w, const float *g, float *gu, float *partial, int64_t B,
                           int64_t S, cudaStream_t stream, tok_status *st)
{
    CUtensorMap umap, gmap;
    memset(&umap, 0, sizeof umap);
    memset(&gmap, 0, sizeof gmap);
    const uint64_t udims[3] = {(uint64_t)S, 16, (uint64_t)B}, ustr[2] = {(uint64_t)S * 4, (uint64_t)S * 64};
    const uint64_t gdims[3] = {(uint64_t)S, 6, (uint64_t)B}, gstr[2] = {(uint64_t)S * 4, (uint64_t)S * 24};
    const uint32_t ubox[3] = {(uint32_t)kTileTokens, 16, 1}, gbox[3] = {(uint32_t)kTileTokens, 6, 1};
    if (!encode_tensor_map(&umap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, u, udims, ustr, ubox) ||
        !encode_tensor_map(&gmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, g, gdims, gstr, gbox))
        return false;
    auto kern = fsq_encode_bwd_tma_kernel<TPR, STAGES>;
    constexpr int smem = enc_smem<STAGES>();
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        *st = TOK_ERR_CUDA;
        return true;
    }
    const int64_t ntx = (S + kTileTokens - 1) / kTileTokens, ntiles = ntx * B;
    const unsigned grid = (unsigned)((ntiles + TPR - 1) / TPR);
    kern<<<grid, 32, smem, stream>>>(umap, gmap, w, gu, partial, S, FastDiv((uint32_t)ntx), (uint32_t)ntiles,
                                     slope_consts());
    *st = launch_status();
    return true;
}

template <int TPR, int STAGES>
bool launch_decode_bwd_tma(const int32_t *idx, const float *w, const float *g, float *gcodes, float *partial,
                           int64_t B, int64_t S, cudaStream_t stream, tok_status *st)
{
    CUtensorMap gmap, imap;
    memset(&gmap, 0, sizeof gmap);
    memset(&imap, 0, sizeof imap);
    const uint64_t gdims[3] = {(uint64_t)S, 16, (uint64_t)B}, gstr[2] = {(uint64_t)S * 4, (uint64_t)S * 64};
    const uint64_t idims[2] = {(uint64_t)S, (uint64_t)B}, istr[1] = {(uint64_t)S * 4};
    const uint32_t gbox[3] = {(uint32_t)kTileTokens, 16, 1}, ibox[2] = {(uint32_t)kTileTokens, 1};
    if (!encode_tensor_map(&gmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, g, gdims, gstr, gbox) ||
        !encode_tensor_map(&imap, CU_TENSOR_MAP_DATA_TYPE_INT32, 2, idx, idims, istr, ibox))
        return false;
    auto kern = fsq_decode_bwd_tma_kernel<TPR, STAGES>;
    constexpr int smem = dec_smem<STAGES>();
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        *st = TOK_ERR_CUDA;
        return true;
    }
    const int64_t ntx = (S + kTileTokens - 1) / kTileTokens, ntiles = ntx * B;
    const unsigned grid = (unsigned)((ntiles + TPR - 1) / TPR);
    kern<<<grid, 32, smem, stream>>>(gmap, imap, w, gcodes, partial, S, FastDiv((uint32_t)ntx), (uint32_t)ntiles);
    *st = launch_status();
    return true;
}

bool shape_ok(int64_t B, int64_t C, int64_t S, int64_t *N)
{
    int64_t bytes;
    return B >= 0 && S >= 0 && C >= 1 && C <= kMaxC && prod_ok({B, S}, N) && prod_ok({*N, C, 4}, &bytes);
}

int64_t blocks_for(int64_t N) { return (N + kTokensPerCta - 1) / kTokensPerCta; }

// Workspace rows of either path: the register kernels write one row per 2048 tokens,
// the main path one row per kTilesPerRow tiles.
int64_t workspace_rows(int64_t B, int64_t S, int64_t N)
{
    const int64_t rows_reg = blocks_for(N), rows_tma = (tma_tiles(B, S) + kTilesPerRow - 1) / kTilesPerRow;
    return rows_reg > rows_tma ? rows_reg : rows_tma;
}

} // namespace

int64_t fsq_backward_workspace_bytes(int64_t B, int64_t C, int64_t S)
{
    int64_t N;
    if (!shape_ok(B, C, S, &N))
        return -1;
    return workspace_rows(B, S, N) * 6 * C * (int64_t)sizeof(float);
}

tok_status read_and_clear_fsq_bwd_timeouts(cudaStream_t stream, unsigned int *count)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(count, g_bwd_wait_timeouts, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && *count)
        e = cudaMemcpyToSymbolAsync(g_bwd_wait_timeouts, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice,
                                    stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return TOK_ERR_CUDA;
    }
    return TOK_OK;
}

// Encode backward on whichever path suits the call; the workspace holds
// fsq_backward_workspace_bytes(B, C, S).
tok_status encode_bwd_run(const float *u, const float *w, const float *g, float *gu, float *gw, float *partial,
                          int64_t B, int64_t C, int64_t S, int64_t N, cudaStream_t stream)
{
    int64_t rows = blocks_for(N);
    tok_status st = TOK_OK;
    bool done = false;
    if (N > 0 && bwd_tma_eligible(B, C, S, u, g, gu)) {
        done = launch_encode_bwd_tma<kTilesPerRow, kStages>(u, w, g, gu, partial, B, S, stream, &st);
        if (done)
            rows = (tma_tiles(B, S) + kTilesPerRow - 1) / kTilesPerRow;
        if (st != TOK_OK)
            return st;
    }
    if (!done && rows > 0)
        fsq_encode_bwd_kernel<<<(unsigned)rows, kThreads, 0, stream>>>(u, w, g, gu, partial, B, (int)C, S,
                                                                       slope_consts());
    const cudaError_t e = launch_sum_rows(partial, rows, (int)(6 * C), gw, stream);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return TOK_ERR_CUDA;
    }
    return launch_status();
}

tok_status decode_bwd_run(const int32_t *idx, const float *w, const float *g, float *gc, float *gw, float *partial,
                          int64_t B, int64_t C, int64_t S, int64_t N, cudaStream_t stream)
{
    int64_t rows = blocks_for(N);
    tok_status st = TOK_OK;
    bool done = false;
    if (N > 0 && bwd_tma_eligible(B, C, S, idx, g, gc)) {
        done = launch_decode_bwd_tma<kTilesPerRow, kStages>(idx, w, g, gc, partial, B, S, stream, &st);
        if (done)
            rows = (tma_tiles(B, S) + kTilesPerRow - 1) / kTilesPerRow;
        if (st != TOK_OK)
            return st;
    }
    if (!done && rows > 0)
        fsq_decode_bwd_kernel<<<(unsigned)rows, kThreads, 0, stream>>>(idx, w, g, gc, partial, B, (int)C, S);
    const cudaError_t e = launch_sum_rows(partial, rows, (int)(6 * C), gw, stream);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return TOK_ERR_CUDA;
    }
    return launch_status();
}

} // namespace tok

// ---------------------------------------------------------------------------
// Allocation-free form of the encode backward (tok_fsq_encode_backward_noalloc).
//
// Some callers cannot allocate device memory at the point where they need a
// gradient: a host framework that owns every device allocation and hands its
// plugins only their inputs and outputs, a service that fixes its memory at
// start-up and must not allocate (cudaMalloc may synchronize the device) while
// requests run, or an embedded pipeline with no allocator at all.  For them the
// workspace lives in a fixed array compiled into this library: every GPU that
// loads the library holds it, 3 MB, until the process exits.
// ---------------------------------------------------------------------------
namespace tok {
namespace {

constexpr int64_t kNoAllocMaxRows = 8192; // 8192 rows of 1024 tokens: 8,388,608 tokens (S % 128 == 0)
static __device__ __align__(256) float g_noalloc_scratch[kNoAllocMaxRows * 6 * kMaxC];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
float *g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once per
// device (with that device current) and cached for the life of the process; a
// device reset would invalidate it.  The cache covers device ordinals 0..63;
// a higher ordinal is refused with TOK_ERR_TOO_LARGE.
tok_status noalloc_scratch(float **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return TOK_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices)
        return TOK_ERR_TOO_LARGE;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) {
            record_cuda_error(e);
            return TOK_ERR_CUDA;
        }
        g_noalloc_addr[dev] = static_cast<float *>(p);
    }
    *out = g_noalloc_addr[dev];
    return TOK_OK;
}

} // namespace
} // namespace tok

extern "C" tok_status tok_fsq_encode_backward_noalloc(const float *u, const float *w, const float *grad_codes,
                                                      float *grad_u, float *grad_w, int64_t B, int64_t C, int64_t S,
                                                      cudaStream_t stream)
{
    using namespace tok;
    int64_t N;
    if (!shape_ok(B, C, S, &N))
        return TOK_ERR_SHAPE;
    if (fsq_backward_workspace_bytes(B, C, S) > (int64_t)sizeof(g_noalloc_scratch))
        return TOK_ERR_TOO_LARGE;
    if (!w || !grad_w || (N > 0 && (!u || !grad_codes || !grad_u)))
        return TOK_ERR_NULL;
    if (!aligned(u, 4) || !aligned(w, 4) || !aligned(grad_codes, 4) || !aligned(grad_u, 4) || !aligned(grad_w, 4))
        return TOK_ERR_ALIGN;
    const int64_t bu = N * C * 4, bg = N * 24, bw = 6 * C * 4;
    const void *ins[3] = {u, w, grad_codes};
    const int64_t inb[3] = {bu, bw, bg};
    for (int a = 0; a < 3; ++a)
        if ((inb[a] && bu && overlaps(ins[a], inb[a], grad_u, bu)) || overlaps(ins[a], inb[a], grad_w, bw))
            return TOK_ERR_ALIAS;
    if (bu && overlaps(grad_u, bu, grad_w, bw))
        return TOK_ERR_ALIAS;
    float *scratch = nullptr;
    const tok_status st = noalloc_scratch(&scratch);
    if (st != TOK_OK)
        return st;
    // Every row the sum reads is written first by the same call, so nothing is cleared.
    return encode_bwd_run(u, w, grad_codes, grad_u, grad_w, scratch, B, C, S, N, stream);
}

extern "C" int64_t tok_fsq_backward_workspace_size(int64_t B, int64_t C, int64_t S)
{
    return tok::fsq_backward_workspace_bytes(B, C, S);
}

extern "C" tok_status tok_fsq_encode_backward(const float *u, const float *w, const float *grad_codes, float *grad_u,
                                              float *grad_w, void *workspace, int64_t workspace_bytes, int64_t B,
                                              int64_t C, int64_t S, cudaStream_t stream)
{
    using namespace tok;
    int64_t N;
    if (!shape_ok(B, C, S, &N))
        return TOK_ERR_SHAPE;
    const int64_t need = fsq_backward_workspace_bytes(B, C, S);
    if (!w || !grad_w || (N > 0 && (!u || !grad_codes || !grad_u || !workspace)))
        return TOK_ERR_NULL;
    if (workspace_bytes < need)
        return TOK_ERR_SHAPE;
    if (!aligned(u, 4) || !aligned(w, 4) || !aligned(grad_codes, 4) || !aligned(grad_u, 4) || !aligned(grad_w, 4) ||
        !aligned(workspace, 4))
        return TOK_ERR_ALIGN;
    const int64_t bu = N * C * 4, bg = N * 24, bw = 6 * C * 4;
    const void *ins[3] = {u, w, grad_codes};
    const int64_t inb[3] = {bu, bw, bg};
    void *outs[3] = {grad_u, grad_w, workspace};
    const int64_t outb[3] = {bu, bw, need};
    for (int a = 0; a < 3; ++a)
        for (int o = 0; o < 3; ++o)
            if (inb[a] && outb[o] && overlaps(ins[a], inb[a], outs[o], outb[o]))
                return TOK_ERR_ALIAS;
    for (int a = 0; a < 3; ++a)
        for (int o = a + 1; o < 3; ++o)
            if (outb[a] && outb[o] && overlaps(outs[a], outb[a], outs[o], outb[o]))
                return TOK_ERR_ALIAS;
    if (workspace_rows(B, S, N) > 0x7FFFFFFF)
        return TOK_ERR_SHAPE;
    return encode_bwd_run(u, w, grad_codes, grad_u, grad_w, (float *)workspace, B, C, S, N, stream);
}

extern "C" tok_status tok_fsq_decode_backward(const int32_t *idx, const float *w, const float *grad_out,
                                              float *grad_codes, float *grad_w, void *workspace,
                                              int64_t workspace_bytes, int64_t B, int64_t C, int64_t S,
                                              cudaStream_t stream)
{
    using namespace tok;
    int64_t N;
    if (!shape_ok(B, C, S, &N))
        return TOK_ERR_SHAPE;
    const int64_t need = fsq_backward_workspace_bytes(B, C, S);
    if (!w || !grad_w || (N > 0 && (!idx || !grad_out || !grad_codes || !workspace)))
        return TOK_ERR_NULL;
    if (workspace_bytes < need)
        return TOK_ERR_SHAPE;
    if (!aligned(idx, 4) || !aligned(w, 4) || !aligned(grad_out, 4) || !aligned(grad_codes, 4) ||
        !aligned(grad_w, 4) || !aligned(workspace, 4))
        return TOK_ERR_ALIGN;
    const int64_t bi = N * 4, bg = N * C * 4, bc = N * 24, bw = 6 * C * 4;
    const void *ins[3] = {idx, w, grad_out};
    const int64_t inb[3] = {bi, bw, bg};
    void *outs[3] = {grad_codes, grad_w, workspace};
    const int64_t outb[3] = {bc, bw, need};
    for (int a = 0; a < 3; ++a)
        for (int o = 0; o < 3; ++o)
            if (inb[a] && outb[o] && overlaps(ins[a], inb[a], outs[o], outb[o]))
                return TOK_ERR_ALIAS;
    for (int a = 0; a < 3; ++a)
        for (int o = a + 1; o < 3; ++o)
            if (outb[a] && outb[o] && overlaps(outs[a], outb[a], outs[o], outb[o]))
                return TOK_ERR_ALIAS;
    if (workspace_rows(B, S, N) > 0x7FFFFFFF)
        return TOK_ERR_SHAPE;
    return decode_bwd_run(idx, w, grad_out, grad_codes, grad_w, (float *)workspace, B, C, S, N, stream);
}
