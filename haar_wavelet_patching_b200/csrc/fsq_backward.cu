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
// sech^2(x) is evaluated as 4a / (1 + a)^2 with a = exp(-2|x|): accurate where
// tanh saturates, unlike 1 - tanh^2.
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
// batch row, then position).
// A two-stage ring of TMA loads brings a tile's inputs into shared memory while
// the previous tile is computed; each lane owns 4 consecutive tokens, reads
// them with 16-byte shared loads and writes its outputs with 16-byte global
// stores.  The grad_w accumulators stay in registers across the CTA's tiles and
// are reduced by a shuffle butterfly into the CTA's workspace row.  Other
// shapes take the register kernels (2048 tokens per CTA, 128 threads).
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
    float shift[6]; // atanh(off / half)
    float scale[6]; // half / floor(L / 2)
};

SlopeConsts slope_consts()
{
    static const int L[6] = {8, 8, 8, 5, 5, 5};
    SlopeConsts k{};
    for (int i = 0; i < 6; ++i) {
        const double half = (L[i] - 1) * (1.0 + 1e-3) / 2.0;
        const double off = (L[i] % 2 == 0) ? 0.5 : 0.0;
        k.shift[i] = (float)std::atanh(off / half);
        k.scale[i] = (float)(half / (double)(L[i] / 2));
    }
    return k;
}

// sech^2(x) = 4a / (1 + a)^2 with a = e^{-2|x|} in (0, 1]: the quotient's
// denominator lies in [1, 4], where the fast division is accurate to a few ulp;
// the fast exponential's relative error grows like |x| * 2^-24, so sech^2 keeps
// about 1e-6 relative accuracy for |x| <= 20 (beyond, a < 5e-18 is negligible
// next to the slopes that matter).
__device__ __forceinline__ float sech2(float x)
{
    const float a = __expf(-2.0f * fabsf(x));
    const float d = 1.0f + a;
    return __fdividef(4.0f * a, d * d);
}

// Reduces the per-thread accumulators acc[i * kMaxC + c] over the CTA in a fixed
// order and writes the CTA's row of 6*C sums, row[i * C + c].  All indices into
// acc are compile-time constants, so it stays in registers.
__device__ __forceinline__ void reduce_rows(const float (&acc)[6 * kMaxC], int C, float *red, float *row)
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
        row[k] = s;
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
            t[i] = g[(b * 6 + i) * S + s] * (k.scale[i] * sech2(z + k.shift[i]));
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
    reduce_rows(acc, C, red, partial + (int64_t)blockIdx.x * 6 * C);
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
    reduce_rows(acc, C, red, partial + (int64_t)blockIdx.x * 6 * C);
}

// grad_w[k] = sum over the rows of partial, in double, in a fixed order: one CTA
// per entry k; thread t sums rows t, t + 256, ... in order, then a pairwise tree
// over the threads.
constexpr int kSumThreads = 256;
__global__ void __launch_bounds__(kSumThreads)
    fsq_bwd_sum_rows_kernel(const float *__restrict__ partial, int64_t rows, int K, float *__restrict__ out)
{
    __shared__ double part[kSumThreads];
    const int k = blockIdx.x;
    double s = 0.0;
#pragma unroll 8
    for (int64_t r = threadIdx.x; r < rows; r += kSumThreads)
        s += (double)partial[r * K + k];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int half = kSumThreads / 2; half > 0; half >>= 1) {
        if (threadIdx.x < half)
            part[threadIdx.x] += part[threadIdx.x + half];
        __syncthreads();
    }
    if (threadIdx.x == 0)
        out[k] = (float)part[0];
}

// ---------------------------------------------------------------------------
// Main path.
// ---------------------------------------------------------------------------

// grad_w on the main path.  A pair of lanes (2p, 2p + 1) covers the pair's 8 tokens
// 8p .. 8p + 7 of the tile; lane 2p + h accumulates the channels c = 8h .. 8h + 7, so
// a lane holds 48 sums acc[i * 8 + cc] (c = 8h + cc) instead of 96.
constexpr int kHalfC = 8;

// Sums acc over the 16 lanes of the same half (xor butterfly over lane bits 1..4:
// every lane ends with the same sums in the same order) and writes them to
// row[i * 16 + 8h + cc], three entries per lane.
__device__ __forceinline__ void warp_row_half(float (&acc)[6 * kHalfC], float *row)
{
    const int lane = threadIdx.x & 31, h = lane & 1;
#pragma unroll
    for (int q = 0; q < 6 * kHalfC; ++q) {
        float v = acc[q];
#pragma unroll
        for (int off = 16; off > 1; off >>= 1)
            v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
        if ((q & 15) == (lane >> 1))
            row[(q / kHalfC) * 16 + kHalfC * h + (q % kHalfC)] = v;
    }
}

// Weights in shared memory as ws[c * 8 + i] = w[i][c] (i < 6; 6 and 7 are zero),
// so one 16-byte and one 8-byte load give a channel's six weights.
__device__ __forceinline__ void stage_ws16(const float *__restrict__ w, float *ws)
{
    for (int q = threadIdx.x; q < 16 * 8; q += 32) {
        const int c = q >> 3, i = q & 7;
        ws[q] = i < 6 ? w[i * 16 + c] : 0.0f;
    }
}

__device__ __forceinline__ void weights_of(const float *ws, int c, float (&wc)[6])
{
    const float4 wa = *reinterpret_cast<const float4 *>(ws + c * 8);
    const float2 wb = *reinterpret_cast<const float2 *>(ws + c * 8 + 4);
    wc[0] = wa.x, wc[1] = wa.y, wc[2] = wa.z, wc[3] = wa.w, wc[4] = wb.x, wc[5] = wb.y;
}

// Digits of a valid index, as normalized codes; an invalid index gives zeros.
__device__ __forceinline__ void zhat_of(int32_t id, float (&zh)[6])
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
    zh[0] = v * ((float)(d0 - 4) * 0.25f);
    zh[1] = v * ((float)(d1 - 4) * 0.25f);
    zh[2] = v * ((float)(d2 - 4) * 0.25f);
    zh[3] = v * ((float)(d3 - 2) * 0.5f);
    zh[4] = v * ((float)(d4 - 2) * 0.5f);
    zh[5] = v * ((float)(d5 - 2) * 0.5f);
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

// Encode backward, C = 16.  Stage layout: u tile [16][128] then g tile [6][128] (fp32);
// each lane overwrites its own tokens' g with t = g * slope(z), which the lane pair
// then reads back for grad_w.
template <int TPR, int STAGES>
__global__ void __launch_bounds__(32)
    fsq_encode_bwd_tma_kernel(const __grid_constant__ CUtensorMap umap, const __grid_constant__ CUtensorMap gmap,
                              const float *__restrict__ w, float *__restrict__ gu, float *__restrict__ partial,
                              int64_t S, FastDiv ntx, uint32_t ntiles, SlopeConsts k)
{
    constexpr int U_BYTES = 16 * kTileTokens * 4, STAGE = U_BYTES + 6 * kTileTokens * 4;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + STAGES * STAGE);
    float *ws = reinterpret_cast<float *>(smem_raw + STAGES * STAGE + 16 * STAGES); // 16-byte aligned
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
    stage_ws16(w, ws);
    __syncwarp();

    float acc[6 * kHalfC];
#pragma unroll
    for (int q = 0; q < 6 * kHalfC; ++q)
        acc[q] = 0.0f;

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
                float wc[6];
                weights_of(ws, c, wc);
#pragma unroll
                for (int i = 0; i < 6; ++i) {
                    const float2 wi = make_float2(wc[i], wc[i]);
                    z[i][0] = __ffma2_rn(wi, make_float2(q.x, q.y), z[i][0]);
                    z[i][1] = __ffma2_rn(wi, make_float2(q.z, q.w), z[i][1]);
                }
            }
            // t_i = g_i * slope_i(z_i), kept in registers and written over g.
            float t[6][4];
#pragma unroll
            for (int i = 0; i < 6; ++i) {
                float4 *gp = reinterpret_cast<float4 *>(tg + i * kTileTokens + 4 * lane);
                const float4 gq = *gp;
                const float zz[4] = {z[i][0].x, z[i][0].y, z[i][1].x, z[i][1].y}, gg[4] = {gq.x, gq.y, gq.z, gq.w};
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    t[i][m] = gg[m] * (k.scale[i] * sech2(zz[m] + k.shift[i]));
                *gp = make_float4(t[i][0], t[i][1], t[i][2], t[i][3]);
            }
            // grad_u = sum_i w[i][c] t_i, the chain over i from 0, for the lane's tokens.
            const int64_t t0 = (int64_t)tx * kTileTokens + 4 * lane;
            if (t0 < S) { // S % 4 == 0: a lane's four tokens are all in range or all out
                float *gub = gu + (int64_t)b * 16 * S + t0;
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    float wc[6];
                    weights_of(ws, c, wc);
                    float o[4];
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        float a = 0.0f;
#pragma unroll
                        for (int i = 0; i < 6; ++i)
                            a = fmaf(wc[i], t[i][m], a);
                        o[m] = a;
                    }
                    *reinterpret_cast<float4 *>(gub) = make_float4(o[0], o[1], o[2], o[3]);
                    gub += S;
                }
            }
        }
        __syncwarp(); // t of the partner lane is in shared memory
        // grad_w: the pair's 8 tokens, channels 8h .. 8h + 7, tokens in increasing order.
#pragma unroll
        for (int g2 = 0; g2 < 2; ++g2) {
            const int col = 4 * ((lane & ~1) + g2);
            float t[6][4];
#pragma unroll
            for (int i = 0; i < 6; ++i) {
                const float4 tq = *reinterpret_cast<const float4 *>(tg + i * kTileTokens + col);
                t[i][0] = tq.x, t[i][1] = tq.y, t[i][2] = tq.z, t[i][3] = tq.w;
            }
#pragma unroll
            for (int cc = 0; cc < kHalfC; ++cc) {
                const float4 q = *reinterpret_cast<const float4 *>(tu + (kHalfC * h + cc) * kTileTokens + col);
                const float uq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int i = 0; i < 6; ++i)
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        acc[i * kHalfC + cc] = fmaf(t[i][m], uq[m], acc[i * kHalfC + cc]);
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
    warp_row_half(acc, partial + (int64_t)blockIdx.x * 6 * kMaxC);
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
    float *ws = reinterpret_cast<float *>(smem_raw + STAGES * STAGE + 16 * STAGES); // 16-byte aligned
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
    stage_ws16(w, ws);
    __syncwarp();

    float acc[6 * kHalfC];
#pragma unroll
    for (int q = 0; q < 6 * kHalfC; ++q)
        acc[q] = 0.0f;

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
            const bool valid[4] = {(uint32_t)iq.x < (uint32_t)TOK_FSQ_CODEBOOK,
                                   (uint32_t)iq.y < (uint32_t)TOK_FSQ_CODEBOOK,
                                   (uint32_t)iq.z < (uint32_t)TOK_FSQ_CODEBOOK,
                                   (uint32_t)iq.w < (uint32_t)TOK_FSQ_CODEBOOK};
            float gc[6][4];
#pragma unroll
            for (int i = 0; i < 6; ++i)
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    gc[i][m] = 0.0f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float4 q = *reinterpret_cast<const float4 *>(tgl + c * kTileTokens + 4 * lane);
                const float gq[4] = {q.x, q.y, q.z, q.w};
                float wc[6];
                weights_of(ws, c, wc);
#pragma unroll
                for (int i = 0; i < 6; ++i)
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        gc[i][m] = fmaf(wc[i], gq[m], gc[i][m]);
            }
            float *gcb = gcodes + (int64_t)b * 6 * S + t0;
#pragma unroll
            for (int i = 0; i < 6; ++i)
                *reinterpret_cast<float4 *>(gcb + (int64_t)i * S) =
                    make_float4(valid[0] ? gc[i][0] : 0.0f, valid[1] ? gc[i][1] : 0.0f, valid[2] ? gc[i][2] : 0.0f,
                                valid[3] ? gc[i][3] : 0.0f);
        }
        // grad_w: the pair's 8 tokens, channels 8h .. 8h + 7, tokens in increasing order.
#pragma unroll
        for (int g2 = 0; g2 < 2; ++g2) {
            const int col = 4 * ((lane & ~1) + g2);
            const int4 iq = *reinterpret_cast<const int4 *>(tid + col);
            const int32_t ids[4] = {iq.x, iq.y, iq.z, iq.w};
            float zh[4][6];
#pragma unroll
            for (int m = 0; m < 4; ++m)
                zhat_of(ids[m], zh[m]);
#pragma unroll
            for (int cc = 0; cc < kHalfC; ++cc) {
                const float4 q = *reinterpret_cast<const float4 *>(tgl + (kHalfC * h + cc) * kTileTokens + col);
                const float gq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                for (int i = 0; i < 6; ++i)
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        acc[i * kHalfC + cc] = fmaf(zh[m][i], gq[m], acc[i * kHalfC + cc]);
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
    warp_row_half(acc, partial + (int64_t)blockIdx.x * 6 * kMaxC);
}

// Shared memory: the stages (multiples of 128 bytes), one 16-byte slot per stage for
// its barrier, then the weights.
template <int STAGES> constexpr int enc_smem() { return STAGES * (22 * kTileTokens * 4 + 16) + 16 * 8 * 4; }
template <int STAGES> constexpr int dec_smem() { return STAGES * (17 * kTileTokens * 4 + 16) + 16 * 8 * 4; }

// Tiles of the main path: B * ceil(S / 128).
int64_t tma_tiles(int64_t B, int64_t S) { return B * ((S + kTileTokens - 1) / kTileTokens); }

// The main path takes C = 16 with S % 4 == 0 (16-byte rows for TMA and for the
// lanes' 16-byte stores) and 16-byte-aligned tensors.
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
    fsq_bwd_sum_rows_kernel<<<(unsigned)(6 * C), kSumThreads, 0, stream>>>(partial, rows, (int)(6 * C), gw);
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
    fsq_bwd_sum_rows_kernel<<<(unsigned)(6 * C), kSumThreads, 0, stream>>>(partial, rows, (int)(6 * C), gw);
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
// device (with that device current) and cached.
tok_status noalloc_scratch(float **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return TOK_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices)
        return TOK_ERR_CUDA;
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
