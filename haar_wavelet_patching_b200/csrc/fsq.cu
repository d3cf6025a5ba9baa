// Fused projection + FSQ encode, and FSQ decode + projection, for sm_100a.
//
// Sources: "NVIDIA Cosmos Tokenizer 完全指南", section 7.2 (six channels with
// levels [8,8,8,5,5,5], a tanh-based bound then rounding, implicit codebook of
// 64000, mixed-radix codes_to_indices / indices_to_codes) and section 6.2
// (indices [B,t,h,w], codes [B,6,t,h,w]); "Cosmos World Foundation Model
// Platform for Physical AI (Cosmos-Predict1)" notes, model architecture item 1.
// The bound's constants follow the published FSQ method (Mentzer et al., 2023):
// half = (L-1)(1+1e-3)/2, off = 0.5 for even L, shift = atanh(off/half),
// q = round(tanh(z + shift)*half - off).
//
// Encode evaluates no tanh.  The bound is strictly increasing in z, so q is
// fixed by how many of the L-1 rounding boundaries z exceeds; boundary m sits at
// theta_m = atanh((q_min + m + 0.5 + off)/half) - shift.  The host computes each
// theta_m in double and passes the smallest fp32 value above it, t_m; for an
// fp32 z, "z > theta_m" is exactly "z >= t_m", so the digit is a count of
// comparisons and agrees with the rounded tanh except for z within double
// rounding of a boundary.
//
// The projection z_i = sum_c w[i][c] u_c is a chain of fused multiply-adds
// over c = 0..C-1 starting from 0, the same fp32 value on any conforming FMA.
//
// Memory: encode reads 4C bytes and writes 4 bytes per token (plus 24 with
// codes); decode reads 4 and writes 4C.  At C = 16 that is 68 bytes against
// ~96 FMAs and 33 compares per token, under the HBM roofline.
//
// Encode at C = 16 with 16-byte-aligned tensors (the main path): one-shot
// single-warp CTAs, each owning one tile of 128 consecutive tokens x 16
// channel planes (8 KB); lane 0 issues its TMA load, the lanes take
// 4 tokens each and run the projection as packed f32x2 fused multiply-adds
// (two tokens per instruction, each lane of the pair the same fp32 chain).  A
// grid of small CTAs in token order keeps the working set a compact, moving
// window, which measured well above a grid of large CTAs on B200.
// Other shapes, and decode, use CTAs of 256 threads in which a thread owns 4
// consecutive tokens of one batch item: one 16-byte load or store per channel
// plane, 512 contiguous bytes per warp.  The weight lives in shared memory as
// [c][8] (6 used), read with two broadcast vector loads per channel.
#include <cmath>
#include <cstring>

#include "tma.cuh"
#include "tok_common.cuh"
#include "tok_internal.h"

namespace tok {

// FSQ kernels that gave up on a barrier wait since the last check.
static __device__ unsigned int g_fsq_wait_timeouts = 0;

namespace {

constexpr int kThreads = 256;
constexpr int kMaxC = 1024;

struct Thresholds {
    float t8[7]; // L = 8: z >= t8[m] <=> z is above boundary m
    float t5[4]; // L = 5
};

void fill_thresholds(int L, float *t)
{
    const double half = (L - 1) * (1.0 + 1e-3) / 2.0;
    const double off = (L % 2 == 0) ? 0.5 : 0.0;
    const double shift = std::atanh(off / half);
    const int q_min = -(L / 2);
    for (int m = 0; m < L - 1; ++m) {
        const double theta = std::atanh((q_min + m + 0.5 + off) / half) - shift;
        float f = (float)theta;
        if ((double)f <= theta)
            f = std::nextafterf(f, INFINITY);
        t[m] = f;
    }
}

const Thresholds &thresholds()
{
    static const Thresholds th = [] {
        Thresholds t{};
        fill_thresholds(8, t.t8);
        fill_thresholds(5, t.t5);
        return t;
    }();
    return th;
}

template <int N> __device__ __forceinline__ int count_at_or_above(float z, const float (&t)[N])
{
    int d = 0;
#pragma unroll
    for (int m = 0; m < N; ++m)
        d += (z >= t[m]) ? 1 : 0;
    return d;
}

// Stage w [6][C] as ws[c*8 + i] so channel c's six weights are two float4 loads.
__device__ __forceinline__ void stage_weight(const float *__restrict__ w, float *ws, int C)
{
    for (int k = threadIdx.x; k < 8 * C; k += blockDim.x) {
        const int c = k >> 3, i = k & 7;
        ws[k] = (i < 6) ? w[i * C + c] : 0.0f;
    }
    __syncthreads();
}

template <int TPT, bool VEC> __device__ __forceinline__ void load_tokens(const float *p, float *v)
{
    if constexpr (VEC) {
        const uint4 r = ld_stream_u4(p);
        v[0] = __uint_as_float(r.x);
        v[1] = __uint_as_float(r.y);
        v[2] = __uint_as_float(r.z);
        v[3] = __uint_as_float(r.w);
    } else {
#pragma unroll
        for (int t = 0; t < TPT; ++t)
            v[t] = __uint_as_float(ld_stream_u1(p + t));
    }
}

template <int TPT, bool VEC> __device__ __forceinline__ void store_tokens(float *p, const float *v)
{
    if constexpr (VEC)
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else
#pragma unroll
        for (int t = 0; t < TPT; ++t)
            p[t] = v[t];
}

// CT: compile-time channel count (0 = runtime C).  TPT tokens per thread
// (VEC: 4 with 16-byte accesses; else 1).
template <int CT, int TPT, bool VEC>
__global__ void __launch_bounds__(kThreads)
    fsq_encode_kernel(const float *__restrict__ u, const float *__restrict__ w, int32_t *__restrict__ idx,
                      float *__restrict__ codes, int64_t B, int C_rt, int64_t S, Thresholds th)
{
    extern __shared__ float4 ws4[];
    const int C = CT > 0 ? CT : C_rt;
    stage_weight(w, reinterpret_cast<float *>(ws4), C);

    const int64_t groups = S / TPT, n = B * groups;
    for (int64_t gi = (int64_t)blockIdx.x * kThreads + threadIdx.x; gi < n; gi += (int64_t)gridDim.x * kThreads) {
        const int64_t b = gi / groups;
        const int64_t s = (gi - b * groups) * TPT;
        const float *ub = u + b * C * S + s;
        float z[6][TPT];
#pragma unroll
        for (int i = 0; i < 6; ++i)
#pragma unroll
            for (int t = 0; t < TPT; ++t)
                z[i][t] = 0.0f;
        auto step = [&](int c) {
            float uv[TPT];
            load_tokens<TPT, VEC>(ub + (int64_t)c * S, uv);
            const float4 wa = ws4[2 * c], wb = ws4[2 * c + 1];
#pragma unroll
            for (int t = 0; t < TPT; ++t) {
                z[0][t] = fmaf(wa.x, uv[t], z[0][t]);
                z[1][t] = fmaf(wa.y, uv[t], z[1][t]);
                z[2][t] = fmaf(wa.z, uv[t], z[2][t]);
                z[3][t] = fmaf(wa.w, uv[t], z[3][t]);
                z[4][t] = fmaf(wb.x, uv[t], z[4][t]);
                z[5][t] = fmaf(wb.y, uv[t], z[5][t]);
            }
        };
        if constexpr (CT > 0) {
#pragma unroll
            for (int c = 0; c < CT; ++c)
                step(c);
        } else {
#pragma unroll 4
            for (int c = 0; c < C; ++c)
                step(c);
        }
        float id[TPT];
        float zh[6][TPT];
#pragma unroll
        for (int t = 0; t < TPT; ++t) {
            const int d0 = count_at_or_above(z[0][t], th.t8);
            const int d1 = count_at_or_above(z[1][t], th.t8);
            const int d2 = count_at_or_above(z[2][t], th.t8);
            const int d3 = count_at_or_above(z[3][t], th.t5);
            const int d4 = count_at_or_above(z[4][t], th.t5);
            const int d5 = count_at_or_above(z[5][t], th.t5);
            id[t] = __int_as_float(d0 + 8 * d1 + 64 * d2 + 512 * d3 + 2560 * d4 + 12800 * d5);
            zh[0][t] = (float)(d0 - 4) * 0.25f;
            zh[1][t] = (float)(d1 - 4) * 0.25f;
            zh[2][t] = (float)(d2 - 4) * 0.25f;
            zh[3][t] = (float)(d3 - 2) * 0.5f;
            zh[4][t] = (float)(d4 - 2) * 0.5f;
            zh[5][t] = (float)(d5 - 2) * 0.5f;
        }
        store_tokens<TPT, VEC>(reinterpret_cast<float *>(idx + b * S + s), id);
        if (codes) {
#pragma unroll
            for (int i = 0; i < 6; ++i)
                store_tokens<TPT, VEC>(codes + (b * 6 + i) * S + s, zh[i]);
        }
    }
}

// ---------------------------------------------------------------------------
// Encode, TMA path (C = 16).
// ---------------------------------------------------------------------------
constexpr int kEncTokens = 128; // tokens per tile: 16 planes x 512 bytes = 8 KB
constexpr int kEncKT = 1;       // tiles per CTA (one: more resident warps measured faster than two or four)
constexpr int kEncSmem = kEncKT * 16 * kEncTokens * 4 + 16 * kEncKT + 16 * 8 * 4; // tiles, barriers, weights

template <bool CODES>
__global__ void __launch_bounds__(32)
    fsq_encode_tma_kernel(const __grid_constant__ CUtensorMap umap, const float *__restrict__ w,
                          int32_t *__restrict__ idx, float *__restrict__ codes, int64_t S, FastDiv ntx,
                          uint32_t ntiles, Thresholds th)
{
    constexpr int TILE = 16 * kEncTokens;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    float *tiles = reinterpret_cast<float *>(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + kEncKT * TILE * 4);
    float *ws = reinterpret_cast<float *>(smem_raw + kEncKT * TILE * 4 + 16 * kEncKT); // [16][8], 16-byte aligned
    const int lane = threadIdx.x;
    const uint32_t first = blockIdx.x * (uint32_t)kEncKT;
    const int count = (int)min((uint32_t)kEncKT, ntiles - first);

    if (lane == 0) {
        for (int s = 0; s < kEncKT; ++s)
            mbar_init(smem_addr(bars + s), 1);
        fence_barrier_init();
        for (int s = 0; s < count; ++s) {
            const uint32_t n = first + s, b = ntx.div(n), tx = n - b * ntx.d;
            const uint32_t bar = smem_addr(bars + s);
            mbar_expect_tx(bar, TILE * 4);
            tma_load_3d(smem_addr(tiles + s * TILE), &umap, (int)(tx * kEncTokens), 0, (int)b, bar);
        }
    }
    for (int k = lane; k < 16 * 8; k += 32) {
        const int c = k >> 3, i = k & 7;
        ws[k] = (i < 6) ? w[i * 16 + c] : 0.0f;
    }
    __syncwarp();

    int s = 0;
    for (; s < count; ++s) {
        const bool ok = mbar_wait(smem_addr(bars + s), 0u);
        if (__any_sync(0xFFFFFFFFu, !ok))
            break;
        const uint32_t n = first + s, b = ntx.div(n), tx = n - b * ntx.d;
        const float *tin = tiles + s * TILE;
        // z[i][0] holds tokens (0, 1) of this lane, z[i][1] tokens (2, 3).
        float2 z[6][2];
#pragma unroll
        for (int i = 0; i < 6; ++i)
            z[i][0] = z[i][1] = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const float4 q = *reinterpret_cast<const float4 *>(tin + c * kEncTokens + 4 * lane);
            const float4 wa = *reinterpret_cast<const float4 *>(ws + c * 8);
            const float2 wb = *reinterpret_cast<const float2 *>(ws + c * 8 + 4);
            const float wc[6] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y};
            const float2 u01 = make_float2(q.x, q.y), u23 = make_float2(q.z, q.w);
#pragma unroll
            for (int i = 0; i < 6; ++i) {
                const float2 wi = make_float2(wc[i], wc[i]);
                z[i][0] = __ffma2_rn(wi, u01, z[i][0]);
                z[i][1] = __ffma2_rn(wi, u23, z[i][1]);
            }
        }
        const int64_t t0 = (int64_t)tx * kEncTokens + 4 * lane;
        if (t0 >= S) // S % 4 == 0: a lane's four tokens are all in range or all out
            continue;
        float id[4], zh[6][4];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            float zt[6];
#pragma unroll
            for (int i = 0; i < 6; ++i) {
                const float2 p = z[i][t >> 1];
                zt[i] = (t & 1) ? p.y : p.x;
            }
            const int d0 = count_at_or_above(zt[0], th.t8), d1 = count_at_or_above(zt[1], th.t8);
            const int d2 = count_at_or_above(zt[2], th.t8), d3 = count_at_or_above(zt[3], th.t5);
            const int d4 = count_at_or_above(zt[4], th.t5), d5 = count_at_or_above(zt[5], th.t5);
            id[t] = __int_as_float(d0 + 8 * d1 + 64 * d2 + 512 * d3 + 2560 * d4 + 12800 * d5);
            if constexpr (CODES) {
                zh[0][t] = (float)(d0 - 4) * 0.25f;
                zh[1][t] = (float)(d1 - 4) * 0.25f;
                zh[2][t] = (float)(d2 - 4) * 0.25f;
                zh[3][t] = (float)(d3 - 2) * 0.5f;
                zh[4][t] = (float)(d4 - 2) * 0.5f;
                zh[5][t] = (float)(d5 - 2) * 0.5f;
            }
        }
        *reinterpret_cast<float4 *>(idx + (int64_t)b * S + t0) = make_float4(id[0], id[1], id[2], id[3]);
        if constexpr (CODES) {
#pragma unroll
            for (int i = 0; i < 6; ++i)
                *reinterpret_cast<float4 *>(codes + ((int64_t)b * 6 + i) * S + t0) =
                    make_float4(zh[i][0], zh[i][1], zh[i][2], zh[i][3]);
        }
    }

    if (s < count && lane == 0) {
        for (int r = s; r < count; ++r) // drain, each wait again bounded
            mbar_wait(smem_addr(bars + r), 0u);
        atomicAdd(&g_fsq_wait_timeouts, 1u);
    }
    __syncwarp();
}

// Launches the TMA encode, or returns false if the layout does not suit it.
bool try_encode_tma(const float *u, const float *w, int32_t *idx, float *codes, int64_t B, int64_t C, int64_t S,
                    cudaStream_t stream, tok_status *st)
{
    if (C != 16 || S % 4 != 0 || !aligned(u, 16) || !aligned(idx, 16) || (codes && !aligned(codes, 16)))
        return false;
    const int64_t ntx = (S + kEncTokens - 1) / kEncTokens, ntiles = ntx * B;
    if (S >= ((int64_t)1 << 31) || B >= ((int64_t)1 << 31) || ntiles >= ((int64_t)1 << 32) || sm_count() <= 0)
        return false;
    CUtensorMap umap;
    memset(&umap, 0, sizeof umap);
    const uint64_t dims[3] = {(uint64_t)S, 16, (uint64_t)B}, strides[2] = {(uint64_t)S * 4, (uint64_t)S * 16 * 4};
    const uint32_t box[3] = {(uint32_t)kEncTokens, 16, 1};
    if (!encode_tensor_map(&umap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, u, dims, strides, box))
        return false;
    auto kern = codes ? fsq_encode_tma_kernel<true> : fsq_encode_tma_kernel<false>;
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kEncSmem);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        *st = TOK_ERR_CUDA;
        return true;
    }
    const unsigned grid = (unsigned)((ntiles + kEncKT - 1) / kEncKT);
    kern<<<grid, 32, kEncSmem, stream>>>(umap, w, idx, codes, S, FastDiv((uint32_t)ntx), (uint32_t)ntiles,
                                         thresholds());
    *st = launch_status();
    return true;
}

template <int CT, int TPT, bool VEC>
__global__ void __launch_bounds__(kThreads)
    fsq_decode_kernel(const int32_t *__restrict__ idx, const float *__restrict__ w, float *__restrict__ out,
                      int32_t *__restrict__ bad_count, int64_t B, int C_rt, int64_t S)
{
    extern __shared__ float4 ws4[];
    const int C = CT > 0 ? CT : C_rt;
    stage_weight(w, reinterpret_cast<float *>(ws4), C);

    int n_bad = 0;
    const int64_t groups = S / TPT, n = B * groups;
    for (int64_t gi = (int64_t)blockIdx.x * kThreads + threadIdx.x; gi < n; gi += (int64_t)gridDim.x * kThreads) {
        const int64_t b = gi / groups;
        const int64_t s = (gi - b * groups) * TPT;
        float raw[TPT];
        load_tokens<TPT, VEC>(reinterpret_cast<const float *>(idx + b * S + s), raw);
        float zh[6][TPT];
        bool bad[TPT];
#pragma unroll
        for (int t = 0; t < TPT; ++t) {
            const int32_t id = __float_as_int(raw[t]);
            bad[t] = (uint32_t)id >= (uint32_t)TOK_FSQ_CODEBOOK;
            n_bad += bad[t] ? 1 : 0;
            uint32_t r = bad[t] ? 0u : (uint32_t)id;
            const int d0 = r % 8u; r /= 8u;
            const int d1 = r % 8u; r /= 8u;
            const int d2 = r % 8u; r /= 8u;
            const int d3 = r % 5u; r /= 5u;
            const int d4 = r % 5u; r /= 5u;
            const int d5 = (int)r;
            zh[0][t] = (float)(d0 - 4) * 0.25f;
            zh[1][t] = (float)(d1 - 4) * 0.25f;
            zh[2][t] = (float)(d2 - 4) * 0.25f;
            zh[3][t] = (float)(d3 - 2) * 0.5f;
            zh[4][t] = (float)(d4 - 2) * 0.5f;
            zh[5][t] = (float)(d5 - 2) * 0.5f;
        }
        float *ob = out + b * C * S + s;
        auto step = [&](int c) {
            const float4 wa = ws4[2 * c], wb = ws4[2 * c + 1];
            float o[TPT];
#pragma unroll
            for (int t = 0; t < TPT; ++t) {
                float acc = fmaf(wa.x, zh[0][t], 0.0f);
                acc = fmaf(wa.y, zh[1][t], acc);
                acc = fmaf(wa.z, zh[2][t], acc);
                acc = fmaf(wa.w, zh[3][t], acc);
                acc = fmaf(wb.x, zh[4][t], acc);
                acc = fmaf(wb.y, zh[5][t], acc);
                o[t] = bad[t] ? __int_as_float(0x7FC00000) : acc;
            }
            store_tokens<TPT, VEC>(ob + (int64_t)c * S, o);
        };
        if constexpr (CT > 0) {
#pragma unroll
            for (int c = 0; c < CT; ++c)
                step(c);
        } else {
#pragma unroll 4
            for (int c = 0; c < C; ++c)
                step(c);
        }
    }
    if (bad_count) {
        const int warp_bad = __reduce_add_sync(0xFFFFFFFFu, n_bad);
        if ((threadIdx.x & 31) == 0 && warp_bad)
            atomicAdd(bad_count, warp_bad);
    }
}

unsigned grid_for(int64_t n)
{
    const int64_t blocks = (n + kThreads - 1) / kThreads;
    return (unsigned)(blocks < 0x7FFFFFFF ? (blocks > 0 ? blocks : 1) : 0x7FFFFFFF);
}

} // namespace

tok_status read_and_clear_fsq_timeouts(cudaStream_t stream, unsigned int *count)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(count, g_fsq_wait_timeouts, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && *count)
        e = cudaMemcpyToSymbolAsync(g_fsq_wait_timeouts, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice,
                                    stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return TOK_ERR_CUDA;
    }
    return TOK_OK;
}

} // namespace tok

extern "C" tok_status tok_fsq_encode(const float *u, const float *w, int32_t *idx, float *codes, int64_t B, int64_t C,
                                     int64_t S, cudaStream_t stream)
{
    using namespace tok;
    if (B < 0 || S < 0 || C < 1 || C > kMaxC)
        return TOK_ERR_SHAPE;
    int64_t nu, ntok, bu, bi, bc;
    if (!prod_ok({B, C, S}, &nu) || !prod_ok({B, S}, &ntok) || !prod_ok({nu, 4}, &bu) || !prod_ok({ntok, 4}, &bi) ||
        !prod_ok({ntok, 24}, &bc))
        return TOK_ERR_SHAPE;
    if (ntok == 0)
        return TOK_OK;
    if (!u || !w || !idx)
        return TOK_ERR_NULL;
    if (!aligned(u, 4) || !aligned(w, 4) || !aligned(idx, 4) || (codes && !aligned(codes, 4)))
        return TOK_ERR_ALIGN;
    const int64_t bw = 6 * C * 4;
    if (overlaps(u, bu, idx, bi) || overlaps(w, bw, idx, bi) ||
        (codes && (overlaps(u, bu, codes, bc) || overlaps(w, bw, codes, bc) || overlaps(idx, bi, codes, bc))))
        return TOK_ERR_ALIAS;
    tok_status st = TOK_OK;
    if (try_encode_tma(u, w, idx, codes, B, C, S, stream, &st))
        return st;
    const bool vec = S % 4 == 0 && aligned(u, 16) && aligned(idx, 16) && (!codes || aligned(codes, 16));
    const size_t smem = (size_t)C * 8 * sizeof(float);
    const Thresholds &th = thresholds();
    if (vec) {
        const unsigned grid = grid_for(B * (S / 4));
        if (C == 16)
            fsq_encode_kernel<16, 4, true><<<grid, kThreads, smem, stream>>>(u, w, idx, codes, B, (int)C, S, th);
        else
            fsq_encode_kernel<0, 4, true><<<grid, kThreads, smem, stream>>>(u, w, idx, codes, B, (int)C, S, th);
    } else {
        fsq_encode_kernel<0, 1, false><<<grid_for(ntok), kThreads, smem, stream>>>(u, w, idx, codes, B, (int)C, S, th);
    }
    return launch_status();
}

extern "C" tok_status tok_fsq_decode(const int32_t *idx, const float *w, float *out, int32_t *bad_count, int64_t B,
                                     int64_t C, int64_t S, cudaStream_t stream)
{
    using namespace tok;
    if (B < 0 || S < 0 || C < 1 || C > kMaxC)
        return TOK_ERR_SHAPE;
    int64_t nout, ntok, bo, bi;
    if (!prod_ok({B, C, S}, &nout) || !prod_ok({B, S}, &ntok) || !prod_ok({nout, 4}, &bo) || !prod_ok({ntok, 4}, &bi))
        return TOK_ERR_SHAPE;
    if (ntok == 0)
        return TOK_OK;
    if (!idx || !w || !out)
        return TOK_ERR_NULL;
    if (!aligned(idx, 4) || !aligned(w, 4) || !aligned(out, 4) || (bad_count && !aligned(bad_count, 4)))
        return TOK_ERR_ALIGN;
    const int64_t bw = 6 * C * 4;
    if (overlaps(idx, bi, out, bo) || overlaps(w, bw, out, bo) || (bad_count && overlaps(bad_count, 4, out, bo)))
        return TOK_ERR_ALIAS;
    const bool vec = S % 4 == 0 && aligned(idx, 16) && aligned(out, 16);
    const size_t smem = (size_t)C * 8 * sizeof(float);
    if (vec) {
        const unsigned grid = grid_for(B * (S / 4));
        if (C == 16)
            fsq_decode_kernel<16, 4, true><<<grid, kThreads, smem, stream>>>(idx, w, out, bad_count, B, (int)C, S);
        else
            fsq_decode_kernel<0, 4, true><<<grid, kThreads, smem, stream>>>(idx, w, out, bad_count, B, (int)C, S);
    } else {
        fsq_decode_kernel<0, 1, false><<<grid_for(ntok), kThreads, smem, stream>>>(idx, w, out, bad_count, B, (int)C, S);
    }
    return launch_status();
}
