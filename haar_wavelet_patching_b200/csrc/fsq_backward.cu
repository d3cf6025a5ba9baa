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
#include <cmath>
#include <mutex>

#include "tok_common.cuh"
#include "tok_internal.h"

namespace tok {
namespace {

constexpr int kThreads = 128;
constexpr int kTokensPerCta = 2048; // 16 tokens per thread
constexpr int kMaxC = 16;           // channel count held in registers

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

__device__ __forceinline__ float sech2(float x)
{
    const float a = expf(-2.0f * fabsf(x));
    const float d = 1.0f + a;
    return 4.0f * a / (d * d);
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

bool shape_ok(int64_t B, int64_t C, int64_t S, int64_t *N)
{
    int64_t bytes;
    return B >= 0 && S >= 0 && C >= 1 && C <= kMaxC && prod_ok({B, S}, N) && prod_ok({*N, C, 4}, &bytes);
}

int64_t blocks_for(int64_t N) { return (N + kTokensPerCta - 1) / kTokensPerCta; }

} // namespace

int64_t fsq_backward_workspace_bytes(int64_t B, int64_t C, int64_t S)
{
    int64_t N;
    if (!shape_ok(B, C, S, &N))
        return -1;
    return blocks_for(N) * 6 * C * (int64_t)sizeof(float);
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
// loads the library holds it, 1.5 MB, until the process exits.
// ---------------------------------------------------------------------------
namespace tok {
namespace {

constexpr int64_t kNoAllocMaxRows = 4096; // token blocks: at most 4096 * 2048 = 8,388,608 tokens
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
    const int64_t rows = blocks_for(N);
    if (rows > kNoAllocMaxRows)
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
    if (rows > 0)
        fsq_encode_bwd_kernel<<<(unsigned)rows, kThreads, 0, stream>>>(u, w, grad_codes, grad_u, scratch, B, (int)C,
                                                                       S, slope_consts());
    fsq_bwd_sum_rows_kernel<<<(unsigned)(6 * C), kSumThreads, 0, stream>>>(scratch, rows, (int)(6 * C), grad_w);
    return launch_status();
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
    const int64_t rows = blocks_for(N);
    if (rows > 0x7FFFFFFF)
        return TOK_ERR_SHAPE;
    if (rows > 0)
        fsq_encode_bwd_kernel<<<(unsigned)rows, kThreads, 0, stream>>>(u, w, grad_codes, grad_u, (float *)workspace, B,
                                                                       (int)C, S, slope_consts());
    fsq_bwd_sum_rows_kernel<<<(unsigned)(6 * C), kSumThreads, 0, stream>>>((const float *)workspace, rows,
                                                                             (int)(6 * C), grad_w);
    return launch_status();
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
    const int64_t rows = blocks_for(N);
    if (rows > 0x7FFFFFFF)
        return TOK_ERR_SHAPE;
    if (rows > 0)
        fsq_decode_bwd_kernel<<<(unsigned)rows, kThreads, 0, stream>>>(idx, w, grad_out, grad_codes,
                                                                       (float *)workspace, B, (int)C, S);
    fsq_bwd_sum_rows_kernel<<<(unsigned)(6 * C), kSumThreads, 0, stream>>>((const float *)workspace, rows,
                                                                             (int)(6 * C), grad_w);
    return launch_status();
}
