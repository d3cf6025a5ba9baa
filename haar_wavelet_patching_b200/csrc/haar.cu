// Two-level causal full-packet Haar patcher and unpatcher for sm_100a.
//
// Sources: "NVIDIA Cosmos Tokenizer 完全指南", section 7.1 (Patcher, Patcher3D,
// UnPatcher, UnPatcher3D; taps 1/sqrt(2); c -> 4c / 8c per level; frame 0
// repeated; patch_size=4 = two levels), sections 6.1 and 7.3 (t = 1 + (T-1)/4);
// "nvidia/Cosmos-Tokenize1-CV8x8x8-720p" model card, Model Architecture.
//
// Kernel design.  The two levels are not run as two passes: along one axis,
// two full-packet levels on four samples are the 4-point Walsh-Hadamard
// transform (coefficient k = 2*b2 + b1 equals (1/2) sum_n (-1)^popcount(k&n) x_n),
// and the two frame-0 replicas compose into "output frame 0 reads four copies of
// frame 0, output frame t' >= 1 reads frames 4t'-3 .. 4t'".  So every 4x4x4 block
// of the clip maps to one value in each of 64C channel planes, with +-1
// butterflies in fp32 and one exact scale by 1/8 (1/4 in 2D).  The
// transform is its own inverse up to that scale, so the unpatcher runs the same
// butterflies; its output frame 0 is sample 3 of window 0 (the replicas are
// dropped level by level, which keeps the last copy).
//
// This file holds the register kernels, taken when the TMA path of haar_tma.cu
// cannot be (rows not a multiple of 16 bytes, or pointers not 16-byte aligned).
//
// Memory: the path moves each input byte and each output byte once and does
// ~7 flops per element, so it is bound by HBM.  A thread owns NB horizontally
// adjacent blocks: it reads 16 (3D) or 4 (2D) input rows of 4*NB contiguous
// elements (one or two 16-byte loads per row; a warp covers 512 contiguous
// bytes per row) and writes NB contiguous elements to each of the 64C (16C)
// channel planes (a warp covers 32*NB contiguous elements per plane).  All
// arithmetic stays in registers; nothing is staged through shared memory.
#include "tok_common.cuh"
#include "tok_internal.h"

namespace tok {
namespace {

// One axis of the two-level transform, unnormalized, in place (natural order).
__device__ __forceinline__ void haar4(float &a0, float &a1, float &a2, float &a3)
{
    const float l0 = a0 + a1, h0 = a0 - a1, l1 = a2 + a3, h1 = a2 - a3; // level 1
    a0 = l0 + l1;                                                        // k = 0: low, low
    a1 = h0 + h1;                                                        // k = 1: level-1 high
    a2 = l0 - l1;                                                        // k = 2: level-2 high
    a3 = h0 - h1;                                                        // k = 3: high, high
}

// Output channel group (in units of C) of the coefficient with per-axis index k.
// s_l = 4*bt_l + 2*by_l + bx_l; channel group = 8*s2 + s1 (2D: 4*s2 + s1).
__host__ __device__ constexpr int group3d(int kt, int ky, int kx)
{
    return 8 * (4 * (kt >> 1) + 2 * (ky >> 1) + (kx >> 1)) + (4 * (kt & 1) + 2 * (ky & 1) + (kx & 1));
}
__host__ __device__ constexpr int group2d(int ky, int kx)
{
    return 4 * (2 * (ky >> 1) + (kx >> 1)) + (2 * (ky & 1) + (kx & 1));
}

// Per-axis indices of channel group g (the inverse of group3d / group2d), so the
// kernels can walk the channel planes in address order with one pointer.
__host__ __device__ constexpr int kt_of(int g) { return 2 * ((g >> 3) >> 2) + ((g & 7) >> 2); }
__host__ __device__ constexpr int ky_of(int g) { return 2 * (((g >> 3) >> 1) & 1) + (((g & 7) >> 1) & 1); }
__host__ __device__ constexpr int kx_of(int g) { return 2 * ((g >> 3) & 1) + (g & 1); }
__host__ __device__ constexpr int ky2_of(int g) { return 2 * ((g >> 2) >> 1) + ((g & 3) >> 1); }
__host__ __device__ constexpr int kx2_of(int g) { return 2 * ((g >> 2) & 1) + (g & 1); }
static_assert(group3d(kt_of(37), ky_of(37), kx_of(37)) == 37, "group3d inverse");
static_assert(group2d(ky2_of(13), kx2_of(13)) == 13, "group2d inverse");

constexpr int kThreads = 64; // small CTAs: more resident warps per SM measured faster on B200

struct Geometry {
    int64_t BC;       // B*C (plane pairs)
    int64_t C;        // input channels
    int64_t T, H, W;  // pixel extents
    int64_t Tq, h, w; // latent extents
    int64_t tq0, nq;  // latent frames processed: [tq0, tq0 + nq)
    int64_t wn;       // thread columns per row = w / NB
};

// ---------------------------------------------------------------------------
// Forward, video: x [B,C,T,H,W] -> y [B,64C,Tq,h,w].
// grid.x covers the (i, jn) items of one latent frame, grid.y the latent frame,
// grid.z the (b, c) pair; y and z loop when the grid is capped.
// ---------------------------------------------------------------------------
// ADJ: the unpatcher's adjoint (window 0 takes (0, 0, 0, frame 0) in time).
template <typename T, int NB, bool VEC, bool ADJ>
__global__ void __launch_bounds__(kThreads) haar3d_fwd_kernel(const T *__restrict__ x, T *__restrict__ y, Geometry g)
{
    const int64_t item = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (item >= g.h * g.wn)
        return;
    const int64_t i = item / g.wn;
    const int64_t j0 = (item - i * g.wn) * NB;
    const int64_t plane_in = g.H * g.W, plane_out = g.Tq * g.h * g.w;
    const int64_t pair = (int64_t)blockIdx.z * gridDim.y + blockIdx.y; // (b, c, t')
    if (pair >= g.BC * g.nq)
        return;
    const int64_t bc = pair / g.nq, tq = g.tq0 + (pair - bc * g.nq);
    const int64_t b = bc / g.C, c = bc - b * g.C;
    const T *xc = x + bc * g.T * plane_in + (4 * i) * g.W + 4 * j0;
    T *yc = y + (b * 64 * g.C + c) * plane_out + i * g.w + j0;
    {
        {
            float v[NB][4][4][4]; // [block][t][y][x]
            if (tq == 0) {
                // Output frame 0 reads frame 0 four times (the adjoint: once, as the last sample).
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    float row[4 * NB];
                    Row<T, 4 * NB, VEC>::load(xc + r * g.W, row);
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                        for (int d = 0; d < 4; ++d) {
                            const float s = row[4 * nb + d];
                            v[nb][0][r][d] = ADJ ? 0.0f : s;
                            v[nb][1][r][d] = ADJ ? 0.0f : s;
                            v[nb][2][r][d] = ADJ ? 0.0f : s;
                            v[nb][3][r][d] = s;
                        }
                }
            } else {
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        float row[4 * NB];
                        Row<T, 4 * NB, VEC>::load(xc + (4 * tq - 3 + a) * plane_in + r * g.W, row);
#pragma unroll
                        for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                            for (int d = 0; d < 4; ++d)
                                v[nb][a][r][d] = row[4 * nb + d];
                    }
            }
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        haar4(v[nb][a][r][0], v[nb][a][r][1], v[nb][a][r][2], v[nb][a][r][3]);
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int d = 0; d < 4; ++d)
                        haar4(v[nb][a][0][d], v[nb][a][1][d], v[nb][a][2][d], v[nb][a][3][d]);
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int d = 0; d < 4; ++d)
                        haar4(v[nb][0][r][d], v[nb][1][r][d], v[nb][2][r][d], v[nb][3][r][d]);
            }
            T *yp = yc + tq * g.h * g.w;
            const int64_t cstride = g.C * plane_out;
#pragma unroll
            for (int grp = 0; grp < 64; ++grp, yp += cstride) {
                float o[NB];
#pragma unroll
                for (int nb = 0; nb < NB; ++nb)
                    o[nb] = v[nb][kt_of(grp)][ky_of(grp)][kx_of(grp)] * 0.125f;
                Row<T, NB, VEC>::store(yp, o);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Inverse, video: y [B,64C,Tq,h,w] -> x [B,C,T,H,W].
// ---------------------------------------------------------------------------
// ADJ: the patcher's adjoint (frame 0 receives the sum of window 0's four rebuilt frames).
template <typename T, int NB, bool VEC, bool ADJ>
__global__ void __launch_bounds__(kThreads) haar3d_inv_kernel(const T *__restrict__ y, T *__restrict__ x, Geometry g)
{
    const int64_t item = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (item >= g.h * g.wn)
        return;
    const int64_t i = item / g.wn;
    const int64_t j0 = (item - i * g.wn) * NB;
    const int64_t plane_in = g.Tq * g.h * g.w, plane_out = g.H * g.W;
    const int64_t pair = (int64_t)blockIdx.z * gridDim.y + blockIdx.y; // (b, c, t')
    if (pair >= g.BC * g.nq)
        return;
    const int64_t bc = pair / g.nq, tq = g.tq0 + (pair - bc * g.nq);
    const int64_t b = bc / g.C, c = bc - b * g.C;
    const T *yc = y + (b * 64 * g.C + c) * plane_in + i * g.w + j0;
    T *xc = x + bc * g.T * plane_out + (4 * i) * g.W + 4 * j0;
    {
        {
            float v[NB][4][4][4]; // [block][kt][ky][kx] -> [block][t][y][x]
            const T *yp = yc + tq * g.h * g.w;
            const int64_t cstride = g.C * plane_in;
#pragma unroll
            for (int grp = 0; grp < 64; ++grp, yp += cstride) {
                float in[NB];
                Row<T, NB, VEC>::load(yp, in);
#pragma unroll
                for (int nb = 0; nb < NB; ++nb)
                    v[nb][kt_of(grp)][ky_of(grp)][kx_of(grp)] = in[nb];
            }
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        haar4(v[nb][a][r][0], v[nb][a][r][1], v[nb][a][r][2], v[nb][a][r][3]);
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int d = 0; d < 4; ++d)
                        haar4(v[nb][a][0][d], v[nb][a][1][d], v[nb][a][2][d], v[nb][a][3][d]);
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int d = 0; d < 4; ++d)
                        haar4(v[nb][0][r][d], v[nb][1][r][d], v[nb][2][r][d], v[nb][3][r][d]);
            }
            // Window 0 rebuilds frame 0 as its last sample; window t' >= 1 rebuilds frames 4t'-3 .. 4t'.
            if (ADJ && tq == 0) {
#pragma unroll
                for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                    for (int r = 0; r < 4; ++r)
#pragma unroll
                        for (int d = 0; d < 4; ++d)
                            v[nb][3][r][d] = ((v[nb][0][r][d] + v[nb][1][r][d]) + v[nb][2][r][d]) + v[nb][3][r][d];
            }
            const int a_first = (tq == 0) ? 3 : 0;
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                if (a < a_first)
                    continue;
                const int64_t f = (tq == 0) ? 0 : 4 * tq - 3 + a;
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    float row[4 * NB];
#pragma unroll
                    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                        for (int d = 0; d < 4; ++d)
                            row[4 * nb + d] = v[nb][a][r][d] * 0.125f;
                    Row<T, 4 * NB, VEC>::store(xc + f * plane_out + r * g.W, row);
                }
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Image path (T == 1): x [B,C,1,H,W] <-> y [B,16C,1,h,w].
// ---------------------------------------------------------------------------
template <typename T, int NB, bool VEC>
__global__ void __launch_bounds__(kThreads) haar2d_fwd_kernel(const T *__restrict__ x, T *__restrict__ y, Geometry g)
{
    const int64_t item = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (item >= g.h * g.wn)
        return;
    const int64_t i = item / g.wn;
    const int64_t j0 = (item - i * g.wn) * NB;
    const int64_t plane_out = g.h * g.w;
    const int64_t bc = (int64_t)blockIdx.z * gridDim.y + blockIdx.y;
    if (bc >= g.BC)
        return;
    {
        const int64_t b = bc / g.C, c = bc - b * g.C;
        const T *xc = x + bc * g.H * g.W + (4 * i) * g.W + 4 * j0;
        T *yc = y + (b * 16 * g.C + c) * plane_out + i * g.w + j0;
        float v[NB][4][4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float row[4 * NB];
            Row<T, 4 * NB, VEC>::load(xc + r * g.W, row);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int d = 0; d < 4; ++d)
                    v[nb][r][d] = row[4 * nb + d];
        }
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
                haar4(v[nb][r][0], v[nb][r][1], v[nb][r][2], v[nb][r][3]);
#pragma unroll
            for (int d = 0; d < 4; ++d)
                haar4(v[nb][0][d], v[nb][1][d], v[nb][2][d], v[nb][3][d]);
        }
        T *yp = yc;
        const int64_t cstride = g.C * plane_out;
#pragma unroll
        for (int grp = 0; grp < 16; ++grp, yp += cstride) {
            float o[NB];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
                o[nb] = v[nb][ky2_of(grp)][kx2_of(grp)] * 0.25f;
            Row<T, NB, VEC>::store(yp, o);
        }
    }
}

template <typename T, int NB, bool VEC>
__global__ void __launch_bounds__(kThreads) haar2d_inv_kernel(const T *__restrict__ y, T *__restrict__ x, Geometry g)
{
    const int64_t item = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (item >= g.h * g.wn)
        return;
    const int64_t i = item / g.wn;
    const int64_t j0 = (item - i * g.wn) * NB;
    const int64_t plane_in = g.h * g.w;
    const int64_t bc = (int64_t)blockIdx.z * gridDim.y + blockIdx.y;
    if (bc >= g.BC)
        return;
    {
        const int64_t b = bc / g.C, c = bc - b * g.C;
        const T *yc = y + (b * 16 * g.C + c) * plane_in + i * g.w + j0;
        T *xc = x + bc * g.H * g.W + (4 * i) * g.W + 4 * j0;
        float v[NB][4][4];
        const T *yp = yc;
        const int64_t cstride = g.C * plane_in;
#pragma unroll
        for (int grp = 0; grp < 16; ++grp, yp += cstride) {
            float in[NB];
            Row<T, NB, VEC>::load(yp, in);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
                v[nb][ky2_of(grp)][kx2_of(grp)] = in[nb];
        }
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
#pragma unroll
            for (int r = 0; r < 4; ++r)
                haar4(v[nb][r][0], v[nb][r][1], v[nb][r][2], v[nb][r][3]);
#pragma unroll
            for (int d = 0; d < 4; ++d)
                haar4(v[nb][0][d], v[nb][1][d], v[nb][2][d], v[nb][3][d]);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            float row[4 * NB];
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
#pragma unroll
                for (int d = 0; d < 4; ++d)
                    row[4 * nb + d] = v[nb][r][d] * 0.25f;
            Row<T, 4 * NB, VEC>::store(xc + r * g.W, row);
        }
    }
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
constexpr int64_t kMaxGridYZ = 65535;

template <typename T, int NB, bool VEC, bool ADJ>
tok_status launch3d(bool fwd, const void *in, void *out, Geometry g, cudaStream_t stream)
{
    g.wn = g.w / NB;
    const int64_t gx = (g.h * g.wn + kThreads - 1) / kThreads;
    if (gx > 0x7FFFFFFF)
        return TOK_ERR_SHAPE;
    const int64_t pairs = g.BC * g.nq;
    const unsigned gy = (unsigned)(pairs < kMaxGridYZ ? pairs : kMaxGridYZ);
    const int64_t gz = (pairs + gy - 1) / gy;
    if (gz > kMaxGridYZ)
        return TOK_ERR_SHAPE;
    const dim3 grid((unsigned)gx, gy, (unsigned)gz);
    if (fwd)
        haar3d_fwd_kernel<T, NB, VEC, ADJ><<<grid, kThreads, 0, stream>>>((const T *)in, (T *)out, g);
    else
        haar3d_inv_kernel<T, NB, VEC, ADJ><<<grid, kThreads, 0, stream>>>((const T *)in, (T *)out, g);
    return launch_status();
}

template <typename T, int NB, bool VEC>
tok_status launch2d(bool fwd, const void *in, void *out, Geometry g, cudaStream_t stream)
{
    g.wn = g.w / NB;
    const int64_t gx = (g.h * g.wn + kThreads - 1) / kThreads;
    if (gx > 0x7FFFFFFF)
        return TOK_ERR_SHAPE;
    const unsigned gy = (unsigned)(g.BC < kMaxGridYZ ? g.BC : kMaxGridYZ);
    const int64_t gz = (g.BC + gy - 1) / gy;
    if (gz > kMaxGridYZ)
        return TOK_ERR_SHAPE;
    const dim3 grid((unsigned)gx, gy, (unsigned)gz);
    if (fwd)
        haar2d_fwd_kernel<T, NB, VEC><<<grid, kThreads, 0, stream>>>((const T *)in, (T *)out, g);
    else
        haar2d_inv_kernel<T, NB, VEC><<<grid, kThreads, 0, stream>>>((const T *)in, (T *)out, g);
    return launch_status();
}

// Latent frames [t_begin, t_end) of the full tensors; t_end < 0 means "through the last".
template <typename T, int NB, bool VEC>
tok_status launch3d_any(bool fwd, bool adj, const void *in, void *out, Geometry g, cudaStream_t stream)
{
    return adj ? launch3d<T, NB, VEC, true>(fwd, in, out, g, stream) : launch3d<T, NB, VEC, false>(fwd, in, out, g, stream);
}

// fwd: pixels -> coefficients.  adj: the adjoint variants (the gradient of the other
// direction's operation); on images the transform is orthogonal and adj changes nothing.
tok_status haar_call(bool fwd, bool adj, const void *in, void *out, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                     int64_t H, int64_t W, int64_t t_begin, int64_t t_end, cudaStream_t stream)
{
    if (dt != TOK_F32 && dt != TOK_BF16)
        return TOK_ERR_DTYPE;
    if (B < 0 || C < 0 || T < 1 || H < 0 || W < 0 || H % 4 || W % 4 || (T != 1 && T % 4 != 1))
        return TOK_ERR_SHAPE;
    const int64_t es = dt == TOK_F32 ? 4 : 2;
    Geometry g{};
    g.C = C;
    g.T = T;
    g.H = H;
    g.W = W;
    g.Tq = T == 1 ? 1 : 1 + (T - 1) / 4;
    g.h = H / 4;
    g.w = W / 4;
    if (t_end < 0)
        t_end = g.Tq;
    if (t_begin < 0 || t_begin > t_end || t_end > g.Tq)
        return TOK_ERR_SHAPE;
    g.tq0 = t_begin;
    g.nq = t_end - t_begin;
    int64_t nx, ny, bytes_x, bytes_y;
    if (!prod_ok({B, C}, &g.BC) || !prod_ok({g.BC, T, H, W}, &nx) || !prod_ok({nx, es}, &bytes_x) ||
        !prod_ok({g.BC, T == 1 ? 16 : 64, g.Tq, g.h, g.w}, &ny) || !prod_ok({ny, es}, &bytes_y))
        return TOK_ERR_SHAPE;
    if (nx == 0 || g.nq == 0)
        return TOK_OK;
    if (!in || !out)
        return TOK_ERR_NULL;
    if (!aligned(in, es) || !aligned(out, es))
        return TOK_ERR_ALIGN;
    const int64_t bytes_in = fwd ? bytes_x : bytes_y, bytes_out = fwd ? bytes_y : bytes_x;
    if (overlaps(in, bytes_in, out, bytes_out))
        return TOK_ERR_ALIAS;

    HaarDims dims{B, C, T, H, W, g.Tq, g.h, g.w, g.tq0, g.nq};
    dims.video = T > 1;
    const HaarTmaForm form = haar_tma_form(fwd, in, out, dt, dims);
    if (form != HaarTmaForm::none)
        return haar_tma_launch(fwd, adj, form, in, out, dt, dims, stream);

    // Register path: any 4-aligned W and element-aligned pointers.
    const bool a16 = aligned(in, 16) && aligned(out, 16);
    if (T > 1) {
        // Two adjacent blocks per thread: 8 input elements per row, pairs per plane.
        const bool vec = a16 && W % 8 == 0;
        if (dt == TOK_BF16)
            return vec ? launch3d_any<__nv_bfloat16, 2, true>(fwd, adj, in, out, g, stream)
                       : launch3d_any<__nv_bfloat16, 1, false>(fwd, adj, in, out, g, stream);
        return vec ? launch3d_any<float, 2, true>(fwd, adj, in, out, g, stream)
                   : launch3d_any<float, 1, false>(fwd, adj, in, out, g, stream);
    }
    // Image path: four adjacent blocks per thread: 16 input elements per row, quads per plane.
    const bool vec = a16 && W % 16 == 0;
    if (dt == TOK_BF16)
        return vec ? launch2d<__nv_bfloat16, 4, true>(fwd, in, out, g, stream)
                   : launch2d<__nv_bfloat16, 1, false>(fwd, in, out, g, stream);
    return vec ? launch2d<float, 4, true>(fwd, in, out, g, stream) : launch2d<float, 1, false>(fwd, in, out, g, stream);
}

// ---------------------------------------------------------------------------
// Extended form, register path: padding / cropping and streaming chunks for the
// shapes the TMA path cannot take (rows not a multiple of 16 bytes, unaligned
// pointers).  One thread per block; element loads with bounds (zeros past the
// pixel tensor's rows and columns, frames mirrored past its last frame) and
// element stores with bounds (the inverse crops).  Same butterflies and order.
// ---------------------------------------------------------------------------
struct ExtGeometry {
    int64_t BC, C;
    int64_t T, H, W;  // pixel tensor
    int64_t Tq, h, w; // latent tensor
    int64_t fbase;    // first frame of window tq (not the replica window): 4*tq + fbase
    int rep;          // window 0 is the frame-0 replica window
};

__device__ __forceinline__ int64_t mirror_frame_ext(int64_t f, int64_t T)
{
    if (f < T)
        return f;
    if (T == 1)
        return 0;
    const int64_t period = 2 * (T - 1), r = f % period;
    return r < T ? r : period - r;
}

template <typename T> __device__ __forceinline__ float elem_to_f(T v);
template <> __device__ __forceinline__ float elem_to_f<float>(float v) { return v; }
template <> __device__ __forceinline__ float elem_to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T f_to_elem(float v);
template <> __device__ __forceinline__ float f_to_elem<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 f_to_elem<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

template <typename T, bool VIDEO, bool FWD>
__global__ void __launch_bounds__(kThreads) haar_ext_kernel(const T *__restrict__ in, T *__restrict__ out, ExtGeometry g)
{
    constexpr int NA = VIDEO ? 4 : 1, G = VIDEO ? 64 : 16;
    constexpr float SCALE = VIDEO ? 0.125f : 0.25f;
    const int64_t item = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (item >= g.h * g.w)
        return;
    const int64_t i = item / g.w, j = item - i * g.w;
    const int64_t pair = (int64_t)blockIdx.z * gridDim.y + blockIdx.y; // (b, c, t')
    if (pair >= g.BC * g.Tq)
        return;
    const int64_t bc = pair / g.Tq, tq = pair - bc * g.Tq;
    const int64_t b = bc / g.C, c = bc - b * g.C;
    const bool replica = VIDEO && g.rep && tq == 0;
    const int64_t plane_lat = g.Tq * g.h * g.w, cstride = g.C * plane_lat;
    const int64_t lat0 = (b * G * g.C + c) * plane_lat + (tq * g.h + i) * g.w + j;

    float v[NA][4][4];
    if constexpr (FWD) {
#pragma unroll
        for (int a = 0; a < NA; ++a) {
            const int64_t f = !VIDEO ? 0 : replica ? 0 : mirror_frame_ext(4 * tq + g.fbase + a, g.T);
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int d = 0; d < 4; ++d) {
                    const int64_t yy = 4 * i + r, xx = 4 * j + d;
                    v[a][r][d] = (yy < g.H && xx < g.W) ? elem_to_f(in[((bc * g.T + f) * g.H + yy) * g.W + xx]) : 0.0f;
                }
        }
    } else {
#pragma unroll
        for (int grp = 0; grp < G; ++grp) {
            const float p = elem_to_f(in[lat0 + grp * cstride]);
            if constexpr (VIDEO)
                v[kt_of(grp)][ky_of(grp)][kx_of(grp)] = p;
            else
                v[0][ky2_of(grp)][kx2_of(grp)] = p;
        }
    }
#pragma unroll
    for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int r = 0; r < 4; ++r)
            haar4(v[a][r][0], v[a][r][1], v[a][r][2], v[a][r][3]);
#pragma unroll
    for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int d = 0; d < 4; ++d)
            haar4(v[a][0][d], v[a][1][d], v[a][2][d], v[a][3][d]);
    if constexpr (VIDEO) {
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int d = 0; d < 4; ++d)
                haar4(v[0][r][d], v[1][r][d], v[2][r][d], v[3][r][d]);
    }
    if constexpr (FWD) {
#pragma unroll
        for (int grp = 0; grp < G; ++grp) {
            const float p = VIDEO ? v[kt_of(grp)][ky_of(grp)][kx_of(grp)] : v[0][ky2_of(grp)][kx2_of(grp)];
            out[lat0 + grp * cstride] = f_to_elem<T>(p * SCALE);
        }
    } else {
#pragma unroll
        for (int a = 0; a < NA; ++a) {
            if (replica && a != 3)
                continue;
            const int64_t f = !VIDEO ? 0 : replica ? 0 : 4 * tq + g.fbase + a;
            if (f >= g.T)
                continue;
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int d = 0; d < 4; ++d) {
                    const int64_t yy = 4 * i + r, xx = 4 * j + d;
                    if (yy < g.H && xx < g.W)
                        out[((bc * g.T + f) * g.H + yy) * g.W + xx] = f_to_elem<T>(v[a][r][d] * SCALE);
                }
        }
    }
}

template <typename T, bool VIDEO, bool FWD>
tok_status launch_ext(const void *in, void *out, const ExtGeometry &g, cudaStream_t stream)
{
    const int64_t items = g.h * g.w, pairs = g.BC * g.Tq;
    const int64_t gy = pairs < 65535 ? pairs : 65535, gz = (pairs + gy - 1) / gy;
    if ((items + kThreads - 1) / kThreads > 0x7FFFFFFF || gz > 65535)
        return TOK_ERR_SHAPE;
    const dim3 grid((unsigned)((items + kThreads - 1) / kThreads), (unsigned)gy, (unsigned)gz);
    haar_ext_kernel<T, VIDEO, FWD><<<grid, kThreads, 0, stream>>>((const T *)in, (T *)out, g);
    return launch_status();
}

// Extended call: pixels [B, C, T, H, W] <-> coefficients [B, G*C, Tq, Hp/4, Wp/4] with
// (Tp, Hp, Wp) the padded extents, windows as described for ExtGeometry.
tok_status haar_ext_call(bool fwd, const void *in, void *out, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                         int64_t H, int64_t W, int64_t Tp, int64_t Hp, int64_t Wp, int64_t fbase, int rep, bool video,
                         cudaStream_t stream)
{
    if (dt != TOK_F32 && dt != TOK_BF16)
        return TOK_ERR_DTYPE;
    const int64_t es = dt == TOK_F32 ? 4 : 2;
    ExtGeometry g{};
    g.C = C;
    g.T = T;
    g.H = H;
    g.W = W;
    g.Tq = !video ? 1 : rep ? 1 + (Tp - 1) / 4 : Tp / 4;
    g.h = Hp / 4;
    g.w = Wp / 4;
    g.fbase = fbase;
    g.rep = rep;
    int64_t nx, ny, bytes_x, bytes_y;
    if (!prod_ok({B, C}, &g.BC) || !prod_ok({g.BC, T, H, W}, &nx) || !prod_ok({nx, es}, &bytes_x) ||
        !prod_ok({g.BC, video ? 64 : 16, g.Tq, g.h, g.w}, &ny) || !prod_ok({ny, es}, &bytes_y))
        return TOK_ERR_SHAPE;
    if (nx == 0 || ny == 0)
        return TOK_OK;
    if (!in || !out)
        return TOK_ERR_NULL;
    if (!aligned(in, es) || !aligned(out, es))
        return TOK_ERR_ALIGN;
    const int64_t bytes_in = fwd ? bytes_x : bytes_y, bytes_out = fwd ? bytes_y : bytes_x;
    if (overlaps(in, bytes_in, out, bytes_out))
        return TOK_ERR_ALIAS;

    HaarDims dims{B, C, T, H, W, g.Tq, g.h, g.w, 0, g.Tq};
    dims.fbase = fbase;
    dims.rep = rep;
    dims.video = video;
    // The extended form only where frames, rows or columns are padded or cropped: a chunk, or a
    // clip that needs no padding, takes the plain forms with its window rule (fbase, rep).
    dims.ext = Tp != T || Hp != H || Wp != W;
    const HaarTmaForm form = haar_tma_form(fwd, in, out, dt, dims);
    if (form != HaarTmaForm::none)
        return haar_tma_launch(fwd, false, form, in, out, dt, dims, stream);
    if (dt == TOK_BF16) {
        using B16 = __nv_bfloat16;
        if (video)
            return fwd ? launch_ext<B16, true, true>(in, out, g, stream) : launch_ext<B16, true, false>(in, out, g, stream);
        return fwd ? launch_ext<B16, false, true>(in, out, g, stream) : launch_ext<B16, false, false>(in, out, g, stream);
    }
    if (video)
        return fwd ? launch_ext<float, true, true>(in, out, g, stream) : launch_ext<float, true, false>(in, out, g, stream);
    return fwd ? launch_ext<float, false, true>(in, out, g, stream) : launch_ext<float, false, false>(in, out, g, stream);
}

// ---------------------------------------------------------------------------
// Single level (patch_size=2), register path for shapes the TMA kernel cannot take:
// one thread per 2x2x2 block (2x2 on images), element loads and stores.
// ---------------------------------------------------------------------------
struct SingleGeometry {
    int64_t BC, C, T, H, W, Tq, h, w;
};

template <typename T, bool VIDEO, bool FWD>
__global__ void __launch_bounds__(kThreads)
    haar_single_reg_kernel(const T *__restrict__ in, T *__restrict__ out, SingleGeometry g)
{
    constexpr int NA = VIDEO ? 2 : 1, G = VIDEO ? 8 : 4;
    constexpr float SCALE = VIDEO ? 0.353553390593273762f : 0.5f;
    const int64_t item = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (item >= g.h * g.w)
        return;
    const int64_t i = item / g.w, j = item - i * g.w;
    const int64_t pair = (int64_t)blockIdx.z * gridDim.y + blockIdx.y;
    if (pair >= g.BC * g.Tq)
        return;
    const int64_t bc = pair / g.Tq, tq = pair - bc * g.Tq;
    const int64_t b = bc / g.C, c = bc - b * g.C;
    const bool replica = VIDEO && tq == 0;
    const int64_t plane = g.Tq * g.h * g.w, cstride = g.C * plane;
    const int64_t lat0 = (b * G * g.C + c) * plane + (tq * g.h + i) * g.w + j;
    float v[NA][2][2];
    if constexpr (FWD) {
#pragma unroll
        for (int a = 0; a < NA; ++a) {
            const int64_t f = !VIDEO ? 0 : replica ? 0 : 2 * tq - 1 + a;
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int d = 0; d < 2; ++d)
                    v[a][r][d] = elem_to_f(in[((bc * g.T + f) * g.H + 2 * i + r) * g.W + 2 * j + d]);
        }
    } else {
#pragma unroll
        for (int grp = 0; grp < G; ++grp) {
            const float p = elem_to_f(in[lat0 + grp * cstride]);
            if constexpr (VIDEO)
                v[grp >> 2][(grp >> 1) & 1][grp & 1] = p;
            else
                v[0][grp >> 1][grp & 1] = p;
        }
    }
#pragma unroll
    for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const float l = v[a][r][0] + v[a][r][1], hgh = v[a][r][0] - v[a][r][1];
            v[a][r][0] = l, v[a][r][1] = hgh;
        }
#pragma unroll
    for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int d = 0; d < 2; ++d) {
            const float l = v[a][0][d] + v[a][1][d], hgh = v[a][0][d] - v[a][1][d];
            v[a][0][d] = l, v[a][1][d] = hgh;
        }
    if constexpr (VIDEO) {
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int d = 0; d < 2; ++d) {
                const float l = v[0][r][d] + v[1][r][d], hgh = v[0][r][d] - v[1][r][d];
                v[0][r][d] = l, v[1][r][d] = hgh;
            }
    }
    if constexpr (FWD) {
#pragma unroll
        for (int grp = 0; grp < G; ++grp) {
            const float p = VIDEO ? v[grp >> 2][(grp >> 1) & 1][grp & 1] : v[0][grp >> 1][grp & 1];
            out[lat0 + grp * cstride] = f_to_elem<T>(p * SCALE);
        }
    } else {
#pragma unroll
        for (int a = 0; a < NA; ++a) {
            if (replica && a != 1)
                continue;
            const int64_t f = !VIDEO ? 0 : replica ? 0 : 2 * tq - 1 + a;
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
                for (int d = 0; d < 2; ++d)
                    out[((bc * g.T + f) * g.H + 2 * i + r) * g.W + 2 * j + d] = f_to_elem<T>(v[a][r][d] * SCALE);
        }
    }
}

template <typename T, bool VIDEO, bool FWD>
tok_status launch_single_reg(const void *in, void *out, const SingleGeometry &g, cudaStream_t stream)
{
    const int64_t items = g.h * g.w, pairs = g.BC * g.Tq;
    const int64_t gy = pairs < 65535 ? pairs : 65535, gz = (pairs + gy - 1) / gy;
    if ((items + kThreads - 1) / kThreads > 0x7FFFFFFF || gz > 65535)
        return TOK_ERR_SHAPE;
    const dim3 grid((unsigned)((items + kThreads - 1) / kThreads), (unsigned)gy, (unsigned)gz);
    haar_single_reg_kernel<T, VIDEO, FWD><<<grid, kThreads, 0, stream>>>((const T *)in, (T *)out, g);
    return launch_status();
}

tok_status single_call(bool fwd, const void *in, void *out, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                       int64_t H, int64_t W, cudaStream_t stream)
{
    if (dt != TOK_F32 && dt != TOK_BF16)
        return TOK_ERR_DTYPE;
    if (B < 0 || C < 0 || T < 1 || H < 0 || W < 0 || H % 2 || W % 2 || (T != 1 && T % 2 == 0))
        return TOK_ERR_SHAPE;
    const bool video = T > 1;
    const int64_t es = dt == TOK_F32 ? 4 : 2;
    SingleGeometry g{};
    g.C = C;
    g.T = T;
    g.H = H;
    g.W = W;
    g.Tq = video ? (T + 1) / 2 : 1;
    g.h = H / 2;
    g.w = W / 2;
    int64_t nx, ny, bytes_x, bytes_y;
    if (!prod_ok({B, C}, &g.BC) || !prod_ok({g.BC, T, H, W}, &nx) || !prod_ok({nx, es}, &bytes_x) ||
        !prod_ok({g.BC, video ? 8 : 4, g.Tq, g.h, g.w}, &ny) || !prod_ok({ny, es}, &bytes_y))
        return TOK_ERR_SHAPE;
    if (nx == 0)
        return TOK_OK;
    if (!in || !out)
        return TOK_ERR_NULL;
    if (!aligned(in, es) || !aligned(out, es))
        return TOK_ERR_ALIGN;
    if (overlaps(in, fwd ? bytes_x : bytes_y, out, fwd ? bytes_y : bytes_x))
        return TOK_ERR_ALIAS;
    HaarDims dims{B, C, T, H, W, g.Tq, g.h, g.w, 0, g.Tq};
    dims.video = video;
    const HaarTmaForm form = haar_single_tma_form(fwd, in, out, dt, dims);
    if (form != HaarTmaForm::none)
        return haar_single_tma_launch(fwd, form, in, out, dt, dims, stream);
    if (dt == TOK_BF16) {
        using B16 = __nv_bfloat16;
        if (video)
            return fwd ? launch_single_reg<B16, true, true>(in, out, g, stream)
                       : launch_single_reg<B16, true, false>(in, out, g, stream);
        return fwd ? launch_single_reg<B16, false, true>(in, out, g, stream)
                   : launch_single_reg<B16, false, false>(in, out, g, stream);
    }
    if (video)
        return fwd ? launch_single_reg<float, true, true>(in, out, g, stream)
                   : launch_single_reg<float, true, false>(in, out, g, stream);
    return fwd ? launch_single_reg<float, false, true>(in, out, g, stream)
               : launch_single_reg<float, false, false>(in, out, g, stream);
}

// ---------------------------------------------------------------------------
// Channels-last two-level patcher, register path (any C, shapes the TMA kernel
// cannot take): one thread per block of one (b, c, t'); element loads, the 64 (16)
// results stored at y[b][t'][i][j][g*C + c].
// ---------------------------------------------------------------------------
template <typename T, bool VIDEO>
__global__ void __launch_bounds__(kThreads) haar_cl_reg_kernel(const T *__restrict__ x, T *__restrict__ y, Geometry g)
{
    constexpr int NA = VIDEO ? 4 : 1, G = VIDEO ? 64 : 16;
    constexpr float SCALE = VIDEO ? 0.125f : 0.25f;
    const int64_t item = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    if (item >= g.h * g.w)
        return;
    const int64_t i = item / g.w, j = item - i * g.w;
    const int64_t pair = (int64_t)blockIdx.z * gridDim.y + blockIdx.y;
    if (pair >= g.BC * g.Tq)
        return;
    const int64_t bc = pair / g.Tq, tq = pair - bc * g.Tq;
    const int64_t b = bc / g.C, c = bc - b * g.C;
    float v[NA][4][4];
#pragma unroll
    for (int a = 0; a < NA; ++a) {
        const int64_t f = (!VIDEO || tq == 0) ? 0 : 4 * tq - 3 + a;
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int d = 0; d < 4; ++d)
                v[a][r][d] = elem_to_f(x[((bc * g.T + f) * g.H + 4 * i + r) * g.W + 4 * j + d]);
    }
#pragma unroll
    for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int r = 0; r < 4; ++r)
            haar4(v[a][r][0], v[a][r][1], v[a][r][2], v[a][r][3]);
#pragma unroll
    for (int a = 0; a < NA; ++a)
#pragma unroll
        for (int d = 0; d < 4; ++d)
            haar4(v[a][0][d], v[a][1][d], v[a][2][d], v[a][3][d]);
    if constexpr (VIDEO) {
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
            for (int d = 0; d < 4; ++d)
                haar4(v[0][r][d], v[1][r][d], v[2][r][d], v[3][r][d]);
    }
    T *yb = y + (((b * g.Tq + tq) * g.h + i) * g.w + j) * G * g.C + c;
#pragma unroll
    for (int grp = 0; grp < G; ++grp) {
        const float p = VIDEO ? v[kt_of(grp)][ky_of(grp)][kx_of(grp)] : v[0][ky2_of(grp)][kx2_of(grp)];
        yb[grp * g.C] = f_to_elem<T>(p * SCALE);
    }
}

tok_status channels_last_call(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C, int64_t T, int64_t H,
                              int64_t W, cudaStream_t stream)
{
    if (dt != TOK_F32 && dt != TOK_BF16)
        return TOK_ERR_DTYPE;
    if (B < 0 || C < 0 || T < 1 || H < 0 || W < 0 || H % 4 || W % 4 || (T != 1 && T % 4 != 1))
        return TOK_ERR_SHAPE;
    const bool video = T > 1;
    const int64_t es = dt == TOK_F32 ? 4 : 2;
    Geometry g{};
    g.C = C;
    g.T = T;
    g.H = H;
    g.W = W;
    g.Tq = video ? 1 + (T - 1) / 4 : 1;
    g.h = H / 4;
    g.w = W / 4;
    g.tq0 = 0;
    g.nq = g.Tq;
    int64_t nx, ny, bytes_x, bytes_y;
    if (!prod_ok({B, C}, &g.BC) || !prod_ok({g.BC, T, H, W}, &nx) || !prod_ok({nx, es}, &bytes_x) ||
        !prod_ok({g.BC, video ? 64 : 16, g.Tq, g.h, g.w}, &ny) || !prod_ok({ny, es}, &bytes_y))
        return TOK_ERR_SHAPE;
    if (nx == 0)
        return TOK_OK;
    if (!x || !y)
        return TOK_ERR_NULL;
    if (!aligned(x, es) || !aligned(y, es))
        return TOK_ERR_ALIGN;
    if (overlaps(x, bytes_x, y, bytes_y))
        return TOK_ERR_ALIAS;
    HaarDims dims{B, C, T, H, W, g.Tq, g.h, g.w, 0, g.Tq};
    dims.video = video;
    if (haar_cl_tma_eligible(x, y, dt, dims))
        return haar_cl_tma_launch(x, y, dt, dims, stream);
    const int64_t items = g.h * g.w, pairs = g.BC * g.Tq;
    const int64_t gy = pairs < 65535 ? pairs : 65535, gz = (pairs + gy - 1) / gy;
    if ((items + kThreads - 1) / kThreads > 0x7FFFFFFF || gz > 65535)
        return TOK_ERR_SHAPE;
    const dim3 grid((unsigned)((items + kThreads - 1) / kThreads), (unsigned)gy, (unsigned)gz);
    if (dt == TOK_BF16) {
        using B16 = __nv_bfloat16;
        if (video)
            haar_cl_reg_kernel<B16, true><<<grid, kThreads, 0, stream>>>((const B16 *)x, (B16 *)y, g);
        else
            haar_cl_reg_kernel<B16, false><<<grid, kThreads, 0, stream>>>((const B16 *)x, (B16 *)y, g);
    } else if (video) {
        haar_cl_reg_kernel<float, true><<<grid, kThreads, 0, stream>>>((const float *)x, (float *)y, g);
    } else {
        haar_cl_reg_kernel<float, false><<<grid, kThreads, 0, stream>>>((const float *)x, (float *)y, g);
    }
    return launch_status();
}

bool padded_extents(int64_t T, int64_t H, int64_t W, int64_t ms, int64_t mt, int64_t *Tp, int64_t *Hp, int64_t *Wp)
{
    if (T < 1 || H < 0 || W < 0 || ms < 4 || ms % 4 != 0 || mt < 4 || mt % 4 != 0)
        return false;
    if (H > ((int64_t)1 << 40) || W > ((int64_t)1 << 40) || T > ((int64_t)1 << 40) || ms > ((int64_t)1 << 20) ||
        mt > ((int64_t)1 << 20))
        return false;
    *Hp = (H + ms - 1) / ms * ms;
    *Wp = (W + ms - 1) / ms * ms;
    *Tp = T == 1 ? 1 : 1 + (T - 1 + mt - 1) / mt * mt;
    return true;
}

tok_status padded_call(bool fwd, const void *in, void *out, tok_dtype dt, int64_t B, int64_t C, int64_t T, int64_t H,
                       int64_t W, int64_t ms, int64_t mt, cudaStream_t stream)
{
    int64_t Tp, Hp, Wp;
    if (B < 0 || C < 0 || !padded_extents(T, H, W, ms, mt, &Tp, &Hp, &Wp))
        return TOK_ERR_SHAPE;
    return haar_ext_call(fwd, in, out, dt, B, C, T, H, W, Tp, Hp, Wp, -3, 1, T > 1, stream);
}

tok_status chunk_call(bool fwd, const void *in, void *out, tok_dtype dt, int64_t B, int64_t C, int64_t T, int64_t H,
                      int64_t W, int first, cudaStream_t stream)
{
    if (B < 0 || C < 0 || H < 0 || W < 0 || H % 4 || W % 4)
        return TOK_ERR_SHAPE;
    if (first ? (T < 1 || T % 4 != 1) : (T < 4 || T % 4 != 0))
        return TOK_ERR_SHAPE;
    return haar_ext_call(fwd, in, out, dt, B, C, T, H, W, T, H, W, first ? -3 : 0, first ? 1 : 0, true, stream);
}

} // namespace
} // namespace tok

extern "C" tok_status tok_haar_fwd(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C, int64_t T, int64_t H,
                                   int64_t W, cudaStream_t stream)
{
    return tok::haar_call(true, false, x, y, dt, B, C, T, H, W, 0, -1, stream);
}

extern "C" tok_status tok_haar_inv(const void *y, void *x, tok_dtype dt, int64_t B, int64_t C, int64_t T, int64_t H,
                                   int64_t W, cudaStream_t stream)
{
    return tok::haar_call(false, false, y, x, dt, B, C, T, H, W, 0, -1, stream);
}

extern "C" tok_status tok_haar_fwd_adjoint(const void *gy, void *gx, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                           int64_t H, int64_t W, cudaStream_t stream)
{
    return tok::haar_call(false, true, gy, gx, dt, B, C, T, H, W, 0, -1, stream);
}

extern "C" tok_status tok_haar_inv_adjoint(const void *gx, void *gy, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                           int64_t H, int64_t W, cudaStream_t stream)
{
    return tok::haar_call(true, true, gx, gy, dt, B, C, T, H, W, 0, -1, stream);
}

extern "C" tok_status tok_haar_fwd_windows(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                           int64_t H, int64_t W, int64_t t_begin, int64_t t_end, cudaStream_t stream)
{
    if (t_end < 0)
        return TOK_ERR_SHAPE;
    return tok::haar_call(true, false, x, y, dt, B, C, T, H, W, t_begin, t_end, stream);
}

extern "C" tok_status tok_haar_inv_windows(const void *y, void *x, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                           int64_t H, int64_t W, int64_t t_begin, int64_t t_end, cudaStream_t stream)
{
    if (t_end < 0)
        return TOK_ERR_SHAPE;
    return tok::haar_call(false, false, y, x, dt, B, C, T, H, W, t_begin, t_end, stream);
}

extern "C" tok_status tok_haar_padded_extents(int64_t T, int64_t H, int64_t W, int64_t spatial_multiple,
                                              int64_t temporal_multiple, int64_t *Tp, int64_t *Hp, int64_t *Wp)
{
    if (!Tp || !Hp || !Wp)
        return TOK_ERR_NULL;
    return tok::padded_extents(T, H, W, spatial_multiple, temporal_multiple, Tp, Hp, Wp) ? TOK_OK : TOK_ERR_SHAPE;
}

extern "C" tok_status tok_haar_fwd_padded(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                          int64_t H, int64_t W, int64_t spatial_multiple, int64_t temporal_multiple,
                                          cudaStream_t stream)
{
    return tok::padded_call(true, x, y, dt, B, C, T, H, W, spatial_multiple, temporal_multiple, stream);
}

extern "C" tok_status tok_haar_inv_cropped(const void *y, void *x, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                           int64_t H, int64_t W, int64_t spatial_multiple, int64_t temporal_multiple,
                                           cudaStream_t stream)
{
    return tok::padded_call(false, y, x, dt, B, C, T, H, W, spatial_multiple, temporal_multiple, stream);
}

extern "C" tok_status tok_haar_fwd_chunk(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                         int64_t H, int64_t W, int first, cudaStream_t stream)
{
    return tok::chunk_call(true, x, y, dt, B, C, T, H, W, first, stream);
}

extern "C" tok_status tok_haar_inv_chunk(const void *y, void *x, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                         int64_t H, int64_t W, int first, cudaStream_t stream)
{
    return tok::chunk_call(false, y, x, dt, B, C, T, H, W, first, stream);
}

extern "C" tok_status tok_haar_fwd_single(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                          int64_t H, int64_t W, cudaStream_t stream)
{
    return tok::single_call(true, x, y, dt, B, C, T, H, W, stream);
}

extern "C" tok_status tok_haar_inv_single(const void *y, void *x, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                          int64_t H, int64_t W, cudaStream_t stream)
{
    return tok::single_call(false, y, x, dt, B, C, T, H, W, stream);
}

extern "C" tok_status tok_haar_fwd_channels_last(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C,
                                                 int64_t T, int64_t H, int64_t W, cudaStream_t stream)
{
    return tok::channels_last_call(x, y, dt, B, C, T, H, W, stream);
}
