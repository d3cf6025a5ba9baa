// TMA-pipelined Haar patcher / unpatcher for sm_100a (the main path).
//
// Same transform as haar.cu (sources: "NVIDIA Cosmos Tokenizer 完全指南" 7.1, 6.1,
// 7.3; "nvidia/Cosmos-Tokenize1-CV8x8x8-720p" model card, Model Architecture):
// every 4x4x4 pixel block maps to one coefficient in each of 64 channel groups
// through the per-axis 4-point transform of the two full-packet levels, with the
// two frame-0 replicas composed into "window 0 reads frame 0 four times".
//
// Design.  Work is cut into warp tiles of 64 horizontally adjacent blocks:
// one block row of one (b, c, t') window on video (4 frames x 4 rows x 256
// pixels <-> 64 planes x 64 coefficients), four block rows on images (4 x 16
// rows of 256 pixels <-> 16 planes x 4 x 64); 4096 elements either way.  Every
// warp of a persistent CTA runs its own pipeline, with no CTA-wide barrier:
//   - lane 0 keeps NI TMA loads in flight into the warp's input buffers (a 3D
//     box of pixels, or one 5D box holding all 64 coefficient planes); each
//     completes on that buffer's mbarrier;
//   - the lanes copy their values into registers, and lane 0 at once refills
//     the buffer with the tile NI steps ahead;
//   - the lanes transform, write the results to the warp's output buffer, and
//     lane 0 issues one TMA store for the whole tile.
// Each lane owns two horizontally adjacent blocks and keeps them in f32x2 pairs
// (block j in .x, block j+1 in .y), so every butterfly is one packed sm_100
// add or fused multiply-add.  TMA clips partial tiles at the tensor edges
// (zero fill on load, nothing stored out of bounds), so any w and h work.
//
// Waits are bounded: a barrier that does not complete within kWaitPolls polls
// makes the warp stop, drain what it issued and count a timeout that
// tok_check_device() reports.  No cluster multicast is used.
#include "tma.cuh"
#include "tok_common.cuh"
#include "tok_internal.h"

namespace tok {

// Kernels of this file that gave up on a barrier wait since the last check.
static __device__ unsigned int g_wait_timeouts = 0;

namespace {

constexpr int kTileBlocks = 64;        // blocks across a warp tile (256 pixels)
constexpr int kTileElems = 4096;       // elements of a warp tile, on either side
constexpr int kSmemBudget = 192 * 1024; // shared memory per CTA

template <typename T> struct WarpPipe {
    static constexpr int NI = sizeof(T) == 2 ? 3 : 2;              // input buffers per warp
    static constexpr int TILE_BYTES = kTileElems * sizeof(T);
    static constexpr int WARP_BYTES = (NI + 1) * TILE_BYTES + 64;   // + output buffer + barriers
    static constexpr int WARPS = kSmemBudget / WARP_BYTES;          // 6 (bf16) or 3 (fp32)
    static constexpr int SMEM = WARPS * WARP_BYTES;
};

struct TileGrid {
    int ntx, nty, Tq, C, T;
    int64_t ntiles;
};

__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
// a - b, exactly as a subtraction rounds (the product b * -1 is exact).
__device__ __forceinline__ float2 sub2(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a); }

// The two-level transform along one axis on four pairs, natural order (k = 2*b2 + b1).
__device__ __forceinline__ void haar4x2(float2 &a0, float2 &a1, float2 &a2, float2 &a3)
{
    const float2 l0 = add2(a0, a1), h0 = sub2(a0, a1), l1 = add2(a2, a3), h1 = sub2(a2, a3);
    a0 = add2(l0, l1);
    a1 = add2(h0, h1);
    a2 = sub2(l0, l1);
    a3 = sub2(h0, h1);
}

__host__ __device__ constexpr int kt_of(int g) { return 2 * ((g >> 3) >> 2) + ((g & 7) >> 2); }
__host__ __device__ constexpr int ky_of(int g) { return 2 * (((g >> 3) >> 1) & 1) + (((g & 7) >> 1) & 1); }
__host__ __device__ constexpr int kx_of(int g) { return 2 * ((g >> 3) & 1) + (g & 1); }
__host__ __device__ constexpr int ky2_of(int g) { return 2 * ((g >> 2) >> 1) + ((g & 3) >> 1); }
__host__ __device__ constexpr int kx2_of(int g) { return 2 * ((g >> 2) & 1) + (g & 1); }

// Shared-memory row of 8 elements (blocks j, j+1) <-> four pairs.
template <typename T> struct SRow;
template <> struct SRow<__nv_bfloat16> {
    static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float2 *v)
    {
        const uint4 r = *reinterpret_cast<const uint4 *>(p);
        v[0] = make_float2(bf16_lo(r.x), bf16_lo(r.z));
        v[1] = make_float2(bf16_hi(r.x), bf16_hi(r.z));
        v[2] = make_float2(bf16_lo(r.y), bf16_lo(r.w));
        v[3] = make_float2(bf16_hi(r.y), bf16_hi(r.w));
    }
    static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float2 *v)
    {
        *reinterpret_cast<uint4 *>(p) = make_uint4(pack_bf16x2(v[0].x, v[1].x), pack_bf16x2(v[2].x, v[3].x),
                                                   pack_bf16x2(v[0].y, v[1].y), pack_bf16x2(v[2].y, v[3].y));
    }
    static __device__ __forceinline__ float2 load_pair(const __nv_bfloat16 *p)
    {
        const uint32_t r = *reinterpret_cast<const uint32_t *>(p);
        return make_float2(bf16_lo(r), bf16_hi(r));
    }
    static __device__ __forceinline__ void store_pair(__nv_bfloat16 *p, float2 v)
    {
        *reinterpret_cast<uint32_t *>(p) = pack_bf16x2(v.x, v.y);
    }
};
template <> struct SRow<float> {
    static __device__ __forceinline__ void load(const float *p, float2 *v)
    {
        const float4 a = *reinterpret_cast<const float4 *>(p), b = *reinterpret_cast<const float4 *>(p + 4);
        v[0] = make_float2(a.x, b.x);
        v[1] = make_float2(a.y, b.y);
        v[2] = make_float2(a.z, b.z);
        v[3] = make_float2(a.w, b.w);
    }
    static __device__ __forceinline__ void store(float *p, const float2 *v)
    {
        *reinterpret_cast<float4 *>(p) = make_float4(v[0].x, v[1].x, v[2].x, v[3].x);
        *reinterpret_cast<float4 *>(p + 4) = make_float4(v[0].y, v[1].y, v[2].y, v[3].y);
    }
    static __device__ __forceinline__ float2 load_pair(const float *p) { return *reinterpret_cast<const float2 *>(p); }
    static __device__ __forceinline__ void store_pair(float *p, float2 v) { *reinterpret_cast<float2 *>(p) = v; }
};

// Video: one block row (tile rows = 1); images: four block rows, done one after another.
template <bool VIDEO> struct TileRows {
    static constexpr int RW = VIDEO ? 1 : 4;
};

template <typename T, bool VIDEO, bool FWD>
__global__ void __launch_bounds__(32 * WarpPipe<T>::WARPS, 1)
    haar_tma_kernel(const __grid_constant__ CUtensorMap xmap4, const __grid_constant__ CUtensorMap xmap1,
                    const __grid_constant__ CUtensorMap ymap, const TileGrid tg)
{
    using P = WarpPipe<T>;
    constexpr int NI = P::NI, WT = kTileBlocks;
    constexpr int RW = TileRows<VIDEO>::RW;
    constexpr int G = VIDEO ? 64 : 16;  // channel groups
    constexpr int NA = VIDEO ? 4 : 1;   // frames of a window
    constexpr int FRAME = 16 * RW * WT; // elements of one frame slice of the tile (4RW x 256)
    static_assert(G * RW * WT == kTileElems && NA * FRAME == kTileElems, "tile sizes");
    constexpr uint32_t TILE_BYTES = kTileElems * sizeof(T), FRAME_BYTES = FRAME * sizeof(T);
    constexpr float SCALE = VIDEO ? 0.125f : 0.25f;

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *wbase = smem_raw + warp * (NI + 1) * TILE_BYTES;
    T *in_buf = reinterpret_cast<T *>(wbase);
    T *out_buf = reinterpret_cast<T *>(wbase + NI * TILE_BYTES);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + P::WARPS * (NI + 1) * TILE_BYTES) + warp * NI;

    auto decode = [&](int64_t n, int &tx, int &ty, int &tq, int64_t &bc) {
        tx = (int)(n % tg.ntx);
        n /= tg.ntx;
        ty = (int)(n % tg.nty);
        n /= tg.nty;
        tq = (int)(n % tg.Tq);
        bc = n / tg.Tq;
    };

    // Lane 0: start the TMA load of tile n into input buffer s.
    auto issue_load = [&](int64_t n, int s) {
        int tx, ty, tq;
        int64_t bc;
        decode(n, tx, ty, tq, bc);
        const uint32_t dst = smem_addr(in_buf + s * kTileElems), bar = smem_addr(bars + s);
        if constexpr (FWD) {
            if (VIDEO && tq > 0) {
                mbar_expect_tx(bar, NA * FRAME_BYTES);
                tma_load_3d(dst, &xmap4, 4 * WT * tx, 4 * RW * ty, (int)(bc * tg.T + 4 * tq - 3), bar);
            } else {
                mbar_expect_tx(bar, FRAME_BYTES);
                tma_load_3d(dst, &xmap1, 4 * WT * tx, 4 * RW * ty, (int)(bc * tg.T), bar);
            }
        } else {
            const int b = (int)(bc / tg.C), c = (int)(bc - (int64_t)b * tg.C);
            mbar_expect_tx(bar, TILE_BYTES);
            tma_load_5d(dst, &ymap, WT * tx, RW * ty, tq, c, G * b, bar);
        }
    };

    const int64_t nwarps = (int64_t)gridDim.x * P::WARPS;
    const int64_t first = (int64_t)blockIdx.x * P::WARPS + warp;
    int64_t issued = 0; // tiles whose load lane 0 has issued
    if (lane == 0) {
        for (int s = 0; s < NI; ++s)
            mbar_init(smem_addr(bars + s), 1);
        fence_barrier_init();
        for (int s = 0; s < NI && first + s * nwarps < tg.ntiles; ++s, ++issued)
            issue_load(first + s * nwarps, s);
    }
    __syncwarp();

    int k = 0;
    bool failed = false;
    for (int64_t n = first; n < tg.ntiles; n += nwarps, ++k) {
        const int s = k % NI;
        const bool ok = mbar_wait(smem_addr(bars + s), (uint32_t)(k / NI) & 1u);
        if (__any_sync(0xFFFFFFFFu, !ok)) {
            failed = true;
            break;
        }
        int tx, ty, tq;
        int64_t bc;
        decode(n, tx, ty, tq, bc);
        const T *tin = in_buf + s * kTileElems;

#pragma unroll
        for (int rw = 0; rw < RW; ++rw) {
            float2 v[NA][4][4]; // FWD: [t][y][x] pixels -> [kt][ky][kx]; INV: the reverse
            if constexpr (FWD) {
#pragma unroll
                for (int a = 0; a < NA; ++a) {
                    const int fa = (VIDEO && tq > 0) ? a : 0; // window 0 reads frame 0 four times
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr)
                        SRow<T>::load(tin + (fa * 4 * RW + 4 * rw + rr) * 4 * WT + 8 * lane, v[a][rr]);
                }
            } else {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float2 p = SRow<T>::load_pair(tin + (g * RW + rw) * WT + 2 * lane);
                    if constexpr (VIDEO)
                        v[kt_of(g)][ky_of(g)][kx_of(g)] = p;
                    else
                        v[0][ky2_of(g)][kx2_of(g)] = p;
                }
            }
            if (rw == RW - 1) {
                // Every lane holds its inputs: hand the buffer back to the TMA engine and
                // start the load NI tiles ahead right away.
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int64_t nn = n + NI * nwarps;
                    if (nn < tg.ntiles) {
                        issue_load(nn, s);
                        ++issued;
                    }
                }
            }

#pragma unroll
            for (int a = 0; a < NA; ++a)
#pragma unroll
                for (int rr = 0; rr < 4; ++rr)
                    haar4x2(v[a][rr][0], v[a][rr][1], v[a][rr][2], v[a][rr][3]);
#pragma unroll
            for (int a = 0; a < NA; ++a)
#pragma unroll
                for (int d = 0; d < 4; ++d)
                    haar4x2(v[a][0][d], v[a][1][d], v[a][2][d], v[a][3][d]);
            if constexpr (VIDEO) {
#pragma unroll
                for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                    for (int d = 0; d < 4; ++d)
                        haar4x2(v[0][rr][d], v[1][rr][d], v[2][rr][d], v[3][rr][d]);
            }
            const float2 scale = make_float2(SCALE, SCALE);
#pragma unroll
            for (int a = 0; a < NA; ++a)
#pragma unroll
                for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                    for (int d = 0; d < 4; ++d)
                        v[a][rr][d] = __fmul2_rn(v[a][rr][d], scale);

            if (rw == 0) {
                // The output buffer is free once the previous tile's store has read it.
                if (lane == 0)
                    bulk_wait_read<0>();
                __syncwarp();
            }
            if constexpr (FWD) {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float2 p = VIDEO ? v[kt_of(g)][ky_of(g)][kx_of(g)] : v[0][ky2_of(g)][kx2_of(g)];
                    SRow<T>::store_pair(out_buf + (g * RW + rw) * WT + 2 * lane, p);
                }
            } else {
#pragma unroll
                for (int a = 0; a < NA; ++a)
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr)
                        SRow<T>::store(out_buf + (a * 4 * RW + 4 * rw + rr) * 4 * WT + 8 * lane, v[a][rr]);
            }
        }
        fence_proxy_async_smem(); // make this lane's results visible to the TMA engine
        __syncwarp();

        if (lane == 0) {
            const uint32_t src = smem_addr(out_buf);
            if constexpr (FWD) {
                const int b = (int)(bc / tg.C), c = (int)(bc - (int64_t)b * tg.C);
                tma_store_5d(&ymap, WT * tx, RW * ty, tq, c, G * b, src);
            } else if (VIDEO && tq > 0) {
                tma_store_3d(&xmap4, 4 * WT * tx, 4 * RW * ty, (int)(bc * tg.T + 4 * tq - 3), src);
            } else {
                // Window 0 keeps the last of its four frames (the others are the replicas); images have one.
                tma_store_3d(&xmap1, 4 * WT * tx, 4 * RW * ty, (int)(bc * tg.T),
                             smem_addr(out_buf + (VIDEO ? 3 * FRAME : 0)));
            }
            bulk_commit();
        }
    }

    if (lane == 0) {
        if (failed) {
            // Drain the loads this warp issued and did not consume, each wait again bounded.
            for (int64_t it = k; it < issued; ++it)
                mbar_wait(smem_addr(bars + (it % NI)), (uint32_t)(it / NI) & 1u);
            atomicAdd(&g_wait_timeouts, 1u);
        }
        bulk_wait_all(); // stores must finish reading shared memory before the CTA exits
    }
    __syncwarp();
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
template <typename T, bool VIDEO, bool FWD> tok_status launch(const void *in, void *out, const HaarDims &d, cudaStream_t stream)
{
    using P = WarpPipe<T>;
    constexpr int G = VIDEO ? 64 : 16, RW = TileRows<VIDEO>::RW, WT = kTileBlocks;
    const CUtensorMapDataType dt = sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const uint64_t es = sizeof(T);
    const void *xp = FWD ? in : out, *yp = FWD ? out : in;

    CUtensorMap xm4, xm1, ym;
    const uint64_t xdims[3] = {(uint64_t)d.W, (uint64_t)d.H, (uint64_t)(d.B * d.C * d.T)};
    const uint64_t xstr[2] = {d.W * es, d.H * d.W * es};
    const uint32_t box4[3] = {4u * WT, 4u * RW, 4u}, box1[3] = {4u * WT, 4u * RW, 1u};
    const uint64_t ydims[5] = {(uint64_t)d.w, (uint64_t)d.h, (uint64_t)d.Tq, (uint64_t)d.C, (uint64_t)(G * d.B)};
    const uint64_t plane = d.Tq * d.h * d.w * es;
    const uint64_t ystr[4] = {d.w * es, d.h * d.w * es, plane, d.C * plane};
    const uint32_t ybox[5] = {(uint32_t)WT, (uint32_t)RW, 1u, 1u, (uint32_t)G};
    if (!encode_tensor_map(&xm1, dt, 3, xp, xdims, xstr, box1) || !encode_tensor_map(&ym, dt, 5, yp, ydims, ystr, ybox))
        return TOK_ERR_SHAPE;
    if (VIDEO) {
        if (!encode_tensor_map(&xm4, dt, 3, xp, xdims, xstr, box4))
            return TOK_ERR_SHAPE;
    } else {
        xm4 = xm1;
    }

    TileGrid tg;
    tg.ntx = (int)((d.w + WT - 1) / WT);
    tg.nty = (int)((d.h + RW - 1) / RW);
    tg.Tq = (int)d.Tq;
    tg.C = (int)d.C;
    tg.T = (int)d.T;
    tg.ntiles = (int64_t)tg.ntx * tg.nty * d.Tq * d.B * d.C;

    // Per call: the attribute belongs to the current device.
    cudaError_t attr_err =
        cudaFuncSetAttribute(haar_tma_kernel<T, VIDEO, FWD>, cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM);
    if (attr_err != cudaSuccess) {
        record_cuda_error(attr_err);
        return TOK_ERR_CUDA;
    }
    const int64_t ctas_needed = (tg.ntiles + P::WARPS - 1) / P::WARPS; // a warp per tile at most
    const int64_t ctas = sm_count();
    const unsigned grid = (unsigned)(ctas_needed < ctas ? ctas_needed : ctas);
    haar_tma_kernel<T, VIDEO, FWD><<<grid, 32 * P::WARPS, P::SMEM, stream>>>(xm4, xm1, ym, tg);
    return launch_status();
}

} // namespace

bool haar_tma_eligible(const void *in, const void *out, tok_dtype dt, const HaarDims &d)
{
    const int64_t es = dt == TOK_F32 ? 4 : 2;
    if (!aligned(in, 16) || !aligned(out, 16))
        return false;
    if ((d.w * es) % 16 != 0) // row strides of both tensors must be multiples of 16 bytes
        return false;
    // Coordinates are 32-bit: frames of the flattened [B*C*T] axis and the group axis must fit.
    if (d.B * d.C * d.T >= (int64_t)1 << 31 || 64 * d.B >= (int64_t)1 << 31 || d.W >= (int64_t)1 << 31 ||
        d.H >= (int64_t)1 << 31)
        return false;
    return sm_count() > 0;
}

tok_status haar_tma_launch(bool fwd, const void *in, void *out, tok_dtype dt, const HaarDims &d, cudaStream_t stream)
{
    const bool video = d.T > 1;
    if (dt == TOK_BF16) {
        if (video)
            return fwd ? launch<__nv_bfloat16, true, true>(in, out, d, stream)
                       : launch<__nv_bfloat16, true, false>(in, out, d, stream);
        return fwd ? launch<__nv_bfloat16, false, true>(in, out, d, stream)
                   : launch<__nv_bfloat16, false, false>(in, out, d, stream);
    }
    if (video)
        return fwd ? launch<float, true, true>(in, out, d, stream) : launch<float, true, false>(in, out, d, stream);
    return fwd ? launch<float, false, true>(in, out, d, stream) : launch<float, false, false>(in, out, d, stream);
}

tok_status read_and_clear_timeouts(cudaStream_t stream, unsigned int *count)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(count, g_wait_timeouts, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && *count)
        e = cudaMemcpyToSymbolAsync(g_wait_timeouts, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return TOK_ERR_CUDA;
    }
    return TOK_OK;
}

} // namespace tok
