// The first causal factorized convolution after the patcher, as hand-written
// implicit GEMMs on the 5th-generation tensor cores.
//
// Source: "Cosmos World Foundation Model Platform for Physical AI (Cosmos-Predict1)"
// notes, model architecture item 1: after the 2-level Haar transform the encoder's
// convolutions are factorized -- a 1 x k x k spatial convolution, then a k x 1 x 1
// temporal convolution padded by k - 1 on the past side only.
//
// Activations are channels-last bf16 [frames, h, w, C]; fp32 accumulation.  The
// MMA is the 2-SM form: a CTA pair (a 2 x 1 x 1 cluster, one CTA per SM) computes
// 256 output positions -- two tiles of 16 rows x 8 columns of one frame, one per
// CTA -- by up to 256 output channels, M = 256 and N = 256, each CTA loading its own
// tile's activations and half of the filter, so the filter crosses L2 half as often
// per flop as with one-CTA 128 x 256 tiles.  Each K block is 64 input channels of one
// tap, and a stage holds kStageK of them.  The pair walks its tiles persistently.
// Warp roles in each CTA:
//   warp 0     tensor copies: per K block, the activation box [64 ch, 8 cols,
//              16 rows] of the tap's frame / shift (zero-filled outside the frame)
//              and its half of the filter box [64 k, N / 2], into one of kStages
//              stages in the 128-byte swizzle the MMA reads; completion is counted
//              on the leader CTA's barrier;
//   warp 1     (leader only) one thread issues tcgen05.mma (4 per K block, K = 16
//              each) into the pair's tensor-memory accumulator, waiting and
//              committing once per stage (each barrier operation costs this thread
//              about as long as one or two MMAs), the commit releasing the stage to
//              both CTAs' copy warps;
//   warps 2-5  epilogue: tensor memory -> registers (each thread one position, its
//              lane of this CTA's accumulator half), round to bf16, through a
//              128-byte-swizzled staging buffer to tensor stores of whole lines.
// Two accumulators in tensor memory (2 x N columns) let a tile's epilogue overlap
// the next tile's MMAs.  The temporal convolution orders tiles time-fastest, so the
// k frames a tile reads are read again by the next tiles while they are in L2; the
// spatial one orders them column-block-fastest for the halo rows.  No load is
// broadcast to the pair: every copy fills only its own CTA's shared memory.
//
// Waits are bounded: a barrier that does not complete in time raises the CTA's
// abort flag, every role leaves its loop, the copies and MMAs already issued are
// waited for (bounded), tensor memory is freed and a timeout is counted for
// tok_check_device().
#include <algorithm>
#include <cstring>

#include "tok_common.cuh"
#include "tok_internal.h"
#include "umma.cuh"

namespace tok {

// Convolution kernels that gave up on a barrier wait since the last check.
static __device__ unsigned int g_conv_timeouts = 0;

namespace {

constexpr int kTileRows = 16, kTileCols = 8, kBM = kTileRows * kTileCols; // positions per CTA tile
constexpr int kBK = 64;                                                   // K per stage: one 128-byte row
constexpr int kStages = 3; // stages of kStageK K blocks
constexpr int kStageK = 2; // (the MMA loop below is written for two)
constexpr int kThreads = 192; // 6 warps
constexpr uint32_t kABytes = kBM * kBK * 2;
constexpr uint16_t kPairMask = 0x3; // both CTAs of the pair

struct ConvGeom {
    int frames;   // B * T
    int T;        // frames per clip
    int h, w;
    int cin;      // input channels (multiple of 64)
    int n;        // output channels
    int bn;       // output channels per pair tile (each CTA loads bn / 2 filter rows)
    int n_tiles;  // n / bn
    int tiles_xp; // column-block pairs
    int tiles_y;
    int npairs;   // pair tiles
    int k;        // taps per axis
    int temporal; // 1: causal temporal (k x 1 x 1), 0: spatial (1 x k x k, 'same' zeros)
    int nstages;  // ring size of the plane kernel
};

struct TileCoord {
    int f;   // frame index in [0, B*T)
    int t;   // frame within its clip
    int y0, x0, n0;
    int kb0; // first K step (temporal: taps before the clip's first frame are skipped)
    int nkb; // K steps of this tile
};

// Pair tile i, this CTA's half (rank): column block 2 * xp + rank.
__device__ __forceinline__ TileCoord decode_tile(const ConvGeom &g, int i, uint32_t rank)
{
    TileCoord c;
    const int nchunk = g.cin / kBK;
    int r = i, xp, yb, nb;
    if (g.temporal) { // time fastest: the k frames a tile reads are read by the next tiles too
        c.t = r % g.T;
        r /= g.T;
        nb = r % g.n_tiles;
        r /= g.n_tiles;
        xp = r % g.tiles_xp;
        r /= g.tiles_xp;
        yb = r % g.tiles_y;
        const int b = r / g.tiles_y;
        c.f = b * g.T + c.t;
        const int dt0 = max(0, g.k - 1 - c.t);
        c.kb0 = dt0 * nchunk;
        c.nkb = (g.k - dt0) * nchunk;
    } else { // output-channel tiles fastest (they share the activations), then column blocks
        nb = r % g.n_tiles;
        r /= g.n_tiles;
        xp = r % g.tiles_xp;
        r /= g.tiles_xp;
        yb = r % g.tiles_y;
        c.f = r / g.tiles_y;
        c.t = 0;
        c.kb0 = 0;
        c.nkb = g.k * g.k * nchunk;
    }
    c.y0 = yb * kTileRows;
    c.x0 = (2 * xp + (int)rank) * kTileCols;
    c.n0 = nb * g.bn;
    return c;
}

__device__ __forceinline__ uint32_t tmem_cols(int bn)
{
    return bn <= 16 ? 32u : bn <= 32 ? 64u : bn <= 64 ? 128u : bn <= 128 ? 256u : 512u;
}

// Epilogue staging per CTA: 4 epilogue warps x NBUF buffers of 4 KB.
constexpr uint32_t epi_bytes(int nbuf) { return 4u * (uint32_t)nbuf * 4096u; }

// Epilogue of one CTA's tile; warp q = warp % 4 holds accumulator lanes 32q .. 32q + 31,
// the tile's rows 4q .. 4q + 3.  Per 64 output channels: tensor memory -> registers ->
// bf16 rows of a 128-byte-swizzled staging buffer of the warp (NBUF, in turn) -> one
// tensor store of the box [64 ch, 8 cols, 4 rows] at (n0 + cb, x0, y0 + 4q, f); the store
// clips positions outside the frame and writes whole lines.  A last group of 32 channels
// (bn % 64 == 32) is stored from registers, positions outside the frame skipped.
template <int NBUF>
__device__ __forceinline__ void store_tile(uint32_t tmem_acc, int q, int lane, const CUtensorMap *omap, int f, int y0,
                                           int x0, int n0, uint32_t stage, unsigned char *stage_ptr, uint32_t &sbuf,
                                           __nv_bfloat16 *o, bool valid, int bn)
{
    const uint32_t t0 = tmem_acc + ((uint32_t)(32 * q) << 16);
    int cb = 0;
    for (; cb + 64 <= bn; cb += 64) {
        uint32_t v[64];
        tmem_ld64(t0 + (uint32_t)cb, v);
        tmem_wait_ld();
        const uint32_t b = sbuf % NBUF;
        if (lane == 0)
            bulk_wait_read<NBUF - 1>(); // the store that last used this buffer has read it
        __syncwarp();
        unsigned char *buf = stage_ptr + b * 4096u;
#pragma unroll
        for (int s8 = 0; s8 < 8; ++s8)
            *reinterpret_cast<uint4 *>(buf + sw128_offset((uint32_t)lane, 8u * s8)) =
                make_uint4(pack_bf16x2(__uint_as_float(v[8 * s8 + 0]), __uint_as_float(v[8 * s8 + 1])),
                           pack_bf16x2(__uint_as_float(v[8 * s8 + 2]), __uint_as_float(v[8 * s8 + 3])),
                           pack_bf16x2(__uint_as_float(v[8 * s8 + 4]), __uint_as_float(v[8 * s8 + 5])),
                           pack_bf16x2(__uint_as_float(v[8 * s8 + 6]), __uint_as_float(v[8 * s8 + 7])));
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_4d(omap, n0 + cb, x0, y0 + 4 * q, f, stage + b * 4096u);
            bulk_commit();
        }
        ++sbuf;
    }
    if (cb < bn) {
        uint32_t v[32];
        tmem_ld32(t0 + (uint32_t)cb, v);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
            for (int s = 0; s < 4; ++s)
                *reinterpret_cast<uint4 *>(o + cb + 8 * s) =
                    make_uint4(pack_bf16x2(__uint_as_float(v[8 * s + 0]), __uint_as_float(v[8 * s + 1])),
                               pack_bf16x2(__uint_as_float(v[8 * s + 2]), __uint_as_float(v[8 * s + 3])),
                               pack_bf16x2(__uint_as_float(v[8 * s + 4]), __uint_as_float(v[8 * s + 5])),
                               pack_bf16x2(__uint_as_float(v[8 * s + 6]), __uint_as_float(v[8 * s + 7])));
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
conv_tc_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
               const __grid_constant__ CUtensorMap omap, __nv_bfloat16 *__restrict__ out, const ConvGeom g)
{
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages], accf[2], acce[2], drain;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
    const uint32_t bbytes = (uint32_t)(g.bn / 2) * kBK * 2; // this CTA's half of a filter K block
    // A stage holds kStageK K blocks: their activation boxes, then their filter halves.
    const uint32_t stage_bytes = kStageK * (kABytes + bbytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const uint32_t ncols = tmem_cols(g.bn);
    const int pair = blockIdx.x >> 1, npair_ctas = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_addr(&full[s]), 1);
            mbar_init(smem_addr(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_addr(&accf[a]), 1);
            mbar_init(smem_addr(&acce[a]), 8); // 4 epilogue warps in each CTA
        }
        mbar_init(smem_addr(&drain), 1);
        abort_s = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(smem_addr(&tmem_base_s), ncols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync(); // both CTAs' barriers exist before any copy or arrive reaches them
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    volatile int *abort = &abort_s;
    const int nchunk = g.cin / kBK;

    if (warp == 0 && lane == 0) {
        // Tensor copies of this CTA's operands; completion counted on the leader's barrier.
        uint32_t it = 0;
        bool ok = true;
        for (int i = pair; i < g.npairs && ok; i += npair_ctas) {
            const TileCoord c = decode_tile(g, i, rank);
            for (int kb = 0; kb < c.nkb; kb += kStageK, ++it) {
                const int nk = min(kStageK, c.nkb - kb);
                const uint32_t s = it % kStages, ph = (it / kStages) & 1u;
                if (!wait_or_abort(smem_addr(&empty[s]), ph ^ 1u, abort)) {
                    ok = false;
                    break;
                }
                const uint32_t sa = base + s * stage_bytes, sb = sa + kStageK * kABytes;
                const uint32_t fb = mapa_shared(smem_addr(&full[s]), 0);
                if (leader)
                    mbar_expect_tx(smem_addr(&full[s]), 2 * (uint32_t)nk * (kABytes + bbytes));
                for (int j = 0; j < nk; ++j) {
                    const int kk = c.kb0 + kb + j, tap = kk / nchunk, ch = (kk - tap * nchunk) * kBK;
                    if (g.temporal)
                        tma_load_4d_pair(sa + j * kABytes, &amap, ch, c.x0, c.y0, c.f - (g.k - 1) + tap, fb);
                    else {
                        const int pad = (g.k - 1) / 2, dy = tap / g.k, dx = tap - dy * g.k;
                        tma_load_4d_pair(sa + j * kABytes, &amap, ch, c.x0 + dx - pad, c.y0 + dy - pad, c.f, fb);
                    }
                    tma_load_2d_pair(sb + j * bbytes, &bmap, kk * kBK, c.n0 + (int)rank * (g.bn / 2), fb);
                }
            }
        }
        if (!ok && leader) // let the copies already issued land before the CTA exits (each wait bounded)
            for (uint32_t j = it > kStages ? it - kStages : 0; j < it; ++j)
                mbar_wait(smem_addr(&full[j % kStages]), (j / kStages) & 1u);
    } else if (warp == 1 && lane == 0 && leader) {
        // MMA issue for the pair: one wait and one commit per stage of kStageK K blocks, ring
        // positions and descriptors kept as running values (this thread is the narrowest point).
        const uint32_t idesc = idesc_bf16_f32(2 * kBM, g.bn);
        const uint64_t adesc0 = sw128_desc(base), bdesc0 = sw128_desc(base + kStageK * kABytes);
        uint32_t s = 0, ph = 0, tc = 0;
        bool ok = true;
        for (int i = pair; i < g.npairs && ok; i += npair_ctas, ++tc) {
            const TileCoord c = decode_tile(g, i, 0);
            const uint32_t acc = tc & 1u, use = tc >> 1;
            if (!wait_or_abort(smem_addr(&acce[acc]), (use & 1u) ^ 1u, abort))
                break;
            tc_fence_after();
            const uint32_t d = tmem + acc * (uint32_t)g.bn;
            for (int kb = 0; kb < c.nkb; kb += kStageK) {
                if (!wait_or_abort(smem_addr(&full[s]), ph, abort)) {
                    ok = false;
                    break;
                }
                const uint64_t a0 = adesc0 + ((s * stage_bytes) >> 4), b0 = bdesc0 + ((s * stage_bytes) >> 4);
                umma_bf16_pair(d, a0, b0, idesc, kb != 0);
                umma_bf16_pair(d, a0 + 2, b0 + 2, idesc, 1u);
                umma_bf16_pair(d, a0 + 4, b0 + 4, idesc, 1u);
                umma_bf16_pair(d, a0 + 6, b0 + 6, idesc, 1u);
                if (kb + 1 < c.nkb) {
                    const uint64_t a1 = a0 + (kABytes >> 4), b1 = b0 + (bbytes >> 4);
                    umma_bf16_pair(d, a1, b1, idesc, 1u);
                    umma_bf16_pair(d, a1 + 2, b1 + 2, idesc, 1u);
                    umma_bf16_pair(d, a1 + 4, b1 + 4, idesc, 1u);
                    umma_bf16_pair(d, a1 + 6, b1 + 6, idesc, 1u);
                }
                umma_commit_pair(smem_addr(&empty[s]), kPairMask);
                if (++s == kStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
            if (ok)
                umma_commit_pair(smem_addr(&accf[acc]), kPairMask);
        }
        // Every MMA issued has completed before tensor memory is freed.
        umma_commit_pair(smem_addr(&drain), 0x1);
        mbar_wait(smem_addr(&drain), 0u);
    } else if (warp >= 2) {
        // Epilogue of this CTA's tile; each warp then frees the accumulator on the leader.
        const int q = warp & 3, row = 32 * q + lane;
        const int r = row / kTileCols, jj = row - r * kTileCols;
        const uint32_t acce0 = mapa_shared(smem_addr(&acce[0]), 0), acce1 = mapa_shared(smem_addr(&acce[1]), 0);
        const uint32_t stage = base + kStages * stage_bytes + (uint32_t)q * 8192u;
        unsigned char *stage_ptr = smem_raw + (stage - smem_addr(smem_raw));
        uint32_t tc = 0, sbuf = 0;
        for (int i = pair; i < g.npairs; i += npair_ctas, ++tc) {
            const TileCoord c = decode_tile(g, i, rank);
            const uint32_t acc = tc & 1u, use = tc >> 1;
            if (!wait_or_abort(smem_addr(&accf[acc]), use & 1u, abort))
                break;
            tc_fence_after();
            const int y = c.y0 + r, x = c.x0 + jj;
            __nv_bfloat16 *o = out + (((int64_t)c.f * g.h + y) * g.w + x) * g.n + c.n0;
            store_tile<2>(tmem + acc * (uint32_t)g.bn, q, lane, &omap, c.f, c.y0, c.x0, c.n0, stage, stage_ptr, sbuf, o,
                          y < g.h && x < g.w, g.bn);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(acc ? acce1 : acce0);
        }
        if (lane == 0)
            bulk_wait_all(); // the tile stores have completed before the CTA exits
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync(); // neither CTA frees the pair's tensor memory while the other still uses it
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, ncols);
    }
    if (threadIdx.x == 0 && *abort)
        atomicAdd(&g_conv_timeouts, 1u);
}

// The spatial convolution with its activation tiles read once per column shift: for
// each 64-channel chunk c and column shift dx, one tensor copy brings the plane of
// 16 + k - 1 rows x 8 columns (rows y0 - pad .., columns x0 + dx - pad ..) in the
// 128-byte swizzle, and the k row shifts dy are that plane seen from row-atom dy (one
// tile row of 8 positions is one 1024-byte swizzle atom).  K order (c, dx, dy).  A
// stage holds one plane and the k filter K blocks it meets, so the MMA thread waits and
// commits once per 4k MMAs: a single issuing thread pays for each barrier operation
// (a wait or a commit costs it about as long as one or two MMAs), and at one wait and
// one commit per K block it could not keep the 2-SM tensor core busy.
constexpr int kMaxPStages = 3;
constexpr int kMaxPlaneK = 5;
constexpr int kPlaneEpiBuf = 1; // one staging buffer per epilogue warp (shared memory goes to the stages)

__host__ __device__ constexpr uint32_t plane_stage_bytes(int bn, int k)
{
    return (uint32_t)(kTileRows + k - 1) * kTileCols * 128 + (uint32_t)k * (uint32_t)(bn / 2) * kBK * 2;
}

__global__ void __launch_bounds__(kThreads, 1)
conv_planes_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                   const __grid_constant__ CUtensorMap omap, __nv_bfloat16 *__restrict__ out, const ConvGeom g)
{
    __shared__ __align__(8) uint64_t full[kMaxPStages], empty[kMaxPStages], accf[2], acce[2], drain;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
    const int nst = g.nstages;
    const uint32_t bbytes = (uint32_t)(g.bn / 2) * kBK * 2;
    const uint32_t plane_bytes = (uint32_t)(kTileRows + g.k - 1) * kTileCols * 128;
    const uint32_t stage_bytes = plane_stage_bytes(g.bn, g.k);
    const uint32_t ebase = base + (uint32_t)nst * stage_bytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const uint32_t ncols = tmem_cols(g.bn);
    const int pair = blockIdx.x >> 1, npair_ctas = gridDim.x >> 1;
    const int nchunk = g.cin / kBK, pad = (g.k - 1) / 2;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mbar_init(smem_addr(&full[s]), 1);
            mbar_init(smem_addr(&empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_addr(&accf[a]), 1);
            mbar_init(smem_addr(&acce[a]), 8);
        }
        mbar_init(smem_addr(&drain), 1);
        abort_s = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(smem_addr(&tmem_base_s), ncols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    volatile int *abort = &abort_s;

    if (warp == 0 && lane == 0) {
        // Per stage: the plane and its k filter halves of this CTA, counted on the leader's barrier.
        uint32_t it = 0;
        bool ok = true;
        for (int i = pair; i < g.npairs && ok; i += npair_ctas) {
            const TileCoord c = decode_tile(g, i, rank);
            for (int ch = 0; ch < nchunk && ok; ++ch)
                for (int dx = 0; dx < g.k; ++dx, ++it) {
                    const uint32_t s = it % nst, ph = (it / nst) & 1u;
                    if (!wait_or_abort(smem_addr(&empty[s]), ph ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    const uint32_t sa = base + s * stage_bytes, sb = sa + plane_bytes;
                    const uint32_t fb = mapa_shared(smem_addr(&full[s]), 0);
                    if (leader)
                        mbar_expect_tx(smem_addr(&full[s]), 2 * stage_bytes);
                    tma_load_4d_pair(sa, &amap, ch * kBK, c.x0 + dx - pad, c.y0 - pad, c.f, fb);
                    for (int dy = 0; dy < g.k; ++dy)
                        tma_load_2d_pair(sb + dy * bbytes, &bmap, (dy * g.k + dx) * g.cin + ch * kBK,
                                         c.n0 + (int)rank * (g.bn / 2), fb);
                }
        }
        if (!ok && leader)
            for (uint32_t j = it > (uint32_t)nst ? it - nst : 0; j < it; ++j)
                mbar_wait(smem_addr(&full[j % nst]), (j / nst) & 1u);
    } else if (warp == 1 && lane == 0 && leader) {
        const uint32_t idesc = idesc_bf16_f32(2 * kBM, g.bn);
        uint32_t it = 0, tc = 0;
        bool ok = true;
        for (int i = pair; i < g.npairs && ok; i += npair_ctas, ++tc) {
            const uint32_t acc = tc & 1u, use = tc >> 1;
            if (!wait_or_abort(smem_addr(&acce[acc]), (use & 1u) ^ 1u, abort))
                break;
            tc_fence_after();
            const uint32_t d = tmem + acc * (uint32_t)g.bn;
            for (int pl = 0; pl < nchunk * g.k; ++pl, ++it) {
                const uint32_t s = it % nst, ph = (it / nst) & 1u;
                if (!wait_or_abort(smem_addr(&full[s]), ph, abort)) {
                    ok = false;
                    break;
                }
                const uint32_t sa = base + s * stage_bytes, sb = sa + plane_bytes;
                for (int dy = 0; dy < g.k; ++dy) {
                    const uint64_t ad = sw128_desc(sa + (uint32_t)dy * 1024u), bd = sw128_desc(sb + dy * bbytes);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        umma_bf16_pair(d, ad + 2 * k, bd + 2 * k, idesc, (pl | dy | k) != 0);
                }
                umma_commit_pair(smem_addr(&empty[s]), kPairMask);
            }
            if (ok)
                umma_commit_pair(smem_addr(&accf[acc]), kPairMask);
        }
        umma_commit_pair(smem_addr(&drain), 0x1);
        mbar_wait(smem_addr(&drain), 0u);
    } else if (warp >= 2) {
        const int q = warp & 3, row = 32 * q + lane;
        const int r = row / kTileCols, jj = row - r * kTileCols;
        const uint32_t acce0 = mapa_shared(smem_addr(&acce[0]), 0), acce1 = mapa_shared(smem_addr(&acce[1]), 0);
        const uint32_t stage = ebase + (uint32_t)q * (kPlaneEpiBuf * 4096u);
        unsigned char *stage_ptr = smem_raw + (stage - smem_addr(smem_raw));
        uint32_t tc = 0, sbuf = 0;
        for (int i = pair; i < g.npairs; i += npair_ctas, ++tc) {
            const TileCoord c = decode_tile(g, i, rank);
            const uint32_t acc = tc & 1u, use = tc >> 1;
            if (!wait_or_abort(smem_addr(&accf[acc]), use & 1u, abort))
                break;
            tc_fence_after();
            const int y = c.y0 + r, x = c.x0 + jj;
            __nv_bfloat16 *o = out + (((int64_t)c.f * g.h + y) * g.w + x) * g.n + c.n0;
            store_tile<kPlaneEpiBuf>(tmem + acc * (uint32_t)g.bn, q, lane, &omap, c.f, c.y0, c.x0, c.n0, stage,
                                     stage_ptr, sbuf, o, y < g.h && x < g.w, g.bn);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(acc ? acce1 : acce0);
        }
        if (lane == 0)
            bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, ncols);
    }
    if (threadIdx.x == 0 && *abort)
        atomicAdd(&g_conv_timeouts, 1u);
}

// Stages of the plane kernel that fit (with the epilogue staging and the alignment slack) in
// the 227 KB of shared memory a CTA may have; 0 if fewer than two fit.
int plane_stages(int bn, int k)
{
    const int64_t room = 232448 - 1024 - 1024 - (int64_t)epi_bytes(kPlaneEpiBuf); // static barriers and slack
    const int n = (int)std::min<int64_t>(kMaxPStages, room / plane_stage_bytes(bn, k));
    return n >= 2 ? n : 0;
}

size_t planes_smem_bytes(int bn, int k, int nst)
{
    return (size_t)nst * plane_stage_bytes(bn, k) + epi_bytes(kPlaneEpiBuf) + 1024;
}

size_t conv_smem_bytes(int bn)
{
    return (size_t)kStages * kStageK * (kABytes + (uint32_t)(bn / 2) * kBK * 2) + epi_bytes(2) + 1024;
}

bool fits_int(int64_t v) { return v >= 0 && v < ((int64_t)1 << 31); }

// The tensor-core form takes Cin a multiple of 64 and Cout a multiple of 32 up to 256
// or a multiple of 256; 32-bit extents.
bool tc_eligible(int64_t Cin, int64_t Cout)
{
    return Cin >= 64 && Cin % 64 == 0 && Cout >= 32 && Cout % 32 == 0 && (Cout <= 256 || Cout % 256 == 0);
}

// Launch a pair kernel: as many pairs as can be resident at once (each CTA needs a whole
// SM), at most one per pair tile.
template <typename K, typename G>
tok_status launch_pairs(K kernel, int64_t npairs, size_t smem, int threads, cudaStream_t stream,
                        const CUtensorMap &m0, const CUtensorMap &m1, const CUtensorMap &m2, __nv_bfloat16 *out,
                        const G &g)
{
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return TOK_ERR_CUDA;
    }
    const int sms = sm_count();
    if (sms <= 0)
        return launch_status();
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)(2 * std::min<int64_t>(npairs, sms / 2)), 1, 1);
    cfg.blockDim = dim3(threads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int resident = 0;
    e = cudaOccupancyMaxActiveClusters(&resident, kernel, &cfg);
    if (e != cudaSuccess || resident <= 0) {
        record_cuda_error(e != cudaSuccess ? e : cudaErrorInvalidConfiguration);
        return TOK_ERR_CUDA;
    }
    cfg.gridDim = dim3((unsigned)(2 * std::min<int64_t>(npairs, resident)), 1, 1);
    e = cudaLaunchKernelEx(&cfg, kernel, m0, m1, m2, out, g);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return TOK_ERR_CUDA;
    }
    return launch_status();
}

tok_status conv_tc_launch(bool temporal, const void *x, const void *wts, void *y, int64_t B, int64_t T, int64_t h,
                          int64_t w, int64_t Cin, int64_t Cout, int64_t k, cudaStream_t stream)
{
    ConvGeom g{};
    g.frames = (int)(B * T);
    g.T = (int)T;
    g.h = (int)h;
    g.w = (int)w;
    g.cin = (int)Cin;
    g.n = (int)Cout;
    g.bn = Cout <= 256 ? (int)Cout : 256;
    g.n_tiles = (int)(Cout / g.bn);
    const int64_t tiles_x = (w + kTileCols - 1) / kTileCols;
    g.tiles_xp = (int)((tiles_x + 1) / 2);
    g.tiles_y = (int)((h + kTileRows - 1) / kTileRows);
    const int64_t npairs = (int64_t)g.frames * g.tiles_xp * g.tiles_y * g.n_tiles;
    if (!fits_int(npairs))
        return TOK_ERR_SHAPE;
    g.npairs = (int)npairs;
    g.k = (int)k;
    g.temporal = temporal ? 1 : 0;

    CUtensorMap amap, bmap;
    const uint64_t adims[4] = {(uint64_t)Cin, (uint64_t)w, (uint64_t)h, (uint64_t)g.frames};
    const uint64_t astr[3] = {(uint64_t)Cin * 2, (uint64_t)w * Cin * 2, (uint64_t)h * w * Cin * 2};
    const uint32_t abox[4] = {kBK, kTileCols, kTileRows, 1};
    const int64_t ktot = (temporal ? k : k * k) * Cin;
    const uint64_t bdims[2] = {(uint64_t)ktot, (uint64_t)Cout};
    const uint64_t bstr[1] = {(uint64_t)ktot * 2};
    const uint32_t bbox[2] = {kBK, (uint32_t)(g.bn / 2)};
    CUtensorMap omap;
    const uint64_t odims[4] = {(uint64_t)Cout, (uint64_t)w, (uint64_t)h, (uint64_t)g.frames};
    const uint64_t ostr[3] = {(uint64_t)Cout * 2, (uint64_t)w * Cout * 2, (uint64_t)h * w * Cout * 2};
    const uint32_t obox[4] = {(uint32_t)std::min<int64_t>(64, Cout), kTileCols, 4, 1};
    g.nstages = temporal || k > kMaxPlaneK ? 0 : plane_stages(g.bn, (int)k);
    if (g.nstages) {
        const uint32_t pbox[4] = {kBK, kTileCols, (uint32_t)(kTileRows + k - 1), 1};
        if (!encode_tensor_map_sw128(&amap, 4, x, adims, astr, pbox) ||
            !encode_tensor_map_sw128(&bmap, 2, wts, bdims, bstr, bbox) ||
            !encode_tensor_map_sw128(&omap, 4, y, odims, ostr, obox))
            return TOK_ERR_SHAPE;
        return launch_pairs(conv_planes_kernel, npairs, planes_smem_bytes(g.bn, (int)k, g.nstages), kThreads, stream,
                            amap, bmap, omap, static_cast<__nv_bfloat16 *>(y), g);
    }
    if (!encode_tensor_map_sw128(&amap, 4, x, adims, astr, abox) ||
        !encode_tensor_map_sw128(&bmap, 2, wts, bdims, bstr, bbox) ||
        !encode_tensor_map_sw128(&omap, 4, y, odims, ostr, obox))
        return TOK_ERR_SHAPE;
    return launch_pairs(conv_tc_kernel, npairs, conv_smem_bytes(g.bn), kThreads, stream, amap, bmap, omap,
                        static_cast<__nv_bfloat16 *>(y), g);
}

// ---------------------------------------------------------------------------
// The patcher fused into the spatial convolution (k = 3).  The A operand of each
// K step is made in shared memory by four Haar warps from the pixels, so the
// coefficients never reach HBM.  Its K order is (input channel c, column shift dx,
// row shift dy, the 64 subbands g of c): plane (c, dx) holds, for the tile's 16 + 2
// latent rows and 8 columns shifted by dx - 1, the 64 coefficients of colour c as one
// 128-byte swizzled row per position (row q = r * 8 + j: one tile row is one 1024-byte
// swizzle atom), and the three K steps dy = 0, 1, 2 are that plane seen from atom dy.
// The filter is read in the same K order from a packed copy (tok_patch_embed_pack_weights).
//   warp 0     tensor copies of the packed filter: a stage holds the three row-shift K blocks
//              [64 k, N / 2] that one plane meets, so the MMA thread waits and commits once
//              per plane and filter stage (12 MMAs) -- with a stage per K block its barrier
//              operations, not the tensor cores, set the pace;
//   warp 1     MMA issue (planes and filter stages as they fill);
//   warps 2-5  epilogue, as in conv_tc_kernel (one staging buffer per warp);
//   warps 6-9  Haar: per colour, one tensor copy of the pixels the tile's 3 x 3
//              neighbourhood reads ([4 frames][72 rows][48 cols]) into the one pixel
//              buffer, which the next colour's copy refills as soon as every Haar thread
//              holds its pixels in registers; each of 90 threads transforms two
//              horizontally adjacent blocks in packed f32x2 pairs -- the butterflies of the
//              planar patcher in its order (columns, rows, frames; then x 1/8), so the
//              coefficients are the patcher's bits -- rounds them to bf16 and writes them
//              into the colour's three planes, each as soon as a plane slot is free.
// Latent positions outside the frame read zero pixels (the tensor copy fills zeros),
// which is exactly the convolution's zero padding of the coefficients.
// ---------------------------------------------------------------------------
constexpr int kFGroup = 3;                       // filter K blocks per stage (the row shifts of a plane)
constexpr int kFStages = 2;                      // filter stages
constexpr int kEmbedEpiBuf = 1;                  // staging buffers per epilogue warp
constexpr int kPlanes = 4;                       // A planes in flight (a ring)
constexpr int kPlaneRows = kTileRows + 2;        // latent rows of a plane
constexpr uint32_t kPlaneBytes = kPlaneRows * kTileCols * 128; // 18 KB
constexpr int kPixCols = 48, kPixRows = 4 * kPlaneRows, kPixFrames = 4;
constexpr uint32_t kPixBytes = kPixCols * kPixRows * kPixFrames * 2; // 27 KB
constexpr int kEmbedThreads = 320;               // 10 warps
constexpr int kHaarThreads = 128;
constexpr int kHaarFirst = 192;                  // first Haar thread

struct EmbedGeom {
    int B, C, Tq, h, w;   // pixels [B, C, 4*Tq - 3, 4h, 4w]; output [B, Tq, h, w, n]
    int n, bn, n_tiles;
    int tiles_xp, tiles_y, npairs;
};

struct EmbedTile {
    int b, tq, y0, x0, n0;
};

// Pair tile i, this CTA's half (rank): column block 2 * xp + rank.
__device__ __forceinline__ EmbedTile decode_embed(const EmbedGeom &g, int i, uint32_t rank)
{
    EmbedTile e;
    const int nb = i % g.n_tiles; // output-channel tiles fastest: they read the same pixels
    int r = i / g.n_tiles;
    const int xp = r % g.tiles_xp;
    r /= g.tiles_xp;
    const int yb = r % g.tiles_y;
    r /= g.tiles_y;
    e.tq = r % g.Tq;
    e.b = r / g.Tq;
    e.y0 = yb * kTileRows;
    e.x0 = (2 * xp + (int)rank) * kTileCols;
    e.n0 = nb * g.bn;
    return e;
}

__device__ __forceinline__ float2 f2add(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 f2sub(float2 a, float2 b) { return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a); }

// Two levels of the causal full-packet Haar transform along one axis on four pairs,
// unnormalized, natural order k = 2 * b2 + b1 (the planar patcher's butterflies).
__device__ __forceinline__ void wht4x2(float2 &a0, float2 &a1, float2 &a2, float2 &a3)
{
    const float2 l0 = f2add(a0, a1), h0 = f2sub(a0, a1), l1 = f2add(a2, a3), h1 = f2sub(a2, a3);
    a0 = f2add(l0, l1);
    a1 = f2add(h0, h1);
    a2 = f2sub(l0, l1);
    a3 = f2sub(h0, h1);
}

// Per-axis indices of subband g = 8 * s2 + s1, s = 4 * b_t + 2 * b_y + b_x (bit 1: high band).
__host__ __device__ constexpr int sb_kt(int g) { return 2 * ((g >> 3) >> 2) + ((g & 7) >> 2); }
__host__ __device__ constexpr int sb_ky(int g) { return 2 * (((g >> 3) >> 1) & 1) + (((g & 7) >> 1) & 1); }
__host__ __device__ constexpr int sb_kx(int g) { return 2 * ((g >> 3) & 1) + (g & 1); }

__device__ __forceinline__ void issue_pixels(const CUtensorMap *xmap, const EmbedTile &e, int c, uint32_t dst,
                                             uint32_t bar)
{
    mbar_expect_tx(bar, kPixBytes);
    tma_load_5d(dst, xmap, 4 * e.x0 - 8, 4 * e.y0 - 4, 4 * e.tq - 3, c, e.b, bar);
}

__global__ void __launch_bounds__(kEmbedThreads, 1)
patch_embed_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap bmap,
                   const __grid_constant__ CUtensorMap omap, __nv_bfloat16 *__restrict__ out, const EmbedGeom g)
{
    __shared__ __align__(8) uint64_t ffull[kFStages], fempty[kFStages], pfull[kPlanes], pempty[kPlanes], xfull,
        accf[2], acce[2], drain, hsync;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t base = (smem_addr(smem_raw) + 1023u) & ~1023u;
    const uint32_t fbytes = (uint32_t)(g.bn / 2) * kBK * 2; // this CTA's half of a filter K block
    const uint32_t fstage = kFGroup * fbytes;               // one filter stage
    const uint32_t fbase = base, pbase = fbase + kFStages * fstage, xbase = pbase + kPlanes * kPlaneBytes;
    const uint32_t ebase = xbase + kPixBytes;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const uint32_t ncols = tmem_cols(g.bn);
    const int pair = blockIdx.x >> 1, npair_ctas = gridDim.x >> 1;
    const int nplanes = 3 * g.C; // planes (and filter stages) per tile

    if (threadIdx.x == 0) {
        for (int s = 0; s < kFStages; ++s) {
            mbar_init(smem_addr(&ffull[s]), 1);
            mbar_init(smem_addr(&fempty[s]), 1);
        }
        for (int p = 0; p < kPlanes; ++p) {
            mbar_init(smem_addr(&pfull[p]), 8); // 4 Haar warps in each CTA
            mbar_init(smem_addr(&pempty[p]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_addr(&accf[a]), 1);
            mbar_init(smem_addr(&acce[a]), 8);
        }
        mbar_init(smem_addr(&xfull), 1);
        mbar_init(smem_addr(&drain), 1);
        mbar_init(smem_addr(&hsync), kHaarThreads);
        abort_s = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc_pair(smem_addr(&tmem_base_s), ncols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    volatile int *abort = &abort_s;

    if (warp == 0 && lane == 0) {
        // This CTA's half of the filter, the three K blocks of one plane per stage in the tile's K
        // order; counted on the leader's barrier.
        uint32_t s = 0, ph = 0, issued = 0;
        bool ok = true;
        for (int i = pair; i < g.npairs && ok; i += npair_ctas) {
            const EmbedTile e = decode_embed(g, i, rank);
            for (int pl = 0; pl < nplanes; ++pl) {
                if (!wait_or_abort(smem_addr(&fempty[s]), ph ^ 1u, abort)) {
                    ok = false;
                    break;
                }
                const uint32_t fb = mapa_shared(smem_addr(&ffull[s]), 0);
                if (leader)
                    mbar_expect_tx(smem_addr(&ffull[s]), 2 * fstage);
                for (int dy = 0; dy < kFGroup; ++dy)
                    tma_load_2d_pair(fbase + s * fstage + dy * fbytes, &bmap, (pl * kFGroup + dy) * kBK,
                                     e.n0 + (int)rank * (g.bn / 2), fb);
                ++issued;
                if (++s == kFStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        if (!ok && leader)
            for (uint32_t j = issued > kFStages ? issued - kFStages : 0; j < issued; ++j)
                mbar_wait(smem_addr(&ffull[j % kFStages]), (j / kFStages) & 1u);
    } else if (warp == 1 && lane == 0 && leader) {
        // MMA issue for the pair.  This single thread is the pipeline's narrowest point (each
        // barrier test or commit costs it about as long as an MMA), so the loop keeps its ring
        // positions and descriptors as running values: per plane (c, dx) one wait and one commit
        // on the plane ring and one on the filter ring, around its 12 MMAs.
        const uint32_t idesc = idesc_bf16_f32(2 * kBM, g.bn);
        const uint64_t adesc0 = sw128_desc(pbase), bdesc0 = sw128_desc(fbase);
        uint32_t fs = 0, fph = 0, ps = 0, pph = 0, tc = 0;
        bool ok = true;
        for (int i = pair; i < g.npairs && ok; i += npair_ctas, ++tc) {
            const uint32_t acc = tc & 1u, use = tc >> 1;
            if (!wait_or_abort(smem_addr(&acce[acc]), (use & 1u) ^ 1u, abort))
                break;
            tc_fence_after();
            const uint32_t d = tmem + acc * (uint32_t)g.bn;
            for (int pl = 0; pl < nplanes && ok; ++pl) {
                if (!wait_or_abort(smem_addr(&pfull[ps]), pph, abort) ||
                    !wait_or_abort(smem_addr(&ffull[fs]), fph, abort)) {
                    ok = false;
                    break;
                }
                const uint64_t ad = adesc0 + ((ps * kPlaneBytes) >> 4), bd = bdesc0 + ((fs * fstage) >> 4);
#pragma unroll
                for (int dy = 0; dy < kFGroup; ++dy) {
                    const uint64_t a = ad + (uint64_t)(dy * 64), b = bd + (uint64_t)((dy * fbytes) >> 4);
                    umma_bf16_pair(d, a, b, idesc, (pl | dy) != 0);
                    umma_bf16_pair(d, a + 2, b + 2, idesc, 1u);
                    umma_bf16_pair(d, a + 4, b + 4, idesc, 1u);
                    umma_bf16_pair(d, a + 6, b + 6, idesc, 1u);
                }
                umma_commit_pair(smem_addr(&fempty[fs]), kPairMask);
                if (++fs == kFStages) {
                    fs = 0;
                    fph ^= 1u;
                }
                umma_commit_pair(smem_addr(&pempty[ps]), kPairMask);
                if (++ps == kPlanes) {
                    ps = 0;
                    pph ^= 1u;
                }
            }
            if (ok)
                umma_commit_pair(smem_addr(&accf[acc]), kPairMask);
        }
        umma_commit_pair(smem_addr(&drain), 0x1);
        mbar_wait(smem_addr(&drain), 0u);
    } else if (warp >= 2 && warp < 6) {
        // Epilogue of this CTA's tile.
        const int q = warp & 3, row = 32 * q + lane;
        const int r = row / kTileCols, jj = row - r * kTileCols;
        const uint32_t acce0 = mapa_shared(smem_addr(&acce[0]), 0), acce1 = mapa_shared(smem_addr(&acce[1]), 0);
        const uint32_t stage = ebase + (uint32_t)q * (kEmbedEpiBuf * 4096u);
        unsigned char *stage_ptr = smem_raw + (stage - smem_addr(smem_raw));
        uint32_t tc = 0, sbuf = 0;
        for (int i = pair; i < g.npairs; i += npair_ctas, ++tc) {
            const EmbedTile e = decode_embed(g, i, rank);
            const uint32_t acc = tc & 1u, use = tc >> 1;
            if (!wait_or_abort(smem_addr(&accf[acc]), use & 1u, abort))
                break;
            tc_fence_after();
            const int y = e.y0 + r, x = e.x0 + jj, f = e.b * g.Tq + e.tq;
            __nv_bfloat16 *o = out + (((int64_t)f * g.h + y) * g.w + x) * g.n + e.n0;
            store_tile<kEmbedEpiBuf>(tmem + acc * (uint32_t)g.bn, q, lane, &omap, f, e.y0, e.x0, e.n0, stage,
                                     stage_ptr, sbuf, o, y < g.h && x < g.w, g.bn);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(acc ? acce1 : acce0);
        }
        if (lane == 0)
            bulk_wait_all();
    } else if (warp >= 6) {
        // Haar warps of this CTA's tile.  Per colour, each of 90 threads transforms two adjacent
        // latent columns u0 = 2 up - 1, u0 + 1 (up = 0..4; u = -1 .. 8 relative to x0) of plane row
        // pr and writes each position into every plane dx whose window holds it (plane column
        // j = u + 1 - dx), plane by plane as slots free up.
        const int ht = threadIdx.x - kHaarFirst;
        const int pr = ht / 5, up = ht - 5 * pr, u0 = 2 * up - 1;
        const bool worker = ht < kPlaneRows * 5;
        uint32_t ci = 0, pi = 0, px_issued = 0; // colours started, planes made, pixel copies issued
        bool ok = true;
        int i = pair;
        if (ht == 0 && i < g.npairs) {
            issue_pixels(&xmap, decode_embed(g, i, rank), 0, xbase, smem_addr(&xfull));
            ++px_issued;
        }
        const unsigned char *pix = smem_raw + (xbase - smem_addr(smem_raw));
        for (; i < g.npairs && ok; i += npair_ctas) {
            const EmbedTile e = decode_embed(g, i, rank);
            for (int c = 0; c < g.C && ok; ++c, ++ci) {
                if (!wait_or_abort(smem_addr(&xfull), ci & 1u, abort)) {
                    ok = false;
                    break;
                }
                // Staged pixel columns of latent u: 4 (u + 2) .. + 3 (the box starts two blocks left of
                // x0); rows 4 pr ..; window 0 reads frame 0 (box frame 3) four times.
                float2 v[4][4][4];
                if (worker) {
                    const int col = 4 * (u0 + 2);
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        const int fa = e.tq == 0 ? 3 : a;
#pragma unroll
                        for (int rr = 0; rr < 4; ++rr) {
                            const unsigned char *rowp = pix + ((fa * kPixRows + 4 * pr + rr) * kPixCols + col) * 2;
                            const uint2 p0 = *reinterpret_cast<const uint2 *>(rowp);
                            const uint2 p1 = *reinterpret_cast<const uint2 *>(rowp + 8);
                            v[a][rr][0] = make_float2(bf16_lo(p0.x), bf16_lo(p1.x));
                            v[a][rr][1] = make_float2(bf16_hi(p0.x), bf16_hi(p1.x));
                            v[a][rr][2] = make_float2(bf16_lo(p0.y), bf16_lo(p1.y));
                            v[a][rr][3] = make_float2(bf16_hi(p0.y), bf16_hi(p1.y));
                        }
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int rr = 0; rr < 4; ++rr)
                            wht4x2(v[a][rr][0], v[a][rr][1], v[a][rr][2], v[a][rr][3]);
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int d = 0; d < 4; ++d)
                            wht4x2(v[a][0][d], v[a][1][d], v[a][2][d], v[a][3][d]);
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                        for (int d = 0; d < 4; ++d)
                            wht4x2(v[0][rr][d], v[1][rr][d], v[2][rr][d], v[3][rr][d]);
                }
                // The 64 coefficients of both blocks as bf16 rows: k8 = 8 subbands (16 bytes) per word group.
                uint4 vlo[8], vhi[8];
                if (worker) {
                    const float2 eighth = make_float2(0.125f, 0.125f);
#pragma unroll
                    for (int k8 = 0; k8 < 8; ++k8) {
                        uint32_t lo[4], hi[4];
#pragma unroll
                        for (int uu = 0; uu < 4; ++uu) {
                            const int g0 = 8 * k8 + 2 * uu, g1 = g0 + 1;
                            const float2 a0 = __fmul2_rn(v[sb_kt(g0)][sb_ky(g0)][sb_kx(g0)], eighth);
                            const float2 a1 = __fmul2_rn(v[sb_kt(g1)][sb_ky(g1)][sb_kx(g1)], eighth);
                            lo[uu] = pack_bf16x2(a0.x, a1.x);
                            hi[uu] = pack_bf16x2(a0.y, a1.y);
                        }
                        vlo[k8] = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                        vhi[k8] = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                    }
                }
                // The coefficients are in registers: once every Haar thread is here (a barrier phase
                // per colour, its wait bounded like the others) the next colour's copy refills the
                // pixel buffer while the planes are written.
                mbar_arrive(smem_addr(&hsync));
                if (!wait_or_abort(smem_addr(&hsync), ci & 1u, abort)) {
                    ok = false;
                    break;
                }
                if (ht == 0) {
                    const bool last_c = c + 1 == g.C;
                    const int ni = last_c ? i + npair_ctas : i;
                    if (ni < g.npairs) {
                        fence_proxy_async_smem();
                        issue_pixels(&xmap, last_c ? decode_embed(g, ni, rank) : e, last_c ? 0 : c + 1, xbase,
                                     smem_addr(&xfull));
                        ++px_issued;
                    }
                }
                unsigned char *planes = smem_raw + (pbase - smem_addr(smem_raw));
                for (int dx = 0; dx < 3; ++dx, ++pi) {
                    const uint32_t slot = pi % kPlanes;
                    if (!wait_or_abort(smem_addr(&pempty[slot]), ((pi / kPlanes) & 1u) ^ 1u, abort)) {
                        ok = false;
                        break;
                    }
                    if (worker) {
                        unsigned char *plane = planes + slot * kPlaneBytes;
                        const int j0 = u0 + 1 - dx, j1 = j0 + 1;
                        if (j0 >= 0 && j0 < kTileCols) {
#pragma unroll
                            for (int k8 = 0; k8 < 8; ++k8)
                                *reinterpret_cast<uint4 *>(plane + sw128_offset(pr * kTileCols + j0, 8 * k8)) =
                                    vlo[k8];
                        }
                        if (j1 >= 0 && j1 < kTileCols) {
#pragma unroll
                            for (int k8 = 0; k8 < 8; ++k8)
                                *reinterpret_cast<uint4 *>(plane + sw128_offset(pr * kTileCols + j1, 8 * k8)) =
                                    vhi[k8];
                        }
                    }
                    fence_proxy_async_smem(); // the plane's writes are visible to the tensor cores
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive_cluster(mapa_shared(smem_addr(&pfull[slot]), 0));
                }
            }
        }
        if (ht == 0 && !ok) // a pixel copy issued and not yet waited for
            for (uint32_t j = ci; j < px_issued; ++j)
                mbar_wait(smem_addr(&xfull), j & 1u);
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, ncols);
    }
    if (threadIdx.x == 0 && *abort)
        atomicAdd(&g_conv_timeouts, 1u);
}

size_t embed_smem_bytes(int bn)
{
    return (size_t)kFStages * kFGroup * (bn / 2) * kBK * 2 + (size_t)kPlanes * kPlaneBytes + (size_t)kPixBytes +
           epi_bytes(kEmbedEpiBuf) + 1024;
}

// Packed filter: wp[n][(c * 3 + dx) * 3 + dy][g] = ws[n][dy][dx][g * C + c].
__global__ void pack_embed_weights_kernel(const __nv_bfloat16 *__restrict__ ws, __nv_bfloat16 *__restrict__ wp,
                                          int C, int64_t total)
{
    const int64_t o = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (o >= total)
        return;
    const int K = 576 * C;
    const int64_t n = o / K;
    const int kk = (int)(o - n * K), kb = kk / 64, gg = kk - kb * 64;
    const int c = kb / 9, dx = (kb / 3) % 3, dy = kb % 3;
    wp[o] = ws[((n * 3 + dy) * 3 + dx) * (int64_t)(64 * C) + gg * C + c];
}

} // namespace

bool conv_tc_eligible(int64_t Cin, int64_t Cout) { return tc_eligible(Cin, Cout); }

tok_status conv_tc_temporal(const void *x, const void *wt, void *y, int64_t B, int64_t T, int64_t h, int64_t w,
                            int64_t Cin, int64_t Cout, int64_t k, cudaStream_t stream)
{
    return conv_tc_launch(true, x, wt, y, B, T, h, w, Cin, Cout, k, stream);
}

tok_status conv_tc_spatial(const void *x, const void *ws, void *y, int64_t B, int64_t T, int64_t h, int64_t w,
                           int64_t Cin, int64_t Cout, int64_t k, cudaStream_t stream)
{
    return conv_tc_launch(false, x, ws, y, B, T, h, w, Cin, Cout, k, stream);
}

bool patch_embed_eligible(int64_t C, int64_t Cmid) { return C >= 1 && C <= 8 && tc_eligible(64 * C, Cmid); }

tok_status patch_embed_pack(const void *ws, void *wp, int64_t C, int64_t Cmid, cudaStream_t stream)
{
    const int64_t total = Cmid * 576 * C;
    if (total == 0)
        return TOK_OK;
    const int threads = 256;
    pack_embed_weights_kernel<<<(unsigned)((total + threads - 1) / threads), threads, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(ws), static_cast<__nv_bfloat16 *>(wp), (int)C, total);
    return launch_status();
}

tok_status patch_embed_launch(const void *x, const void *wp, void *y, int64_t B, int64_t C, int64_t T, int64_t H,
                              int64_t W, int64_t Cmid, cudaStream_t stream)
{
    EmbedGeom g{};
    g.B = (int)B;
    g.C = (int)C;
    g.Tq = (int)(1 + (T - 1) / 4);
    g.h = (int)(H / 4);
    g.w = (int)(W / 4);
    g.n = (int)Cmid;
    g.bn = Cmid <= 256 ? (int)Cmid : 256;
    g.n_tiles = (int)(Cmid / g.bn);
    g.tiles_xp = ((g.w + kTileCols - 1) / kTileCols + 1) / 2;
    g.tiles_y = (g.h + kTileRows - 1) / kTileRows;
    const int64_t npairs = B * g.Tq * (int64_t)g.tiles_xp * g.tiles_y * g.n_tiles;
    if (!fits_int(npairs))
        return TOK_ERR_SHAPE;
    g.npairs = (int)npairs;

    CUtensorMap xmap, bmap;
    const uint64_t xdims[5] = {(uint64_t)W, (uint64_t)H, (uint64_t)T, (uint64_t)C, (uint64_t)B};
    const uint64_t xstr[4] = {(uint64_t)W * 2, (uint64_t)H * W * 2, (uint64_t)T * H * W * 2,
                              (uint64_t)C * T * H * W * 2};
    const uint32_t xbox[5] = {kPixCols, kPixRows, kPixFrames, 1, 1};
    const uint64_t bdims[2] = {(uint64_t)(576 * C), (uint64_t)Cmid};
    const uint64_t bstr[1] = {(uint64_t)(576 * C) * 2};
    const uint32_t bbox[2] = {kBK, (uint32_t)(g.bn / 2)};
    CUtensorMap omap;
    const uint64_t odims[4] = {(uint64_t)Cmid, (uint64_t)g.w, (uint64_t)g.h, (uint64_t)(B * g.Tq)};
    const uint64_t ostr[3] = {(uint64_t)Cmid * 2, (uint64_t)g.w * Cmid * 2, (uint64_t)g.h * g.w * Cmid * 2};
    const uint32_t obox[4] = {(uint32_t)std::min<int64_t>(64, Cmid), kTileCols, 4, 1};
    if (!encode_tensor_map(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, x, xdims, xstr, xbox) ||
        !encode_tensor_map_sw128(&bmap, 2, wp, bdims, bstr, bbox) ||
        !encode_tensor_map_sw128(&omap, 4, y, odims, ostr, obox))
        return TOK_ERR_SHAPE;
    return launch_pairs(patch_embed_kernel, npairs, embed_smem_bytes(g.bn), kEmbedThreads, stream, xmap, bmap, omap,
                        static_cast<__nv_bfloat16 *>(y), g);
}

tok_status read_and_clear_conv_timeouts(cudaStream_t stream, unsigned int *count)
{
    unsigned int zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(count, g_conv_timeouts, sizeof(unsigned int), 0,
                                              cudaMemcpyDeviceToHost, stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    if (e == cudaSuccess && *count)
        e = cudaMemcpyToSymbolAsync(g_conv_timeouts, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, stream);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return TOK_ERR_CUDA;
    }
    return TOK_OK;
}

} // namespace tok

// ---------------------------------------------------------------------------
// C ABI of the fused patch embedding (declared in tok.h).
// ---------------------------------------------------------------------------
extern "C" tok_status tok_patch_embed_pack_weights(const void *ws, void *wp, int64_t C, int64_t Cmid,
                                                    cudaStream_t stream)
{
    using namespace tok;
    if (!patch_embed_eligible(C, Cmid))
        return TOK_ERR_SHAPE;
    if (!ws || !wp)
        return TOK_ERR_NULL;
    if (!aligned(ws, 2) || !aligned(wp, 16))
        return TOK_ERR_ALIGN;
    const int64_t bytes = Cmid * 576 * C * 2;
    if (overlaps(ws, bytes, wp, bytes))
        return TOK_ERR_ALIAS;
    return patch_embed_pack(ws, wp, C, Cmid, stream);
}

extern "C" tok_status tok_patch_embed_spatial(const void *x, const void *wp, void *y, int64_t B, int64_t C,
                                              int64_t T, int64_t H, int64_t W, int64_t Cmid, cudaStream_t stream)
{
    using namespace tok;
    if (B < 0 || T < 5 || T % 4 != 1 || H < 0 || W < 0 || H % 4 || W % 8 || !patch_embed_eligible(C, Cmid))
        return TOK_ERR_SHAPE;
    const int64_t Tq = 1 + (T - 1) / 4, h = H / 4, w = W / 4;
    int64_t nx, ny, pos;
    if (!prod_ok({B, C, T, H, W, 2}, &nx) || !prod_ok({B, Tq, h, w}, &pos) || !prod_ok({pos, Cmid, 2}, &ny) ||
        !fits_int(nx / 2) || !fits_int(ny / 2) || !fits_int(B * C) || H > 65536 || W > 65536)
        return TOK_ERR_SHAPE;
    if (pos == 0)
        return TOK_OK;
    if (!x || !wp || !y)
        return TOK_ERR_NULL;
    if (!aligned(x, 16) || !aligned(wp, 16) || !aligned(y, 16))
        return TOK_ERR_ALIGN;
    const int64_t nw = Cmid * 576 * C * 2;
    if (overlaps(x, nx, y, ny) || overlaps(wp, nw, y, ny))
        return TOK_ERR_ALIAS;
    return patch_embed_launch(x, wp, y, B, C, T, H, W, Cmid, stream);
}
