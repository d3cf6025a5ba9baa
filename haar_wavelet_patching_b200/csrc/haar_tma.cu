// TMA-fed Haar patcher / unpatcher for sm_100a (the main path).
//
// Same transform as haar.cu (sources: "NVIDIA Cosmos Tokenizer 完全指南" 7.1, 6.1,
// 7.3; "nvidia/Cosmos-Tokenize1-CV8x8x8-720p" model card, Model Architecture):
// every 4x4x4 pixel block maps to one coefficient in each of 64 channel groups
// through the per-axis 4-point transform of the two full-packet levels, with the
// two frame-0 replicas composed into "window 0 reads frame 0 four times".
//
// Design.  The path is HBM-bound, so what matters is how many bytes are in
// flight and how compact the region of memory being touched at any moment is.
// Work is cut into warp tiles of 64 horizontally adjacent blocks: one block row
// of one (b, c, t') window on video (4 frames x 4 rows x 256 pixels <-> 64
// planes x 64 coefficients), four block rows on images; 4096 elements either
// way.  Each CTA is one warp that owns KT consecutive tiles:
//   - lane 0 issues the KT TMA loads at once (a 3D box of pixels, or one 5D box
//     holding all 64 coefficient planes), each completing on its own mbarrier;
//   - the lanes take the tiles in order as they land, transform in registers
//     and store straight to global memory (4 bytes per plane per lane on the
//     forward: 128 contiguous bytes per warp per plane; 16 bytes per pixel row
//     on the inverse), predicated at the tensor edges.
// The grid is one-shot (a CTA per KT tiles, launched in tile order) rather than
// persistent: CTAs retire and are replaced in order, so the live working set
// stays a compact, moving window of the tensors, which measured better on
// B200 than persistent CTAs striding over the whole tensor.  Several
// single-warp CTAs share an SM; while one computes, the others' loads are in
// flight.  Each lane owns two horizontally adjacent blocks and keeps them in
// f32x2 pairs (block j in .x, block j+1 in .y), so every butterfly is one packed
// sm_100 add or fused multiply-add.  TMA zero-fills loads past the tensor edges.
//
// Waits are bounded: a barrier that does not complete within kWaitPolls polls
// makes the warp stop, drain what it issued and count a timeout that
// tok_check_device() reports.  Every load fills only this CTA's own shared memory.
#include <cstring>
#include <numeric>
#include <type_traits>

#include "tma.cuh"
#include "tok_common.cuh"
#include "tok_internal.h"

namespace tok {

// Kernels of this file that gave up on a barrier wait since the last check.
static __device__ unsigned int g_wait_timeouts = 0;

namespace {

constexpr int kTileBlocks = 64; // blocks across a warp tile (256 pixels)
constexpr int kGroupSalign = 16; // grouped rows: largest tile shift unit (16 bf16 = one 32-byte sector)
constexpr int kTileElems = 4096; // elements of a warp tile, on either side

template <typename T> struct WarpTiles {
    static constexpr int KT = sizeof(T) == 2 ? 4 : 2; // tiles per CTA, all loaded at once (32 KB)
};

struct TileGrid {
    FastDiv ntx, nty, nq, C; // tiles across, tile rows, latent frames processed, channels
    int T, Tq, tq0;          // frames, latent frames of the tensor, first latent frame processed
    int64_t H, W, h, w;
    uint32_t ntiles;
    // A window tq that is not the frame-0 replica window reads frames 4*tq + fbase .. + 3 of
    // the T-frame pixel tensor; window 0 is the replica window iff rep (fbase = -3, rep = 1
    // for the whole-video transform; fbase = 0, rep = 0 for a continuation chunk).  Extended
    // form (padding, cropping): frames past T - 1 are mirrored about it, and the pixel tensor
    // [T][H][W] may be smaller than the 4h x 4w blocks: the forward reads zeros there (TMA
    // fill), the inverse does not write there.
    int fbase, rep;
    int64_t n_src; // elements of the source tensor (the row form stops its copies at its end)
    // Video forward, box form: when a coefficient row is not a whole number of 32-byte sectors
    // (but a plane is), tiles of block row k = t' h + row start at column 64 tx - (k w mod salign)
    // (salign = 32 bytes / element, a power of two), so every warp's plane store starts on a
    // sector; else 0.
    int salign;
    // Inverse, row form: the plane stride is a multiple of 16 bytes, so the staged rows of one
    // block row (one per group) all sit at the same offset in their staged copies.
    int planes_share_offset;
    // Inverse with run-time store widths: the widest store (bytes, up to 16) that every pixel
    // row of the call allows (the destination's alignment and W elements' bytes).
    int sw;
};

// Source frame of frame f of a T-frame clip mirrored about its last frame (period 2(T-1)).
__device__ __forceinline__ int mirror_frame(int f, int T)
{
    if (f < T)
        return f;
    if (T == 1)
        return 0;
    const int period = 2 * (T - 1), r = f % period;
    return r < T ? r : period - r;
}

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

template <typename T> __device__ __forceinline__ T to_elem(float v);
template <> __device__ __forceinline__ float to_elem<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 to_elem<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// Global stores of results: two coefficients (blocks j, j+1) of one plane, or one
// pixel row of 8 elements (4 of block j, 4 of block j+1).
__device__ __forceinline__ void gstore_pair(__nv_bfloat16 *p, float2 v)
{
    *reinterpret_cast<uint32_t *>(p) = pack_bf16x2(v.x, v.y);
}
__device__ __forceinline__ void gstore_pair(float *p, float2 v) { *reinterpret_cast<float2 *>(p) = v; }
__device__ __forceinline__ void gstore_row(__nv_bfloat16 *p, const float2 *v)
{
    *reinterpret_cast<uint4 *>(p) = make_uint4(pack_bf16x2(v[0].x, v[1].x), pack_bf16x2(v[2].x, v[3].x),
                                               pack_bf16x2(v[0].y, v[1].y), pack_bf16x2(v[2].y, v[3].y));
}
__device__ __forceinline__ void gstore_row(float *p, const float2 *v)
{
    *reinterpret_cast<float4 *>(p) = make_float4(v[0].x, v[1].x, v[2].x, v[3].x);
    *reinterpret_cast<float4 *>(p + 4) = make_float4(v[0].y, v[1].y, v[2].y, v[3].y);
}

// ---------------------------------------------------------------------------
// Row form.  When the source's rows are not whole 16-byte units, a tile cannot be one
// TMA box (a tensor map needs 16-byte strides): its rows start at arbitrary 2- or
// 4-byte offsets.  The row form stages each source row of the tile with one bulk copy
// (cp.async.bulk: 16-byte-aligned addresses and size, no tensor map) from the 16-byte
// boundary at or below the row, with 16 bytes of slack, records the row's offset in
// its staged copy, and reads it back realigned.  The copy stops at the tensor's end
// (the issuing lane copies a last partial 16 bytes element by element).  Stores pick
// their width from the destination address at run time.
// ---------------------------------------------------------------------------
template <typename T, bool FWD, bool ROWS, int GR = 0> struct TileSmem {
    // The row form spends more instructions per tile (row offsets, realigned reads, stores of
    // run-time width), so it trades tiles per CTA for resident warps: ~17 KB per CTA.
    static constexpr int KT = !ROWS ? WarpTiles<T>::KT : sizeof(T) == 2 ? 2 : 1;
    static constexpr int NR = FWD ? 16 : 64;                              // staged rows of a tile
    static constexpr int ROW = (FWD ? 256 : 64) * (int)sizeof(T) + 16;     // a source row and its slack
    // Grouped rows (GR > 0): the 16 pixel rows' 256-element boxes, then 128 bytes of tail slots
    // per part (16 bytes per pixel row, in the order of the part's box rows).
    static constexpr int TILE = ROWS ? NR * ROW : kTileElems * (int)sizeof(T) + GR * 128;
    static constexpr int SMEM = KT * TILE + 8 * KT + (ROWS ? 64 * KT : 0); // tiles, barriers, row offsets
    static_assert(ROW % 16 == 0 && TILE % 16 == 0, "16-byte bulk-copy destinations");
};

// Realigned reads from a 16-byte-aligned staged row, without branches, so the rows of a
// tile are scheduled together: aligned 8- or 4-byte loads from at or below the offset,
// then a select of the word offset and a funnel shift of the byte offset.

// Eight elements (blocks j, j+1 of one pixel row) at byte offset o (even) -> four pairs, as
// SRow::load.  Reads 24 bytes from the 8-byte boundary at or below o.
__device__ __forceinline__ void staged_row8(const unsigned char *row, uint32_t o, __nv_bfloat16 *, float2 *v)
{
    const uint32_t base = o & ~7u, sh = (o & 3u) * 8u;
    const bool odd = (o & 4u) != 0;
    const uint2 a = *reinterpret_cast<const uint2 *>(row + base);
    const uint2 b = *reinterpret_cast<const uint2 *>(row + base + 8);
    const uint2 c = *reinterpret_cast<const uint2 *>(row + base + 16);
    const uint32_t x0 = odd ? a.y : a.x, x1 = odd ? b.x : a.y, x2 = odd ? b.y : b.x, x3 = odd ? c.x : b.y,
                   x4 = odd ? c.y : c.x;
    const uint32_t r0 = __funnelshift_r(x0, x1, sh), r1 = __funnelshift_r(x1, x2, sh);
    const uint32_t r2 = __funnelshift_r(x2, x3, sh), r3 = __funnelshift_r(x3, x4, sh);
    v[0] = make_float2(bf16_lo(r0), bf16_lo(r2));
    v[1] = make_float2(bf16_hi(r0), bf16_hi(r2));
    v[2] = make_float2(bf16_lo(r1), bf16_lo(r3));
    v[3] = make_float2(bf16_hi(r1), bf16_hi(r3));
}
// fp32: o is a multiple of 4; reads 40 bytes from the 8-byte boundary at or below o.
__device__ __forceinline__ void staged_row8(const unsigned char *row, uint32_t o, float *, float2 *v)
{
    const uint32_t base = o & ~7u;
    const bool odd = (o & 4u) != 0;
    float w[10];
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        const float2 q = *reinterpret_cast<const float2 *>(row + base + 8 * k);
        w[2 * k] = q.x;
        w[2 * k + 1] = q.y;
    }
#pragma unroll
    for (int d = 0; d < 4; ++d)
        v[d] = make_float2(odd ? w[d + 1] : w[d], odd ? w[d + 5] : w[d + 4]);
}

// Two adjacent elements (one coefficient of blocks j, j+1) at byte offset o.
__device__ __forceinline__ float2 staged_pair(const unsigned char *row, uint32_t o, __nv_bfloat16 *)
{
    const uint32_t *w = reinterpret_cast<const uint32_t *>(row + (o & ~3u));
    const uint32_t r = __funnelshift_r(w[0], w[1], (o & 3u) * 8u);
    return make_float2(bf16_lo(r), bf16_hi(r));
}
__device__ __forceinline__ float2 staged_pair(const unsigned char *row, uint32_t o, float *)
{
    const float *w = reinterpret_cast<const float *>(row + o); // o is a multiple of 4
    return make_float2(w[0], w[1]);
}

// ---------------------------------------------------------------------------
// Grouped-row form (bf16 video forward, W % 8 == 4, odd w).  A pixel row of W elements is
// not a whole number of 16-byte units, but GR = 2 of them are, so the tensor maps view each
// frame as [H / 2][2 W]: row y of the clip is part p = y % 2 of group row y / 2.  A tile
// takes one tensor box per part, [frames][its two rows of that part][256 elements], from the
// 16-byte boundary at or below the part's first pixel, and, for the part that does not start
// on the boundary (2 W = 8 mod 16 bytes: exactly one of the two), a tail box of the 8
// elements that follow it (16 bytes per pixel row).  A window that runs past the clip takes
// its frames one by one and its tails by one 16-byte bulk copy per pixel row.  The odd w is
// what makes this form pay: tiles may then start one block left of a pair boundary
// (TileGrid::salign), which keeps every coefficient-pair store aligned, where the row form
// falls back to element stores on every other block row.  (With an even w the row form,
// which keeps twice as many warps resident, measured faster.)
// ---------------------------------------------------------------------------

// Eight elements (blocks j, j+1 of one pixel row) at byte offset o (a multiple of 8) of a
// 512-byte box row m whose next 16 bytes are in the tail slot t -> four pairs, as SRow::load.
// Only lane 31 reaches the tail.
__device__ __forceinline__ void grouped_row8(const unsigned char *m, const unsigned char *t, uint32_t o, float2 *v)
{
    const uint2 lo = *reinterpret_cast<const uint2 *>(m + o);
    const uint32_t o2 = o + 8;
    const uint2 hi = *reinterpret_cast<const uint2 *>(o2 < 512 ? m + o2 : t + (o2 - 512));
    v[0] = make_float2(bf16_lo(lo.x), bf16_lo(hi.x));
    v[1] = make_float2(bf16_hi(lo.x), bf16_hi(hi.x));
    v[2] = make_float2(bf16_lo(lo.y), bf16_lo(hi.y));
    v[3] = make_float2(bf16_hi(lo.y), bf16_hi(hi.y));
}

// A pixel-row store whose alignment is known only at run time (the destination's rows are
// not multiples of 16 bytes): the widest stores the address allows.
__device__ __forceinline__ void gstore_row_any(__nv_bfloat16 *p, const float2 *v)
{
    const uint32_t w0 = pack_bf16x2(v[0].x, v[1].x), w1 = pack_bf16x2(v[2].x, v[3].x);
    const uint32_t w2 = pack_bf16x2(v[0].y, v[1].y), w3 = pack_bf16x2(v[2].y, v[3].y);
    const uintptr_t a = (uintptr_t)p;
    if ((a & 15) == 0) {
        *reinterpret_cast<uint4 *>(p) = make_uint4(w0, w1, w2, w3);
    } else if ((a & 7) == 0) {
        *reinterpret_cast<uint2 *>(p) = make_uint2(w0, w1);
        *reinterpret_cast<uint2 *>(p + 4) = make_uint2(w2, w3);
    } else if ((a & 3) == 0) {
        uint32_t *q = reinterpret_cast<uint32_t *>(p);
        q[0] = w0;
        q[1] = w1;
        q[2] = w2;
        q[3] = w3;
    } else {
        unsigned short *q = reinterpret_cast<unsigned short *>(p);
        const uint32_t w[4] = {w0, w1, w2, w3};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            q[2 * k] = (unsigned short)(w[k] & 0xFFFFu);
            q[2 * k + 1] = (unsigned short)(w[k] >> 16);
        }
    }
}
__device__ __forceinline__ void gstore_row_any(float *p, const float2 *v)
{
    const uintptr_t a = (uintptr_t)p;
    if ((a & 15) == 0) {
        gstore_row(p, v);
    } else if ((a & 7) == 0) {
#pragma unroll
        for (int k = 0; k < 4; k += 2) {
            *reinterpret_cast<float2 *>(p + k) = make_float2(v[k].x, v[k + 1].x);
            *reinterpret_cast<float2 *>(p + 4 + k) = make_float2(v[k].y, v[k + 1].y);
        }
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            p[k] = v[k].x;
            p[4 + k] = v[k].y;
        }
    }
}

// One pixel row of blocks j, j+1 (only block j when `both` is false, at the right edge of
// an odd w); the row form does not know the destination's alignment at compile time.
template <bool ROWS, typename T> __device__ __forceinline__ void store_pixel_row(T *p, const float2 *o, bool both)
{
    if constexpr (!ROWS) {
        gstore_row(p, o);
    } else if (both) {
        gstore_row_any(p, o);
    } else {
#pragma unroll
        for (int d = 0; d < 4; ++d)
            p[d] = to_elem<T>(o[d].x);
    }
}

// One pixel row of blocks j, j+1 in stores of SW bytes, SW a width every row of the call allows
// (TileGrid::sw): no test of the address.
template <int SW> __device__ __forceinline__ void store_row_width(__nv_bfloat16 *p, const float2 *v)
{
    const uint32_t w[4] = {pack_bf16x2(v[0].x, v[1].x), pack_bf16x2(v[2].x, v[3].x), pack_bf16x2(v[0].y, v[1].y),
                           pack_bf16x2(v[2].y, v[3].y)};
    if constexpr (SW >= 16) {
        *reinterpret_cast<uint4 *>(p) = make_uint4(w[0], w[1], w[2], w[3]);
    } else if constexpr (SW == 8) {
        *reinterpret_cast<uint2 *>(p) = make_uint2(w[0], w[1]);
        *reinterpret_cast<uint2 *>(p + 4) = make_uint2(w[2], w[3]);
    } else if constexpr (SW == 4) {
#pragma unroll
        for (int k = 0; k < 4; ++k)
            reinterpret_cast<uint32_t *>(p)[k] = w[k];
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            reinterpret_cast<unsigned short *>(p)[2 * k] = (unsigned short)(w[k] & 0xFFFFu);
            reinterpret_cast<unsigned short *>(p)[2 * k + 1] = (unsigned short)(w[k] >> 16);
        }
    }
}
template <int SW> __device__ __forceinline__ void store_row_width(float *p, const float2 *v)
{
    if constexpr (SW >= 16) {
        gstore_row(p, v);
    } else if constexpr (SW == 8) {
#pragma unroll
        for (int k = 0; k < 4; k += 2) {
            *reinterpret_cast<float2 *>(p + k) = make_float2(v[k].x, v[k + 1].x);
            *reinterpret_cast<float2 *>(p + 4 + k) = make_float2(v[k].y, v[k + 1].y);
        }
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            p[k] = v[k].x;
            p[4 + k] = v[k].y;
        }
    }
}

// Video: one block row (tile rows = 1); images: four block rows, done one after another.
template <bool VIDEO> struct TileRows {
    static constexpr int RW = VIDEO ? 1 : 4;
};

// FWD: pixels -> coefficients (the patcher, or with ADJ the unpatcher's adjoint);
// !FWD: coefficients -> pixels (the unpatcher, or with ADJ the patcher's adjoint).
// ADJ changes window 0 only: its time samples are (0, 0, 0, frame 0) instead of four
// copies of frame 0, and frame 0 receives the sum of the four rebuilt samples
// instead of the last one.  EXT: the extended form of TileGrid (padding, cropping,
// streaming chunks).  ROWS: the row form (source rows at any element offset, destination
// stores of any alignment, w may be odd); it reads the source through `src` (tg.n_src
// elements) instead of the tensor maps.  ANYST (inverse, box form): the source takes the box
// form but the pixel rows are not whole 16-byte units, so their stores take the row form's
// run-time widths.  GR = 2 (bf16 video forward): the grouped-row form above; its tiles may start one
// block left of a pair boundary (TileGrid::salign with an odd w), so a lane's pair can
// straddle column 0 or the last column, and such a lane stores its one block alone.
template <typename T, bool VIDEO, bool FWD, bool ADJ, bool EXT, bool ROWS, bool ANYST = false, int GR = 0>
__global__ void __launch_bounds__(32)
    haar_tma_kernel(const __grid_constant__ CUtensorMap xmap4, const __grid_constant__ CUtensorMap xmap1,
                    const __grid_constant__ CUtensorMap ymap, const __grid_constant__ CUtensorMap xtail4,
                    const __grid_constant__ CUtensorMap xtail1, const T *__restrict__ src, T *__restrict__ out,
                    const TileGrid tg)
{
    static_assert(!(EXT && ADJ), "the adjoints take the plain form");
    static_assert(!(ANYST && (FWD || ROWS)), "ANYST: the inverse's box form only");
    static_assert(GR == 0 || (GR == 2 && VIDEO && FWD && !ROWS && sizeof(T) == 2), "grouped rows: bf16 video forward");
    using P = TileSmem<T, FWD, ROWS, GR>;
    constexpr int KT = P::KT, WT = kTileBlocks;
    constexpr int RW = TileRows<VIDEO>::RW;
    constexpr int G = VIDEO ? 64 : 16;  // channel groups
    constexpr int NA = VIDEO ? 4 : 1;   // frames of a window
    constexpr int FRAME = 16 * RW * WT; // elements of one frame slice of the tile (4RW x 256)
    static_assert(G * RW * WT == kTileElems && NA * FRAME == kTileElems, "tile sizes");
    constexpr uint32_t TILE_BYTES = kTileElems * sizeof(T), FRAME_BYTES = FRAME * sizeof(T);
    constexpr float SCALE = VIDEO ? 0.125f : 0.25f;

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const int lane = threadIdx.x;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + KT * P::TILE);
    unsigned char *row_off = reinterpret_cast<unsigned char *>(bars + KT); // ROWS: [tile][staged row]

    // First block column of a tile (see TileGrid::salign).
    auto col0 = [&](int tx, int ty, int tq) -> int {
        if constexpr (FWD && VIDEO && !ROWS) {
            // salign is a power of two, so (k w) mod salign needs only the low bits of k w.
            if (tg.salign)
                return WT * tx - (int)((((uint32_t)tq * (uint32_t)tg.h + (uint32_t)ty) * (uint32_t)tg.w) &
                                       (uint32_t)(tg.salign - 1));
        }
        return WT * tx;
    };

    auto decode = [&](uint32_t n, int &tx, int &ty, int &tq, int64_t &bc) {
        const uint32_t q1 = tg.ntx.div(n), q2 = tg.nty.div(q1), q3 = tg.nq.div(q2);
        tx = (int)(n - q1 * tg.ntx.d);
        ty = (int)(q1 - q2 * tg.nty.d);
        tq = tg.tq0 + (int)(q2 - q3 * tg.nq.d);
        bc = q3;
    };

    const uint32_t first = blockIdx.x * (uint32_t)KT;
    const int count = (int)min((uint32_t)KT, tg.ntiles - first); // tiles of this CTA

    if constexpr (ROWS) {
        if (lane == 0) {
            for (int s = 0; s < KT; ++s)
                mbar_init(smem_addr(bars + s), 1);
            fence_barrier_init();
        }
        __syncwarp();
        constexpr int VE = 16 / (int)sizeof(T); // elements per 16 bytes
        constexpr int PER = FWD ? 1 : 2;        // staged rows issued per lane (16 or 64 per tile)
        for (int s = 0; s < count; ++s) {
            int tx, ty, tq;
            int64_t bc;
            decode(first + s, tx, ty, tq, bc);
            const bool replica = VIDEO && tg.rep && tq == 0;
            int64_t start[PER]; // byte offset of each staged row in the source (16-byte aligned)
            uint32_t nbulk[PER];
            bool ok[PER], zero[PER]; // zero: a row past the clip's last row that the transform reads
            uint32_t tx_bytes = 0;
#pragma unroll
            for (int k = 0; k < PER; ++k) {
                const int r = lane + 32 * k;
                int64_t off = 0;
                if constexpr (FWD) {
                    // Staged row r: frame slot r / (4 RW), pixel row 4 RW ty + r % (4 RW).
                    const int a = r / (4 * RW);
                    const int64_t y = (int64_t)4 * RW * ty + r % (4 * RW);
                    int64_t f = 0;
                    bool loaded = r < P::NR && y < tg.H;
                    if (VIDEO && replica)
                        loaded = loaded && a == 0; // window 0 reads frame 0 only
                    else if (VIDEO)
                        f = EXT ? mirror_frame(4 * tq + tg.fbase + a, tg.T) : 4 * tq + tg.fbase + a;
                    ok[k] = loaded;
                    zero[k] = EXT && r < P::NR && y >= tg.H && !(VIDEO && replica && a != 0);
                    off = ((bc * tg.T + f) * tg.H + y) * tg.W + (int64_t)4 * WT * tx;
                } else {
                    // Staged row r: group r / RW, block row RW ty + r % RW.
                    const int g = r / RW;
                    const int64_t row = (int64_t)RW * ty + r % RW;
                    const int64_t b = tg.C.div((uint32_t)bc), c = bc - b * tg.C.d;
                    const int64_t plane = (int64_t)tg.Tq * tg.h * tg.w;
                    ok[k] = row < tg.h;
                    zero[k] = false;
                    off = ((b * G + g) * tg.C.d + c) * plane + ((int64_t)tq * tg.h + row) * tg.w + (int64_t)WT * tx;
                }
                const int mis = (int)(off % VE);
                start[k] = (off - mis) * (int64_t)sizeof(T);
                // Bytes the bulk copy takes: the staged row, or up to the last 16-byte boundary
                // before the tensor's end (a valid row starts before the end).
                const int64_t avail = tg.n_src * (int64_t)sizeof(T) - start[k];
                nbulk[k] = !ok[k] ? 0u : avail >= P::ROW ? (uint32_t)P::ROW : (uint32_t)(avail & ~(int64_t)15);
                // A row that is not loaded is staged as zeros where its values are used (rows past
                // the clip's last row on the padded forward); elsewhere its results are never
                // stored and it is read at offset 0 of its (stale) staging row.
                if (r < P::NR)
                    row_off[s * 64 + r] = ok[k] ? (unsigned char)(mis * (int)sizeof(T)) : (unsigned char)0;
                tx_bytes += __reduce_add_sync(0xFFFFFFFFu, nbulk[k]);
            }
            const uint32_t bar = smem_addr(bars + s);
            if (lane == 0)
                mbar_expect_tx(bar, tx_bytes);
            __syncwarp();
            unsigned char *tile = smem_raw + s * P::TILE;
            const unsigned char *src_b = reinterpret_cast<const unsigned char *>(src);
#pragma unroll
            for (int k = 0; k < PER; ++k) {
                unsigned char *dst = tile + (lane + 32 * k) * P::ROW;
                if (!ok[k]) {
                    if (zero[k])
                        for (int b = 0; b < P::ROW; b += 16)
                            *reinterpret_cast<uint4 *>(dst + b) = make_uint4(0u, 0u, 0u, 0u);
                    continue;
                }
                if (nbulk[k] > 0)
                    bulk_load(smem_addr(dst), src_b + start[k], nbulk[k], bar);
                if (nbulk[k] < (uint32_t)P::ROW) {
                    // The row reaches the tensor's last, partial 16 bytes: copy those elements.
                    const int64_t end = min(tg.n_src * (int64_t)sizeof(T) - start[k], (int64_t)P::ROW);
                    for (int64_t b = nbulk[k]; b < end; b += (int64_t)sizeof(T))
                        *reinterpret_cast<T *>(dst + b) = *reinterpret_cast<const T *>(src_b + start[k] + b);
                }
            }
        }
    } else if constexpr (GR != 0) {
        if (lane == 0) {
            for (int s = 0; s < KT; ++s)
                mbar_init(smem_addr(bars + s), 1);
            fence_barrier_init();
        }
        __syncwarp();
        constexpr int R = 4 * RW / GR;                                  // rows of a part in one frame slice
        constexpr uint32_t PART = (uint32_t)kTileElems * sizeof(T) / GR; // bytes of one part's box
        constexpr uint32_t TAILS = (uint32_t)kTileElems * sizeof(T);     // the tail slots: 128 bytes per part
        for (int s = 0; s < count; ++s) {
            int tx, ty, tq;
            int64_t bc;
            decode(first + s, tx, ty, tq, bc);
            const int x0 = 4 * col0(tx, ty, tq); // first pixel column (may be negative: TMA fills zeros)
            const bool replica = VIDEO && tg.rep && tq == 0;
            const bool mirrored = VIDEO && EXT && !replica && 4 * tq + tg.fbase + 3 >= tg.T;
            const uint32_t bar = smem_addr(bars + s);
            unsigned char *tile = smem_raw + s * P::TILE;
            const int z0 = (int)(bc * tg.T), gy = R * ty; // frame of the clip, group row of the tile
            if (!mirrored) {
                // One box per part and one tail box per part that does not start on a 16-byte
                // boundary, from one window of frames: all issued by lane 0.
                if (lane == 0) {
                    const int nf = VIDEO && !replica ? NA : 1;
                    const int z = !VIDEO || replica ? z0 : z0 + 4 * tq + tg.fbase;
                    const CUtensorMap *mrow = nf == 1 ? &xmap1 : &xmap4, *mtail = nf == 1 ? &xtail1 : &xtail4;
                    uint32_t nmis = 0;
#pragma unroll
                    for (int pt = 0; pt < GR; ++pt)
                        nmis += ((x0 + pt * (int)tg.W) & 7) != 0;
                    mbar_expect_tx(bar, (uint32_t)nf * (FRAME_BYTES + nmis * R * 16u));
#pragma unroll
                    for (int pt = 0; pt < GR; ++pt) {
                        const int xq = x0 + pt * (int)tg.W, xb = xq - (xq & 7);
                        tma_load_3d(smem_addr(tile + pt * PART), mrow, xb, gy, z, bar);
                        if (xq & 7)
                            tma_load_3d(smem_addr(tile + TAILS + pt * 128), mtail, xb + 4 * WT, gy, z, bar);
                    }
                }
            } else {
                // A window that runs past the clip: frame by frame, mirrored about the last frame;
                // lanes 0 .. 15 copy the tails of staged row `lane` (frame slot a, pixel row yi).
                const unsigned char *src_b = reinterpret_cast<const unsigned char *>(src);
                const int a = lane / (4 * RW), yi = lane % (4 * RW), part = yi % GR;
                const int64_t y = (int64_t)4 * RW * ty + yi;
                const int f = mirror_frame(4 * tq + tg.fbase + a, tg.T);
                const int xp = x0 + part * (int)tg.W;
                const int mis = xp & 7; // elements from the 16-byte boundary below the row's first pixel
                const int64_t tstart = (((bc * tg.T + f) * tg.H + (y - part)) * tg.W + (xp - mis) + 4 * WT) *
                                       (int64_t)sizeof(T); // the 16 bytes after the part's box
                const bool want = lane < 16 && y < tg.H && mis != 0;
                const int64_t avail = tg.n_src * (int64_t)sizeof(T) - tstart;
                const uint32_t nbulk = want && avail >= 16 ? 16u : 0u;
                const uint32_t tail_bytes = __reduce_add_sync(0xFFFFFFFFu, nbulk);
                unsigned char *tslot = tile + TAILS + part * 128 + (a * R + yi / GR) * 16;
                if (lane == 0)
                    mbar_expect_tx(bar, (uint32_t)NA * FRAME_BYTES + tail_bytes);
                __syncwarp();
                if (lane == 0) {
#pragma unroll
                    for (int pt = 0; pt < GR; ++pt) {
                        const int xq = x0 + pt * (int)tg.W, xb = xq - (xq & 7);
                        for (int fa = 0; fa < NA; ++fa)
                            tma_load_3d(smem_addr(tile + pt * PART + fa * R * 512), &xmap1, xb, gy,
                                        z0 + mirror_frame(4 * tq + tg.fbase + fa, tg.T), bar);
                    }
                }
                if (nbulk) {
                    bulk_load(smem_addr(tslot), src_b + tstart, 16u, bar);
                } else if (lane < 16) {
                    // No copy: zeros (rows past the clip read as zeros), or the tensor's last,
                    // partial 16 bytes element by element.
                    *reinterpret_cast<uint4 *>(tslot) = make_uint4(0u, 0u, 0u, 0u);
                    if (want)
                        for (int64_t e = 0; e < avail; e += (int64_t)sizeof(T))
                            *reinterpret_cast<T *>(tslot + e) = *reinterpret_cast<const T *>(src_b + tstart + e);
                }
            }
        }
    } else if (lane == 0) {
        for (int s = 0; s < KT; ++s)
            mbar_init(smem_addr(bars + s), 1);
        fence_barrier_init();
        for (int s = 0; s < count; ++s) {
            int tx, ty, tq;
            int64_t bc;
            decode(first + s, tx, ty, tq, bc);
            const int x0 = 4 * col0(tx, ty, tq); // first pixel column (may be negative: TMA fills zeros)
            const uint32_t dst = smem_addr(smem_raw + s * P::TILE), bar = smem_addr(bars + s);
            if constexpr (FWD && EXT && VIDEO) {
                if (tg.rep && tq == 0) {
                    mbar_expect_tx(bar, FRAME_BYTES);
                    tma_load_3d(dst, &xmap1, x0, 4 * RW * ty, (int)(bc * tg.T), bar);
                } else if (4 * tq + tg.fbase + 3 < tg.T) {
                    mbar_expect_tx(bar, NA * FRAME_BYTES);
                    tma_load_3d(dst, &xmap4, x0, 4 * RW * ty, (int)(bc * tg.T + 4 * tq + tg.fbase), bar);
                } else {
                    // The window runs past the clip: frame by frame, mirrored about the last frame.
                    mbar_expect_tx(bar, NA * FRAME_BYTES);
                    for (int a = 0; a < NA; ++a)
                        tma_load_3d(dst + a * FRAME_BYTES, &xmap1, x0, 4 * RW * ty,
                                    (int)(bc * tg.T + mirror_frame(4 * tq + tg.fbase + a, tg.T)), bar);
                }
            } else if constexpr (FWD) {
                if (VIDEO && !(tg.rep && tq == 0)) {
                    mbar_expect_tx(bar, NA * FRAME_BYTES);
                    tma_load_3d(dst, &xmap4, x0, 4 * RW * ty, (int)(bc * tg.T + 4 * tq + tg.fbase), bar);
                } else {
                    mbar_expect_tx(bar, FRAME_BYTES);
                    tma_load_3d(dst, &xmap1, x0, 4 * RW * ty, (int)(bc * tg.T), bar);
                }
            } else {
                const int b = (int)tg.C.div((uint32_t)bc), c = (int)(bc - (int64_t)b * tg.C.d);
                mbar_expect_tx(bar, TILE_BYTES);
                tma_load_5d(dst, &ymap, WT * tx, RW * ty, tq, c, G * b, bar);
            }
        }
    }
    __syncwarp();

    int s = 0;
    for (; s < count; ++s) {
        const bool ok = mbar_wait(smem_addr(bars + s), 0u);
        if (__any_sync(0xFFFFFFFFu, !ok))
            break;
        int tx, ty, tq;
        int64_t bc;
        decode(first + s, tx, ty, tq, bc);
        const unsigned char *tile = smem_raw + s * P::TILE;
        const T *tin = reinterpret_cast<const T *>(tile);
        const int64_t j0 = (int64_t)col0(tx, ty, tq) + 2 * lane; // this lane's first block column
        // Some block of this lane's pair is in the tensor (the grouped form's shifted tiles can
        // put block j0 = -1 left of column 0); both are (a pair store may be used).
        const bool col_ok = (GR ? j0 >= -1 : j0 >= 0) && j0 < tg.w;
        const bool interior = j0 >= 0 && j0 + 1 < tg.w;
        const bool pair_ok = !ROWS || j0 + 1 < tg.w;    // block j0 + 1 exists (w is even outside the row form)
        const bool replica = VIDEO && tg.rep && tq == 0; // window 0 of a video

#pragma unroll
        for (int rw = 0; rw < RW; ++rw) {
            float2 v[NA][4][4]; // FWD: [t][y][x] pixels -> [kt][ky][kx]; INV: the reverse
            if constexpr (FWD) {
#pragma unroll
                for (int a = 0; a < NA; ++a) {
                    const int fa = replica ? 0 : a; // window 0 reads frame 0 four times
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        if (ADJ && VIDEO && tq == 0 && a != 3) {
#pragma unroll
                            for (int d = 0; d < 4; ++d)
                                v[a][rr][d] = make_float2(0.0f, 0.0f);
                        } else if constexpr (ROWS) {
                            // Rows past the clip's last row were staged as zeros.
                            const int r = fa * 4 * RW + 4 * rw + rr;
                            staged_row8(tile + r * P::ROW, row_off[s * 64 + r] + lane * 8 * (uint32_t)sizeof(T),
                                        (T *)nullptr, v[a][rr]);
                        } else if constexpr (GR != 0) {
                            // Pixel row yi of frame slot fa: row fa * R + yi / GR of part yi % GR's
                            // box and of its tail slots.
                            constexpr int R = 4 * RW / GR;
                            constexpr uint32_t PART = (uint32_t)kTileElems * sizeof(T) / GR;
                            const int yi = 4 * rw + rr, pt = yi % GR;
                            const int x0 = 4 * col0(tx, ty, tq);
                            const uint32_t o = (uint32_t)((x0 + pt * (int)tg.W) & 7) * (uint32_t)sizeof(T) +
                                               16u * (uint32_t)lane;
                            grouped_row8(tile + pt * PART + (fa * R + yi / GR) * 512,
                                             tile + kTileElems * sizeof(T) + pt * 128 + (fa * R + yi / GR) * 16, o,
                                             v[a][rr]);
                        } else {
                            SRow<T>::load(tin + (fa * 4 * RW + 4 * rw + rr) * 4 * WT + 8 * lane, v[a][rr]);
                        }
                    }
                }
                if constexpr (EXT && (ROWS || GR != 0)) {
                    // Columns past the clip's last column read as zeros (a staged row or a part's
                    // box runs on into the next pixel row): one test per tile row, after all its
                    // reads, so that no branch separates them.
                    const int64_t c0 = (GR ? (int64_t)4 * col0(tx, ty, tq) : (int64_t)4 * WT * tx) + 8 * lane;
                    if (c0 + 8 > tg.W) {
#pragma unroll
                        for (int a = 0; a < NA; ++a)
#pragma unroll
                            for (int rr = 0; rr < 4; ++rr)
#pragma unroll
                                for (int d = 0; d < 4; ++d) {
                                    if (c0 + d >= tg.W)
                                        v[a][rr][d].x = 0.0f;
                                    if (c0 + 4 + d >= tg.W)
                                        v[a][rr][d].y = 0.0f;
                                }
                    }
                }
            } else {
                auto put = [&](int g, float2 p) {
                    if constexpr (VIDEO)
                        v[kt_of(g)][ky_of(g)][kx_of(g)] = p;
                    else
                        v[0][ky2_of(g)][kx2_of(g)] = p;
                };
                if constexpr (ROWS) {
                    // When the plane stride is a multiple of 16 bytes, the G staged rows of this block
                    // row share one offset: hoisted, and one aligned load per pair when it allows.
                    const uint32_t o0 = row_off[s * 64 + rw] + lane * 2 * (uint32_t)sizeof(T);
                    const unsigned char *rows0 = tile + rw * P::ROW;
                    if (tg.planes_share_offset && (o0 & (2 * sizeof(T) - 1)) == 0) {
#pragma unroll
                        for (int g = 0; g < G; ++g)
                            put(g, SRow<T>::load_pair(reinterpret_cast<const T *>(rows0 + g * RW * P::ROW + o0)));
                    } else if (tg.planes_share_offset) {
#pragma unroll
                        for (int g = 0; g < G; ++g)
                            put(g, staged_pair(rows0 + g * RW * P::ROW, o0, (T *)nullptr));
                    } else {
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const unsigned mb = row_off[s * 64 + g * RW + rw];
                            put(g, staged_pair(tile + (g * RW + rw) * P::ROW, mb + lane * 2 * (uint32_t)sizeof(T),
                                               (T *)nullptr));
                        }
                    }
                } else {
#pragma unroll
                    for (int g = 0; g < G; ++g)
                        put(g, SRow<T>::load_pair(tin + (g * RW + rw) * WT + 2 * lane));
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

            const int64_t row = (int64_t)ty * RW + rw; // block row
            bool pairs = true;
            if constexpr (FWD && (ROWS || GR != 0)) {
                // A pair store is aligned iff its element offset is even, which alternates with g
                // only when the plane stride is odd.  One warp-wide choice per tile row (taken before
                // any lane leaves; addresses only): pair stores when every lane with a whole pair
                // has its 64 pairs aligned, element stores otherwise.  A lane whose pair is cut by
                // the tensor's edge stores its one block alone either way.
                const int64_t b = tg.C.div((uint32_t)bc), c = bc - b * tg.C.d;
                const int64_t plane = (int64_t)tg.Tq * tg.h * tg.w;
                const T *yq = out + (b * G * tg.C.d + c) * plane + ((int64_t)tq * tg.h + row) * tg.w + j0;
                const uintptr_t amask = 2 * sizeof(T) - 1;
                pairs = __all_sync(0xFFFFFFFFu, !interior || (((uintptr_t)yq & amask) == 0 &&
                                                              ((uintptr_t)(yq + tg.C.d * plane) & amask) == 0));
            }
            if (!col_ok || row >= tg.h)
                continue;
            if constexpr (FWD) {
                // y[b][g*C + c][tq][row][j0 .. j0+1]; the 64 planes are C*plane elements apart, a
                // 32-bit stride (checked on the host), so each address is one wide multiply-add.
                const int64_t b = tg.C.div((uint32_t)bc), c = bc - b * tg.C.d;
                const int64_t plane = (int64_t)tg.Tq * tg.h * tg.w;
                const uint32_t cstride = (uint32_t)(tg.C.d * plane);
                T *yp = out + (b * G * tg.C.d + c) * plane + ((int64_t)tq * tg.h + row) * tg.w + j0;
                if constexpr (ROWS || GR != 0) {
                    if (pairs && interior) {
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const float2 p = VIDEO ? v[kt_of(g)][ky_of(g)][kx_of(g)] : v[0][ky2_of(g)][kx2_of(g)];
                            gstore_pair(yp + (uint64_t)((uint32_t)g * cstride), __fmul2_rn(p, scale));
                        }
                    } else {
                        const bool first_ok = j0 >= 0, second_ok = j0 + 1 < tg.w;
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            const float2 q = __fmul2_rn(
                                VIDEO ? v[kt_of(g)][ky_of(g)][kx_of(g)] : v[0][ky2_of(g)][kx2_of(g)], scale);
                            T *dst = yp + (uint64_t)((uint32_t)g * cstride);
                            if (first_ok)
                                dst[0] = to_elem<T>(q.x);
                            if (second_ok)
                                dst[1] = to_elem<T>(q.y);
                        }
                    }
                } else {
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float2 p = VIDEO ? v[kt_of(g)][ky_of(g)][kx_of(g)] : v[0][ky2_of(g)][kx2_of(g)];
                        gstore_pair(yp + (uint64_t)((uint32_t)g * cstride), __fmul2_rn(p, scale));
                    }
                }
            } else {
                // x[bc][frame][4*row + rr][4*j0 .. 4*j0 + 7]; window 0 keeps its last frame only
                // (the adjoint: the sum of its four frames).
                T *xb = out + (bc * tg.T) * tg.H * tg.W + (4 * row) * tg.W + 4 * j0;
                if (ADJ && replica) {
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        float2 o[4];
#pragma unroll
                        for (int d = 0; d < 4; ++d)
                            o[d] = __fmul2_rn(add2(add2(add2(v[0][rr][d], v[1][rr][d]), v[2][rr][d]), v[3][rr][d]),
                                              scale);
                        store_pixel_row<ROWS || ANYST>(xb + rr * tg.W, o, pair_ok);
                    }
                    continue;
                }
                // Run-time store widths, both blocks' pixels inside the crop: every row stored at the
                // call's one width, with no test per row.  (Not in the row form's extended calls:
                // there the second copy of the store code cost more than the tests it saves.)
                const bool uniform = ((ROWS && !EXT) || ANYST) && pair_ok &&
                                     (!EXT || (4 * row + 3 < tg.H && 4 * j0 + 8 <= tg.W));
                if (uniform) {
                    auto put_all = [&](auto width) {
                        constexpr int SW = decltype(width)::value;
#pragma unroll
                        for (int a = 0; a < NA; ++a) {
                            if (replica && a != 3)
                                continue;
                            const int64_t f = !VIDEO ? 0 : replica ? 0 : 4 * tq + tg.fbase + a;
                            if (EXT && f >= tg.T) // cropped frames
                                continue;
#pragma unroll
                            for (int rr = 0; rr < 4; ++rr) {
                                float2 o[4];
#pragma unroll
                                for (int d = 0; d < 4; ++d)
                                    o[d] = __fmul2_rn(v[a][rr][d], scale);
                                store_row_width<SW>(xb + f * tg.H * tg.W + rr * tg.W, o);
                            }
                        }
                    };
                    if (tg.sw >= 16)
                        put_all(std::integral_constant<int, 16>());
                    else if (tg.sw == 8)
                        put_all(std::integral_constant<int, 8>());
                    else if (tg.sw == 4)
                        put_all(std::integral_constant<int, 4>());
                    else
                        put_all(std::integral_constant<int, 2>());
                } else {
#pragma unroll
                    for (int a = 0; a < NA; ++a) {
                        if (replica && a != 3)
                            continue;
                        const int64_t f = !VIDEO ? 0 : replica ? 0 : 4 * tq + tg.fbase + a;
                        if (EXT && f >= tg.T) // cropped frames
                            continue;
#pragma unroll
                        for (int rr = 0; rr < 4; ++rr) {
                            float2 o[4];
#pragma unroll
                            for (int d = 0; d < 4; ++d)
                                o[d] = __fmul2_rn(v[a][rr][d], scale);
                            T *dst = xb + f * tg.H * tg.W + rr * tg.W;
                            if (!EXT) {
                                store_pixel_row<ROWS || ANYST>(dst, o, pair_ok);
                            } else if (4 * row + rr < tg.H) { // cropped rows and columns
                                const int64_t col = 4 * j0;
                                if (col + 8 <= tg.W) {
                                    store_pixel_row<ROWS || ANYST>(dst, o, true);
                                } else {
#pragma unroll
                                    for (int d = 0; d < 8; ++d)
                                        if (col + d < tg.W)
                                            dst[d] = to_elem<T>(d < 4 ? o[d].x : o[d - 4].y);
                                }
                            }
                        }
                    }
                }
            }
        }
    }

    if (s < count && lane == 0) {
        // A wait ran out: drain the loads still in flight (each wait again bounded), then report.
        for (int r = s; r < count; ++r)
            mbar_wait(smem_addr(bars + r), 0u);
        atomicAdd(&g_wait_timeouts, 1u);
    }
    __syncwarp();
}

// ---------------------------------------------------------------------------
// Channels-last patcher: y [B, Tq, h, w, G*C] (G = 64 on video, 16 on images),
// channel g*C + c as in the planar layout, so a block's G*C coefficients are
// contiguous.  A tile is one block row (four on images) of 64 blocks across with
// all NC input channels on one barrier: NC TMA box loads; when the pixel rows are
// not whole 16-byte units, 3 NC pair-row boxes on video (PAIRS) or 16 NC row copies on
// images (ROWS), both below.  Per channel, each lane
// transforms its two blocks as in the planar kernel and, once the warp has read
// that channel's pixels, writes the results back over them as [row][g][block]
// pairs, rows padded to 66 elements (4-byte shared stores, consecutive across
// lanes).  The copy-out gives each lane a (block pair, 16-byte piece of the run):
// consecutive lanes take consecutive pieces, so a warp's store covers about two
// contiguous runs instead of 32 scattered sectors, and the padding puts the pieces'
// different (g, c) sources in different banks.  With odd w the last block of a row
// of blocks has no partner and is stored alone.
// ---------------------------------------------------------------------------
constexpr int kClPitch = 66; // staged row length in elements (64 blocks + 2 of padding)

template <typename T, int NC, bool ROWS = false> struct ClTiles {
    static constexpr int REGION_ELEMS = 64 * kClPitch; // >= kTileElems; a multiple of 128 bytes
    static constexpr int REGION_BYTES = REGION_ELEMS * sizeof(T);
    static constexpr int KT = (32768 / (NC * REGION_BYTES)) > 0 ? 32768 / (NC * REGION_BYTES) : 1;
    // Row form: a channel's 16 pixel rows staged at ROW bytes each (the row and 16 bytes of
    // slack) fill no more than its region; one offset byte per staged row after the barriers.
    static constexpr int ROW = 256 * (int)sizeof(T) + 16;
    static_assert(16 * ROW <= REGION_BYTES, "staged rows fit a channel's region");
    static constexpr int SMEM = KT * NC * REGION_BYTES + 8 * KT + (ROWS ? 16 * NC * KT : 0);
};

// ROWS: the pixel rows are not whole 16-byte units (bf16 with W % 8 == 4, so w is odd): each
// of a tile's 16 pixel rows per channel is staged by one bulk copy from the 16-byte boundary
// below it and read back realigned (as in the planar kernel's row form).  Staged at ROW-byte
// pitch, block row rw's pixels end where its results (rows of kClPitch) end or earlier, so the
// results still overwrite only pixels already read.
//
// PAIRS (video, bf16, W % 8 == 4): the same rows through tensor boxes.  Two pixel rows taken as
// one row of 2W elements have a 4W-byte stride, a 16-byte multiple, so the maps view each
// frame as [H/2][2W]: the even pixel rows of a tile are one box at x = 256 tx, the odd ones a
// box at x = W + 256 tx - 4 (the 16-byte boundary 4 elements before them: 2W = 8 mod 16
// bytes) and an 8-element box after it for the last 4 pixels.  Per channel: even rows at byte
// 0 of its region, odd rows at 4096, the tail boxes at 8192 (2080 bytes per frame in all).
template <typename T, bool VIDEO, int NC, bool ROWS, bool PAIRS>
__global__ void __launch_bounds__(32)
    haar_cl_kernel(const __grid_constant__ CUtensorMap xmap4, const __grid_constant__ CUtensorMap xmap1,
                   const __grid_constant__ CUtensorMap xtail4, const __grid_constant__ CUtensorMap xtail1,
                   const T *__restrict__ src, T *__restrict__ out, const TileGrid tg)
{
    static_assert(!PAIRS || (VIDEO && !ROWS && sizeof(T) == 2), "pair rows: bf16 video only");
    using P = ClTiles<T, NC, ROWS>;
    constexpr int KT = P::KT, WT = kTileBlocks;
    constexpr int RW = TileRows<VIDEO>::RW;
    constexpr int G = VIDEO ? 64 : 16;
    constexpr int NA = VIDEO ? 4 : 1;
    constexpr int FRAME = 16 * RW * WT;
    constexpr uint32_t FRAME_BYTES = FRAME * sizeof(T);
    constexpr float SCALE = VIDEO ? 0.125f : 0.25f;
    constexpr int VEC = 16 / (int)sizeof(T); // elements per 16-byte store
    static_assert((G * NC) % VEC == 0, "a block's run is whole 16-byte pieces");

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const int lane = threadIdx.x;
    T *buf = reinterpret_cast<T *>(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + KT * NC * P::REGION_BYTES);
    unsigned char *row_off = reinterpret_cast<unsigned char *>(bars + KT); // ROWS: [tile][channel][row]

    auto decode = [&](uint32_t n, int &tx, int &ty, int &tq, int64_t &b) {
        const uint32_t q1 = tg.ntx.div(n), q2 = tg.nty.div(q1), q3 = tg.nq.div(q2);
        tx = (int)(n - q1 * tg.ntx.d);
        ty = (int)(q1 - q2 * tg.nty.d);
        tq = (int)(q2 - q3 * tg.nq.d);
        b = q3;
    };

    const uint32_t first = blockIdx.x * (uint32_t)KT;
    const int count = (int)min((uint32_t)KT, tg.ntiles - first);

    if constexpr (ROWS) {
        if (lane == 0) {
            for (int s = 0; s < KT; ++s)
                mbar_init(smem_addr(bars + s), 1);
            fence_barrier_init();
        }
        __syncwarp();
        constexpr int VE = 16 / (int)sizeof(T);
        const unsigned char *src_b = reinterpret_cast<const unsigned char *>(src);
        for (int s = 0; s < count; ++s) {
            int tx, ty, tq;
            int64_t b;
            decode(first + s, tx, ty, tq, b);
            int64_t start[2];
            uint32_t nbulk[2];
            bool ok[2];
            uint32_t tx_bytes = 0;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                // Staged row r: channel r / 16, frame slot (r % 16) / (4 RW), pixel row
                // 4 RW ty + r % (4 RW); NC * 16 <= 64 rows per tile, two per lane.
                const int r = lane + 32 * k, c = r / 16, rr16 = r % 16, a = rr16 / (4 * RW);
                const int64_t y = (int64_t)4 * RW * ty + rr16 % (4 * RW);
                const bool replica = VIDEO && tq == 0;
                const int64_t f = !VIDEO || replica ? 0 : 4 * tq - 3 + a;
                ok[k] = r < 16 * NC && y < tg.H && !(replica && a != 0); // window 0 reads frame 0 only
                const int64_t off = (((b * NC + c) * tg.T + f) * tg.H + y) * tg.W + (int64_t)4 * WT * tx;
                const int mis = (int)(off % VE);
                start[k] = (off - mis) * (int64_t)sizeof(T);
                const int64_t avail = tg.n_src * (int64_t)sizeof(T) - start[k];
                nbulk[k] = !ok[k] ? 0u : avail >= P::ROW ? (uint32_t)P::ROW : (uint32_t)(avail & ~(int64_t)15);
                if (r < 16 * NC) // a row not loaded is never used for a stored result: offset 0
                    row_off[(s * NC + c) * 16 + rr16] = ok[k] ? (unsigned char)(mis * (int)sizeof(T)) : (unsigned char)0;
                tx_bytes += __reduce_add_sync(0xFFFFFFFFu, nbulk[k]);
            }
            const uint32_t bar = smem_addr(bars + s);
            if (lane == 0)
                mbar_expect_tx(bar, tx_bytes);
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                if (!ok[k])
                    continue;
                const int r = lane + 32 * k, c = r / 16, rr16 = r % 16;
                unsigned char *dst = reinterpret_cast<unsigned char *>(buf + (s * NC + c) * P::REGION_ELEMS) + rr16 * P::ROW;
                if (nbulk[k] > 0)
                    bulk_load(smem_addr(dst), src_b + start[k], nbulk[k], bar);
                if (nbulk[k] < (uint32_t)P::ROW) { // the tensor's last, partial 16 bytes
                    const int64_t end = min(tg.n_src * (int64_t)sizeof(T) - start[k], (int64_t)P::ROW);
                    for (int64_t e = nbulk[k]; e < end; e += (int64_t)sizeof(T))
                        *reinterpret_cast<T *>(dst + e) = *reinterpret_cast<const T *>(src_b + start[k] + e);
                }
            }
        }
    } else if (PAIRS && lane == 0) {
        for (int s = 0; s < KT; ++s)
            mbar_init(smem_addr(bars + s), 1);
        fence_barrier_init();
        for (int s = 0; s < count; ++s) {
            int tx, ty, tq;
            int64_t b;
            decode(first + s, tx, ty, tq, b);
            const uint32_t bar = smem_addr(bars + s);
            const bool full = tq > 0;
            mbar_expect_tx(bar, NC * (full ? NA : 1) * 2080u);
            const int x_even = 4 * WT * tx, x_odd = (int)tg.W + 4 * WT * tx - 4;
            for (int c = 0; c < NC; ++c) {
                const uint32_t dst = smem_addr(buf + (s * NC + c) * P::REGION_ELEMS);
                const int frame0 = (int)((b * NC + c) * tg.T), z = full ? frame0 + 4 * tq - 3 : frame0;
                const CUtensorMap *mrow = full ? &xmap4 : &xmap1, *mtail = full ? &xtail4 : &xtail1;
                tma_load_3d(dst, mrow, x_even, 2 * ty, z, bar);
                tma_load_3d(dst + 4096, mrow, x_odd, 2 * ty, z, bar);
                tma_load_3d(dst + 8192, mtail, x_odd + 4 * WT, 2 * ty, z, bar);
            }
        }
    } else if (lane == 0) {
        for (int s = 0; s < KT; ++s)
            mbar_init(smem_addr(bars + s), 1);
        fence_barrier_init();
        for (int s = 0; s < count; ++s) {
            int tx, ty, tq;
            int64_t b;
            decode(first + s, tx, ty, tq, b);
            const uint32_t bar = smem_addr(bars + s);
            const bool full = VIDEO && tq > 0;
            mbar_expect_tx(bar, NC * (full ? NA * FRAME_BYTES : FRAME_BYTES));
            for (int c = 0; c < NC; ++c) {
                const uint32_t dst = smem_addr(buf + (s * NC + c) * P::REGION_ELEMS);
                const int frame0 = (int)((b * NC + c) * tg.T);
                if (full)
                    tma_load_3d(dst, &xmap4, 4 * WT * tx, 4 * RW * ty, frame0 + 4 * tq - 3, bar);
                else
                    tma_load_3d(dst, &xmap1, 4 * WT * tx, 4 * RW * ty, frame0, bar);
            }
        }
    }
    __syncwarp();

    int s = 0;
    for (; s < count; ++s) {
        const bool ok = mbar_wait(smem_addr(bars + s), 0u);
        if (__any_sync(0xFFFFFFFFu, !ok))
            break;
        int tx, ty, tq;
        int64_t b;
        decode(first + s, tx, ty, tq, b);
        const bool replica = VIDEO && tq == 0;

#pragma unroll 1
        for (int c = 0; c < NC; ++c) {
            T *region = buf + (s * NC + c) * P::REGION_ELEMS;
            // Block rows in descending order: with the padded rows, the results of block row rw
            // reach past its own pixels into those of rows above it, which are then already read.
#pragma unroll
            for (int rr_ = 0; rr_ < RW; ++rr_) {
                const int rw = RW - 1 - rr_;
                float2 v[NA][4][4];
#pragma unroll
                for (int a = 0; a < NA; ++a) {
                    const int fa = replica ? 0 : a;
#pragma unroll
                    for (int rr = 0; rr < 4; ++rr) {
                        if constexpr (ROWS) {
                            const int sr = fa * 4 * RW + 4 * rw + rr;
                            staged_row8(reinterpret_cast<const unsigned char *>(region) + sr * P::ROW,
                                        row_off[(s * NC + c) * 16 + sr] + lane * 8 * (uint32_t)sizeof(T), (T *)nullptr,
                                        v[a][rr]);
                        } else if constexpr (PAIRS) {
                            // Pixel row rr of frame slot fa: box row fa * 2 + rr / 2 of the even
                            // (rr even) or odd box; an odd row starts 4 elements into its box row
                            // and lane 31's last 4 pixels sit in the tail box.
                            const int br = fa * 2 + rr / 2;
                            if (rr % 2 == 0) {
                                SRow<T>::load(region + br * 256 + 8 * lane, v[a][rr]);
                            } else {
                                const T *odd = region + 2048 + br * 256 + 4 + 8 * lane;
                                const uint2 lo = *reinterpret_cast<const uint2 *>(odd);
                                const uint2 hi =
                                    *reinterpret_cast<const uint2 *>(lane < 31 ? odd + 4 : region + 4096 + br * 8);
                                v[a][rr][0] = make_float2(bf16_lo(lo.x), bf16_lo(hi.x));
                                v[a][rr][1] = make_float2(bf16_hi(lo.x), bf16_hi(hi.x));
                                v[a][rr][2] = make_float2(bf16_lo(lo.y), bf16_lo(hi.y));
                                v[a][rr][3] = make_float2(bf16_hi(lo.y), bf16_hi(hi.y));
                            }
                        } else {
                            SRow<T>::load(region + (fa * 4 * RW + 4 * rw + rr) * 4 * WT + 8 * lane, v[a][rr]);
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
                __syncwarp(); // this row's pixels are read: the row may now hold results
                const float2 scale = make_float2(SCALE, SCALE);
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float2 p = VIDEO ? v[kt_of(g)][ky_of(g)][kx_of(g)] : v[0][ky2_of(g)][kx2_of(g)];
                    SRow<T>::store_pair(region + (rw * G + g) * kClPitch + 2 * lane, __fmul2_rn(p, scale));
                }
            }
        }
        __syncwarp(); // every channel is staged
        constexpr int PIECES = G * NC / VEC; // 16-byte pieces of one block's run
        const int64_t nblk = min((int64_t)WT, tg.w - (int64_t)tx * WT); // odd only in a row's last tile
#pragma unroll 1
        for (int rw = 0; rw < RW; ++rw) {
            const int64_t row = (int64_t)ty * RW + rw;
            if (row >= tg.h)
                continue;
            T *yrow = out + (((b * tg.Tq + tq) * tg.h + row) * tg.w + (int64_t)tx * WT) * (G * NC);
            const int total = (int)((nblk + 1) / 2) * PIECES; // (block pair, piece) items
#pragma unroll 2
            for (int it = lane; it < total; it += 32) {
                const int pr = it / PIECES, q = it - pr * PIECES; // block pair, piece
                auto staged = [&](int e) {
                    const int k = q * VEC + e, g = k / NC, c = k - g * NC;
                    return buf + (s * NC + c) * P::REGION_ELEMS + (rw * G + g) * kClPitch + 2 * pr;
                };
                uint4 r0, r1;
                if constexpr (sizeof(T) == 2) {
                    uint32_t wv[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        wv[e] = *reinterpret_cast<const uint32_t *>(staged(e));
                    // low halves: block 2*pr; high halves: block 2*pr + 1
                    r0 = make_uint4(__byte_perm(wv[0], wv[1], 0x5410), __byte_perm(wv[2], wv[3], 0x5410),
                                    __byte_perm(wv[4], wv[5], 0x5410), __byte_perm(wv[6], wv[7], 0x5410));
                    r1 = make_uint4(__byte_perm(wv[0], wv[1], 0x7632), __byte_perm(wv[2], wv[3], 0x7632),
                                    __byte_perm(wv[4], wv[5], 0x7632), __byte_perm(wv[6], wv[7], 0x7632));
                } else {
                    float2 pv[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        pv[e] = *reinterpret_cast<const float2 *>(staged(e));
                    r0 = make_uint4(__float_as_uint(pv[0].x), __float_as_uint(pv[1].x), __float_as_uint(pv[2].x),
                                    __float_as_uint(pv[3].x));
                    r1 = make_uint4(__float_as_uint(pv[0].y), __float_as_uint(pv[1].y), __float_as_uint(pv[2].y),
                                    __float_as_uint(pv[3].y));
                }
                T *dst = yrow + (int64_t)(2 * pr) * (G * NC) + q * VEC;
                *reinterpret_cast<uint4 *>(dst) = r0;
                if (2 * pr + 1 < nblk) // an odd last block has no partner
                    *reinterpret_cast<uint4 *>(dst + G * NC) = r1;
            }
        }
    }

    if (s < count && lane == 0) {
        for (int r = s; r < count; ++r)
            mbar_wait(smem_addr(bars + r), 0u);
        atomicAdd(&g_wait_timeouts, 1u);
    }
    __syncwarp();
}

// ---------------------------------------------------------------------------
// Single-level patcher / unpatcher (patch_size=2: one DWT; guide 7.1).  Same design
// as the two-level kernel with 2x2x2 blocks (2x2 on images): a warp tile is 64
// horizontally adjacent blocks across (128 pixels) and 8 block rows of one (b, c, t')
// window (16 on images), 4096 elements on either side; each lane owns blocks 2*lane
// and 2*lane + 1 as f32x2 pairs.  Window 0 of a video reads frame 0 twice (the
// replica) and its inverse keeps the second sample.  The three +-1 butterflies are
// followed by one fp32 multiply by 1/(2 sqrt 2) on video (the three 1/sqrt 2 taps),
// by the exact 1/2 on images.
// ---------------------------------------------------------------------------
template <bool VIDEO> struct SingleRows {
    static constexpr int RB = VIDEO ? 8 : 16; // block rows of a tile
};

// Shared memory of the single-level kernel; ROWS: the row form, as for the two-level kernel
// (32 staged pixel rows of 128 pixels on the forward, 64 coefficient rows of 64 on the inverse).
template <typename T, bool FWD, bool ROWS> struct SingleSmem {
    static constexpr int KT = !ROWS ? WarpTiles<T>::KT : sizeof(T) == 2 ? 2 : 1;
    static constexpr int NR = FWD ? 32 : 64;
    static constexpr int ROW = (FWD ? 128 : 64) * (int)sizeof(T) + 16;
    static constexpr int TILE = ROWS ? NR * ROW : kTileElems * (int)sizeof(T);
    static constexpr int SMEM = KT * TILE + 8 * KT + (ROWS ? 64 * KT : 0);
    static_assert(ROW % 16 == 0 && TILE % 16 == 0, "16-byte bulk-copy destinations");
};

// Four adjacent elements (the two pixels of blocks j and j + 1 in one pixel row) at byte
// offset o of a 16-byte-aligned staged row, without branches.
__device__ __forceinline__ void staged_quad(const unsigned char *row, uint32_t o, __nv_bfloat16 *, float *p)
{
    const uint32_t *w = reinterpret_cast<const uint32_t *>(row + (o & ~3u));
    const uint32_t sh = (o & 3u) * 8u;
    const uint32_t r0 = __funnelshift_r(w[0], w[1], sh), r1 = __funnelshift_r(w[1], w[2], sh);
    p[0] = bf16_lo(r0), p[1] = bf16_hi(r0), p[2] = bf16_lo(r1), p[3] = bf16_hi(r1);
}
__device__ __forceinline__ void staged_quad(const unsigned char *row, uint32_t o, float *, float *p)
{
    const float *w = reinterpret_cast<const float *>(row + o); // o is a multiple of 4
    p[0] = w[0], p[1] = w[1], p[2] = w[2], p[3] = w[3];
}

template <typename T, bool VIDEO, bool FWD, bool ROWS>
__global__ void __launch_bounds__(32)
    haar_single_kernel(const __grid_constant__ CUtensorMap xmap2, const __grid_constant__ CUtensorMap xmap1,
                       const __grid_constant__ CUtensorMap ymap, const T *__restrict__ src, T *__restrict__ out,
                       const TileGrid tg)
{
    using P = SingleSmem<T, FWD, ROWS>;
    constexpr int KT = P::KT, WT = kTileBlocks;
    constexpr int RB = SingleRows<VIDEO>::RB;
    constexpr int G = VIDEO ? 8 : 4;
    constexpr int NA = VIDEO ? 2 : 1;
    constexpr int FRAME = 2 * RB * 2 * WT; // elements of one frame slice of the tile
    static_assert(G * RB * WT == kTileElems && NA * FRAME == kTileElems, "tile sizes");
    constexpr uint32_t TILE_BYTES = kTileElems * sizeof(T), FRAME_BYTES = FRAME * sizeof(T);
    constexpr float SCALE = VIDEO ? 0.353553390593273762f : 0.5f;

    extern __shared__ __align__(1024) unsigned char smem_raw[];
    const int lane = threadIdx.x;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + KT * P::TILE);
    unsigned char *row_off = reinterpret_cast<unsigned char *>(bars + KT); // ROWS: [tile][staged row]

    auto decode = [&](uint32_t n, int &tx, int &ty, int &tq, int64_t &bc) {
        const uint32_t q1 = tg.ntx.div(n), q2 = tg.nty.div(q1), q3 = tg.nq.div(q2);
        tx = (int)(n - q1 * tg.ntx.d);
        ty = (int)(q1 - q2 * tg.nty.d);
        tq = (int)(q2 - q3 * tg.nq.d);
        bc = q3;
    };

    const uint32_t first = blockIdx.x * (uint32_t)KT;
    const int count = (int)min((uint32_t)KT, tg.ntiles - first);

    if constexpr (ROWS) {
        if (lane == 0) {
            for (int s = 0; s < KT; ++s)
                mbar_init(smem_addr(bars + s), 1);
            fence_barrier_init();
        }
        __syncwarp();
        constexpr int VE = 16 / (int)sizeof(T);
        constexpr int PER = P::NR / 32;
        const unsigned char *src_b = reinterpret_cast<const unsigned char *>(src);
        for (int s = 0; s < count; ++s) {
            int tx, ty, tq;
            int64_t bc;
            decode(first + s, tx, ty, tq, bc);
            int64_t start[PER];
            uint32_t nbulk[PER];
            bool ok[PER];
            uint32_t tx_bytes = 0;
#pragma unroll
            for (int k = 0; k < PER; ++k) {
                const int r = lane + 32 * k;
                int64_t off;
                if constexpr (FWD) {
                    // Staged row r: frame slot r / (2 RB), pixel row 2 RB ty + r % (2 RB).
                    const int a = r / (2 * RB);
                    const int64_t y = (int64_t)2 * RB * ty + r % (2 * RB);
                    const bool replica = VIDEO && tq == 0;
                    const int64_t f = !VIDEO || replica ? 0 : 2 * tq - 1 + a;
                    ok[k] = y < tg.H && !(replica && a != 0); // window 0 reads frame 0 only
                    off = ((bc * tg.T + f) * tg.H + y) * tg.W + (int64_t)2 * WT * tx;
                } else {
                    const int g = r / RB;
                    const int64_t row = (int64_t)RB * ty + r % RB;
                    const int64_t b = tg.C.div((uint32_t)bc), c = bc - b * tg.C.d;
                    const int64_t plane = (int64_t)tg.Tq * tg.h * tg.w;
                    ok[k] = row < tg.h;
                    off = ((b * G + g) * tg.C.d + c) * plane + ((int64_t)tq * tg.h + row) * tg.w + (int64_t)WT * tx;
                }
                const int mis = (int)(off % VE);
                start[k] = (off - mis) * (int64_t)sizeof(T);
                const int64_t avail = tg.n_src * (int64_t)sizeof(T) - start[k];
                nbulk[k] = !ok[k] ? 0u : avail >= P::ROW ? (uint32_t)P::ROW : (uint32_t)(avail & ~(int64_t)15);
                // A row that is not loaded is never used for a stored result: offset 0 keeps the
                // realigned reads inside its staging row.
                row_off[s * 64 + r] = ok[k] ? (unsigned char)(mis * (int)sizeof(T)) : (unsigned char)0;
                tx_bytes += __reduce_add_sync(0xFFFFFFFFu, nbulk[k]);
            }
            const uint32_t bar = smem_addr(bars + s);
            if (lane == 0)
                mbar_expect_tx(bar, tx_bytes);
            __syncwarp();
            unsigned char *tile = smem_raw + s * P::TILE;
#pragma unroll
            for (int k = 0; k < PER; ++k) {
                if (!ok[k])
                    continue;
                unsigned char *dst = tile + (lane + 32 * k) * P::ROW;
                if (nbulk[k] > 0)
                    bulk_load(smem_addr(dst), src_b + start[k], nbulk[k], bar);
                if (nbulk[k] < (uint32_t)P::ROW) { // the tensor's last, partial 16 bytes
                    const int64_t end = min(tg.n_src * (int64_t)sizeof(T) - start[k], (int64_t)P::ROW);
                    for (int64_t b = nbulk[k]; b < end; b += (int64_t)sizeof(T))
                        *reinterpret_cast<T *>(dst + b) = *reinterpret_cast<const T *>(src_b + start[k] + b);
                }
            }
        }
    } else if (lane == 0) {
        for (int s = 0; s < KT; ++s)
            mbar_init(smem_addr(bars + s), 1);
        fence_barrier_init();
        for (int s = 0; s < count; ++s) {
            int tx, ty, tq;
            int64_t bc;
            decode(first + s, tx, ty, tq, bc);
            const uint32_t dst = smem_addr(smem_raw + s * P::TILE), bar = smem_addr(bars + s);
            if constexpr (FWD) {
                if (VIDEO && tq > 0) {
                    mbar_expect_tx(bar, NA * FRAME_BYTES);
                    tma_load_3d(dst, &xmap2, 2 * WT * tx, 2 * RB * ty, (int)(bc * tg.T + 2 * tq - 1), bar);
                } else {
                    mbar_expect_tx(bar, FRAME_BYTES);
                    tma_load_3d(dst, &xmap1, 2 * WT * tx, 2 * RB * ty, (int)(bc * tg.T), bar);
                }
            } else {
                const int b = (int)tg.C.div((uint32_t)bc), c = (int)(bc - (int64_t)b * tg.C.d);
                mbar_expect_tx(bar, TILE_BYTES);
                tma_load_5d(dst, &ymap, WT * tx, RB * ty, tq, c, G * b, bar);
            }
        }
    }
    __syncwarp();

    int s = 0;
    for (; s < count; ++s) {
        const bool ok = mbar_wait(smem_addr(bars + s), 0u);
        if (__any_sync(0xFFFFFFFFu, !ok))
            break;
        int tx, ty, tq;
        int64_t bc;
        decode(first + s, tx, ty, tq, bc);
        const unsigned char *tile = smem_raw + s * P::TILE;
        const T *tin = reinterpret_cast<const T *>(tile);
        const int64_t j0 = (int64_t)tx * WT + 2 * lane; // this lane's first block column
        const bool col_ok = j0 < tg.w;
        const bool pair_ok = !ROWS || j0 + 1 < tg.w;    // block j0 + 1 exists (w is even outside the row form)
        const bool replica = VIDEO && tq == 0;

#pragma unroll 2
        for (int rb = 0; rb < RB; ++rb) {
            float2 v[NA][2][2]; // FWD: [t][y][x] pixels -> [bt][by][bx]; INV: the reverse
            if constexpr (FWD) {
#pragma unroll
                for (int a = 0; a < NA; ++a) {
                    const int fa = replica ? 0 : a;
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        float q[4]; // pixels 0, 1 of block j0, then of block j0 + 1
                        if constexpr (ROWS) {
                            const int sr = fa * 2 * RB + 2 * rb + r;
                            staged_quad(tile + sr * P::ROW, row_off[s * 64 + sr] + lane * 4 * (uint32_t)sizeof(T),
                                        (T *)nullptr, q);
                        } else {
                            const T *px = tin + (fa * 2 * RB + 2 * rb + r) * 2 * WT + 4 * lane;
                            const float2 p01 = SRow<T>::load_pair(px), p23 = SRow<T>::load_pair(px + 2);
                            q[0] = p01.x, q[1] = p01.y, q[2] = p23.x, q[3] = p23.y;
                        }
                        v[a][r][0] = make_float2(q[0], q[2]); // pixel 0 of blocks j0, j0 + 1
                        v[a][r][1] = make_float2(q[1], q[3]); // pixel 1
                    }
                }
            } else {
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float2 p;
                    if constexpr (ROWS)
                        p = staged_pair(tile + (g * RB + rb) * P::ROW,
                                        row_off[s * 64 + g * RB + rb] + lane * 2 * (uint32_t)sizeof(T), (T *)nullptr);
                    else
                        p = SRow<T>::load_pair(tin + (g * RB + rb) * WT + 2 * lane);
                    if constexpr (VIDEO)
                        v[g >> 2][(g >> 1) & 1][g & 1] = p;
                    else
                        v[0][g >> 1][g & 1] = p;
                }
            }
            // one butterfly per axis: (a + b, a - b)
#pragma unroll
            for (int a = 0; a < NA; ++a)
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    const float2 l = add2(v[a][r][0], v[a][r][1]), hgh = sub2(v[a][r][0], v[a][r][1]);
                    v[a][r][0] = l, v[a][r][1] = hgh;
                }
#pragma unroll
            for (int a = 0; a < NA; ++a)
#pragma unroll
                for (int d = 0; d < 2; ++d) {
                    const float2 l = add2(v[a][0][d], v[a][1][d]), hgh = sub2(v[a][0][d], v[a][1][d]);
                    v[a][0][d] = l, v[a][1][d] = hgh;
                }
            if constexpr (VIDEO) {
#pragma unroll
                for (int r = 0; r < 2; ++r)
#pragma unroll
                    for (int d = 0; d < 2; ++d) {
                        const float2 l = add2(v[0][r][d], v[1][r][d]), hgh = sub2(v[0][r][d], v[1][r][d]);
                        v[0][r][d] = l, v[1][r][d] = hgh;
                    }
            }
            const float2 scale = make_float2(SCALE, SCALE);
            const int64_t row = (int64_t)ty * RB + rb; // block row
            bool pairs = true;
            if constexpr (FWD && ROWS) {
                // Pair stores when every storing lane's G pairs are aligned and whole (the alignment
                // alternates with g only when the plane stride is odd), element stores otherwise;
                // one warp-wide vote, taken before any lane leaves.
                const int64_t b = tg.C.div((uint32_t)bc), c = bc - b * tg.C.d;
                const int64_t plane = (int64_t)tg.Tq * tg.h * tg.w;
                const T *yq = out + (b * G * tg.C.d + c) * plane + ((int64_t)tq * tg.h + row) * tg.w + j0;
                const uintptr_t amask = 2 * sizeof(T) - 1;
                pairs = __all_sync(0xFFFFFFFFu, !col_ok || (pair_ok && ((uintptr_t)yq & amask) == 0 &&
                                                            ((uintptr_t)(yq + tg.C.d * plane) & amask) == 0));
            }
            if (!col_ok || row >= tg.h)
                continue;
            if constexpr (FWD) {
                const int64_t b = tg.C.div((uint32_t)bc), c = bc - b * tg.C.d;
                const int64_t plane = (int64_t)tg.Tq * tg.h * tg.w;
                T *yp = out + (b * G * tg.C.d + c) * plane + ((int64_t)tq * tg.h + row) * tg.w + j0;
                if (!ROWS || pairs) {
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float2 p = VIDEO ? v[g >> 2][(g >> 1) & 1][g & 1] : v[0][g >> 1][g & 1];
                        gstore_pair(yp + (int64_t)g * tg.C.d * plane, __fmul2_rn(p, scale));
                    }
                } else {
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float2 q =
                            __fmul2_rn(VIDEO ? v[g >> 2][(g >> 1) & 1][g & 1] : v[0][g >> 1][g & 1], scale);
                        T *dst = yp + (int64_t)g * tg.C.d * plane;
                        dst[0] = to_elem<T>(q.x);
                        if (pair_ok)
                            dst[1] = to_elem<T>(q.y);
                    }
                }
            } else {
                T *xb = out + (bc * tg.T) * tg.H * tg.W + (2 * row) * tg.W + 2 * j0;
#pragma unroll
                for (int a = 0; a < NA; ++a) {
                    if (replica && a != 1) // window 0 keeps its second sample (frame 0)
                        continue;
                    const int64_t f = !VIDEO ? 0 : replica ? 0 : 2 * tq - 1 + a;
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const float2 q0 = __fmul2_rn(v[a][r][0], scale), q1 = __fmul2_rn(v[a][r][1], scale);
                        T *dst = xb + f * tg.H * tg.W + r * tg.W;
                        SRow<T>::store_pair(dst, make_float2(q0.x, q1.x));     // block j0: pixels 0, 1
                        if (pair_ok)
                            SRow<T>::store_pair(dst + 2, make_float2(q0.y, q1.y)); // block j0 + 1
                    }
                }
            }
        }
    }

    if (s < count && lane == 0) {
        for (int r = s; r < count; ++r)
            mbar_wait(smem_addr(bars + r), 0u);
        atomicAdd(&g_wait_timeouts, 1u);
    }
    __syncwarp();
}

// ---------------------------------------------------------------------------
// Host side.
// ---------------------------------------------------------------------------
template <typename T, bool VIDEO, bool FWD, bool ADJ, bool EXT, bool ROWS, bool ANYST = false, int GR = 0>
tok_status launch(const void *in, void *out, const HaarDims &d, cudaStream_t stream)
{
    using P = TileSmem<T, FWD, ROWS, GR>;
    constexpr int G = VIDEO ? 64 : 16, RW = TileRows<VIDEO>::RW, WT = kTileBlocks;
    const CUtensorMapDataType dt = sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const uint64_t es = sizeof(T);
    // Only the input side goes through TMA: pixels on the forward, coefficients on the inverse.
    CUtensorMap xm4, xm1, ym, xt4, xt1;
    memset(&xm4, 0, sizeof xm4);
    memset(&xm1, 0, sizeof xm1);
    memset(&ym, 0, sizeof ym);
    memset(&xt4, 0, sizeof xt4);
    memset(&xt1, 0, sizeof xt1);
    if (ROWS) {
        // The row form reads the source through its pointer (bulk copies); no tensor map.
    } else if (FWD) {
        // Grouped rows: each frame as [H / GR][GR W], GR pixel rows per row of the map (a
        // 16-byte multiple), and a box of the tile's rows of one part.
        const uint64_t g = GR ? (uint64_t)GR : 1u;
        const uint64_t xdims[3] = {g * d.W, d.H / g, (uint64_t)(d.B * d.C * d.T)};
        const uint64_t xstr[2] = {g * d.W * es, d.H * d.W * es};
        const uint32_t rows = 4u * RW / (uint32_t)g;
        const uint32_t box4[3] = {4u * WT, rows, 4u}, box1[3] = {4u * WT, rows, 1u};
        // The 4-frame box serves windows with four frames of the clip, so a frame axis
        // shorter than 4 never uses it and it is not encoded.
        if (!encode_tensor_map(&xm1, dt, 3, in, xdims, xstr, box1) ||
            (VIDEO && xdims[2] >= 4 && !encode_tensor_map(&xm4, dt, 3, in, xdims, xstr, box4)))
            return TOK_ERR_SHAPE;
        if (GR) { // the 8 elements after a part's box
            const uint32_t tail4[3] = {8u, rows, 4u}, tail1[3] = {8u, rows, 1u};
            if (!encode_tensor_map(&xt1, dt, 3, in, xdims, xstr, tail1) ||
                (VIDEO && xdims[2] >= 4 && !encode_tensor_map(&xt4, dt, 3, in, xdims, xstr, tail4)))
                return TOK_ERR_SHAPE;
        }
    } else {
        const uint64_t ydims[5] = {(uint64_t)d.w, (uint64_t)d.h, (uint64_t)d.Tq, (uint64_t)d.C, (uint64_t)(G * d.B)};
        const uint64_t plane = d.Tq * d.h * d.w * es;
        const uint64_t ystr[4] = {d.w * es, d.h * d.w * es, plane, d.C * plane};
        const uint32_t ybox[5] = {(uint32_t)WT, (uint32_t)RW, 1u, 1u, (uint32_t)G};
        if (!encode_tensor_map(&ym, dt, 5, in, ydims, ystr, ybox))
            return TOK_ERR_SHAPE;
    }

    // Sector-aligned plane stores (TileGrid::salign): the shifts k w mod salign are multiples of
    // gcd(w, salign), so a row needs at most ceil((w + salign - gcd) / 64) tiles.
    int salign = 0;
    if (FWD && VIDEO && !ROWS && !GR) {
        const int64_t sa = 32 / (int64_t)es, plane = d.Tq * d.h * d.w;
        if ((d.w * (int64_t)es) % 32 != 0 && (plane * (int64_t)es) % 32 == 0 && aligned(out, 32))
            salign = (int)sa;
    } else if (FWD && VIDEO && GR) {
        // Grouped rows (w may be odd): the largest power of two up to kGroupSalign that divides
        // a plane, so the shifted tiles' pair stores are aligned (sector-aligned at 16).
        const int64_t plane = d.Tq * d.h * d.w;
        for (int64_t sa = kGroupSalign; sa >= 2 && !salign; sa /= 2)
            if (plane % sa == 0 && aligned(out, (size_t)(sa * (int64_t)es)))
                salign = (int)sa;
    }
    const int64_t smax = salign ? salign - std::gcd(d.w, (int64_t)salign) : 0;
    const int64_t ntx = (d.w + smax + WT - 1) / WT, nty = (d.h + RW - 1) / RW;
    TileGrid tg;
    tg.ntx = FastDiv((uint32_t)ntx);
    tg.nty = FastDiv((uint32_t)nty);
    tg.nq = FastDiv((uint32_t)d.nq);
    tg.C = FastDiv((uint32_t)d.C);
    tg.T = (int)d.T;
    tg.Tq = (int)d.Tq;
    tg.tq0 = (int)d.tq0;
    tg.H = d.H;
    tg.W = d.W;
    tg.h = d.h;
    tg.w = d.w;
    tg.ntiles = (uint32_t)(ntx * nty * d.nq * d.B * d.C); // < 2^32: checked by tma_limits_ok
    tg.fbase = (int)d.fbase;
    tg.rep = d.rep;
    tg.n_src = FWD ? d.B * d.C * d.T * d.H * d.W : d.B * G * d.C * d.Tq * d.h * d.w;
    tg.salign = salign;
    tg.planes_share_offset = ((int64_t)d.C * d.Tq * d.h * d.w * (int64_t)es) % 16 == 0;
    {
        const uint64_t bits = (uint64_t)(d.W * (int64_t)es) | (uint64_t)(uintptr_t)out | 16u;
        tg.sw = (int)(bits & (~bits + 1)); // the lowest set bit: 2, 4, 8 or 16
    }

    // Per call: the attribute belongs to the current device.
    const cudaError_t attr_err = cudaFuncSetAttribute(haar_tma_kernel<T, VIDEO, FWD, ADJ, EXT, ROWS, ANYST, GR>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM);
    if (attr_err != cudaSuccess) {
        record_cuda_error(attr_err);
        return TOK_ERR_CUDA;
    }
    const unsigned grid = (unsigned)((tg.ntiles + P::KT - 1) / P::KT);
    haar_tma_kernel<T, VIDEO, FWD, ADJ, EXT, ROWS, ANYST, GR>
        <<<grid, 32, P::SMEM, stream>>>(xm4, xm1, ym, xt4, xt1, (const T *)in, (T *)out, tg);
    return launch_status();
}

template <typename T, bool VIDEO, bool FWD, bool ADJ, bool EXT>
tok_status launch_form(HaarTmaForm form, const void *in, void *out, const HaarDims &d, cudaStream_t stream)
{
    if (form == HaarTmaForm::rows)
        return launch<T, VIDEO, FWD, ADJ, EXT, true>(in, out, d, stream);
    if constexpr (!FWD) {
        if (form == HaarTmaForm::boxes_any_store)
            return launch<T, VIDEO, FWD, ADJ, EXT, false, true>(in, out, d, stream);
    }
    if constexpr (VIDEO && FWD && sizeof(T) == 2) {
        if (form == HaarTmaForm::groups)
            return launch<T, VIDEO, FWD, ADJ, EXT, false, false, 2>(in, out, d, stream);
    }
    return launch<T, VIDEO, FWD, ADJ, EXT, false>(in, out, d, stream);
}

// Limits shared by both forms: 32-bit frame, group and tile numbers, and the 64 planes of
// one channel within a 32-bit element offset.
bool tma_limits_ok(const HaarDims &d)
{
    const int64_t ntiles = ((d.w + 16 + 63) / 64) * ((d.h + 3) / 4 + d.h) * d.Tq * d.B * d.C; // generous bound
    return d.B * d.C * d.T < (int64_t)1 << 31 && 64 * d.B < (int64_t)1 << 31 && d.W < (int64_t)1 << 31 &&
           d.H < (int64_t)1 << 31 && ntiles < (int64_t)1 << 32 && 64 * d.C * d.Tq * d.h * d.w < (int64_t)1 << 32;
}

} // namespace

HaarTmaForm haar_tma_form(bool fwd, const void *in, const void *out, tok_dtype dt, const HaarDims &d)
{
    const int64_t es = dt == TOK_F32 ? 4 : 2;
    if (!tma_limits_ok(d) || sm_count() <= 0)
        return HaarTmaForm::none;
    // Box form: the source's rows are whole 16-byte units (one TMA box per tile); the forward
    // stores coefficient pairs (w even), the inverse 16-byte pixel rows.
    const bool boxes = fwd ? aligned(in, 16) && (d.W * es) % 16 == 0 && aligned(out, 2 * es) && d.w % 2 == 0
                           : aligned(in, 16) && (d.w * es) % 16 == 0 && aligned(out, 16) && (d.W * es) % 16 == 0;
    if (boxes)
        return HaarTmaForm::boxes;
    // Inverse whose source takes the box form but whose pixel rows do not (cropped or chunked
    // odd widths, a destination off a 16-byte boundary): box loads, stores of run-time width.
    if (!fwd && aligned(in, 16) && (d.w * es) % 16 == 0)
        return HaarTmaForm::boxes_any_store;
    // bf16 video forward whose pixel rows are 8-byte units (two of them are 16-byte units), with
    // an odd number of coefficient columns: grouped rows (whole pairs of rows of the clip,
    // coordinates below 2^31).
    if (fwd && es == 2 && d.video && aligned(in, 16) && d.W % 8 == 4 && d.w % 2 == 1 && d.H % 2 == 0 &&
        2 * d.W + 1024 < ((int64_t)1 << 31))
        return HaarTmaForm::groups;
    // Row form: any 16-byte-aligned source.
    return aligned(in, 16) ? HaarTmaForm::rows : HaarTmaForm::none;
}

tok_status haar_tma_launch(bool fwd, bool adj, HaarTmaForm form, const void *in, void *out, tok_dtype dt,
                           const HaarDims &d, cudaStream_t stream)
{
    const bool video = d.video;
    if (d.ext) {
        if (dt == TOK_BF16) {
            using B16 = __nv_bfloat16;
            if (video)
                return fwd ? launch_form<B16, true, true, false, true>(form, in, out, d, stream)
                           : launch_form<B16, true, false, false, true>(form, in, out, d, stream);
            return fwd ? launch_form<B16, false, true, false, true>(form, in, out, d, stream)
                       : launch_form<B16, false, false, false, true>(form, in, out, d, stream);
        }
        if (video)
            return fwd ? launch_form<float, true, true, false, true>(form, in, out, d, stream)
                       : launch_form<float, true, false, false, true>(form, in, out, d, stream);
        return fwd ? launch_form<float, false, true, false, true>(form, in, out, d, stream)
                   : launch_form<float, false, false, false, true>(form, in, out, d, stream);
    }
    if (dt == TOK_BF16) {
        using B16 = __nv_bfloat16;
        if (!video)
            return fwd ? launch_form<B16, false, true, false, false>(form, in, out, d, stream)
                       : launch_form<B16, false, false, false, false>(form, in, out, d, stream);
        if (adj)
            return fwd ? launch_form<B16, true, true, true, false>(form, in, out, d, stream)
                       : launch_form<B16, true, false, true, false>(form, in, out, d, stream);
        return fwd ? launch_form<B16, true, true, false, false>(form, in, out, d, stream)
                   : launch_form<B16, true, false, false, false>(form, in, out, d, stream);
    }
    if (!video)
        return fwd ? launch_form<float, false, true, false, false>(form, in, out, d, stream)
                   : launch_form<float, false, false, false, false>(form, in, out, d, stream);
    if (adj)
        return fwd ? launch_form<float, true, true, true, false>(form, in, out, d, stream)
                   : launch_form<float, true, false, true, false>(form, in, out, d, stream);
    return fwd ? launch_form<float, true, true, false, false>(form, in, out, d, stream)
               : launch_form<float, true, false, false, false>(form, in, out, d, stream);
}

// Self-test of the failure channel: one single-warp CTA whose barrier phase cannot
// complete, because lane 0 declares 16 bytes of transaction that no copy ever
// delivers.  Its wait gives up after `polls` polls, as a TMA kernel's wait does after
// kWaitPolls, and counts a timeout.  No copy was issued, so nothing can land in this
// CTA's shared memory after the kernel exits.
__global__ void __launch_bounds__(32) wait_timeout_selftest_kernel(uint32_t polls)
{
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_addr(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_barrier_init();
    }
    __syncwarp();
    if (threadIdx.x == 0) {
        mbar_expect_tx(b, 16);
        bool done = false;
        for (uint32_t i = 0; i < polls && !done; ++i)
            done = mbar_try_wait(b, 0u);
        if (!done)
            atomicAdd(&g_wait_timeouts, 1u);
    }
    __syncwarp();
}

tok_status read_and_clear_haar_timeouts(cudaStream_t stream, unsigned int *count)
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

namespace tok {
namespace {

template <typename T, bool VIDEO, bool FWD, bool ROWS>
tok_status launch_single(const void *in, void *out, const HaarDims &d, cudaStream_t stream)
{
    using P = SingleSmem<T, FWD, ROWS>;
    constexpr int G = VIDEO ? 8 : 4, RB = SingleRows<VIDEO>::RB, WT = kTileBlocks;
    const CUtensorMapDataType dt = sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const uint64_t es = sizeof(T);
    CUtensorMap xm2, xm1, ym;
    memset(&xm2, 0, sizeof xm2);
    memset(&xm1, 0, sizeof xm1);
    memset(&ym, 0, sizeof ym);
    if (ROWS) {
        // The row form reads the source through its pointer (bulk copies); no tensor map.
    } else if (FWD) {
        const uint64_t xdims[3] = {(uint64_t)d.W, (uint64_t)d.H, (uint64_t)(d.B * d.C * d.T)};
        const uint64_t xstr[2] = {d.W * es, d.H * d.W * es};
        const uint32_t box2[3] = {2u * WT, 2u * RB, 2u}, box1[3] = {2u * WT, 2u * RB, 1u};
        if (!encode_tensor_map(&xm1, dt, 3, in, xdims, xstr, box1) ||
            (VIDEO && !encode_tensor_map(&xm2, dt, 3, in, xdims, xstr, box2)))
            return TOK_ERR_SHAPE;
    } else {
        const uint64_t ydims[5] = {(uint64_t)d.w, (uint64_t)d.h, (uint64_t)d.Tq, (uint64_t)d.C, (uint64_t)(G * d.B)};
        const uint64_t plane = d.Tq * d.h * d.w * es;
        const uint64_t ystr[4] = {d.w * es, d.h * d.w * es, plane, d.C * plane};
        const uint32_t ybox[5] = {(uint32_t)WT, (uint32_t)RB, 1u, 1u, (uint32_t)G};
        if (!encode_tensor_map(&ym, dt, 5, in, ydims, ystr, ybox))
            return TOK_ERR_SHAPE;
    }
    const int64_t ntx = (d.w + WT - 1) / WT, nty = (d.h + RB - 1) / RB;
    TileGrid tg{};
    tg.ntx = FastDiv((uint32_t)ntx);
    tg.nty = FastDiv((uint32_t)nty);
    tg.nq = FastDiv((uint32_t)d.Tq);
    tg.C = FastDiv((uint32_t)d.C);
    tg.T = (int)d.T;
    tg.Tq = (int)d.Tq;
    tg.tq0 = 0;
    tg.H = d.H;
    tg.W = d.W;
    tg.h = d.h;
    tg.w = d.w;
    tg.ntiles = (uint32_t)(ntx * nty * d.Tq * d.B * d.C);
    tg.n_src = FWD ? d.B * d.C * d.T * d.H * d.W : d.B * G * d.C * d.Tq * d.h * d.w;
    const cudaError_t attr_err = cudaFuncSetAttribute(haar_single_kernel<T, VIDEO, FWD, ROWS>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM);
    if (attr_err != cudaSuccess) {
        record_cuda_error(attr_err);
        return TOK_ERR_CUDA;
    }
    const unsigned grid = (unsigned)((tg.ntiles + P::KT - 1) / P::KT);
    haar_single_kernel<T, VIDEO, FWD, ROWS>
        <<<grid, 32, P::SMEM, stream>>>(xm2, xm1, ym, (const T *)in, (T *)out, tg);
    return launch_status();
}

template <typename T, bool VIDEO, bool FWD>
tok_status launch_single_form(bool rows, const void *in, void *out, const HaarDims &d, cudaStream_t stream)
{
    return rows ? launch_single<T, VIDEO, FWD, true>(in, out, d, stream)
                : launch_single<T, VIDEO, FWD, false>(in, out, d, stream);
}

} // namespace

HaarTmaForm haar_single_tma_form(bool fwd, const void *in, const void *out, tok_dtype dt, const HaarDims &d)
{
    const int64_t es = dt == TOK_F32 ? 4 : 2;
    const int64_t ntiles = ((d.w + 63) / 64) * (d.h / 8 + 1) * d.Tq * d.B * d.C;
    if (d.B * d.C * d.T >= (int64_t)1 << 31 || 8 * d.B >= (int64_t)1 << 31 || d.W >= (int64_t)1 << 31 ||
        d.H >= (int64_t)1 << 31 || ntiles >= (int64_t)1 << 32 || sm_count() <= 0 || !aligned(in, 16))
        return HaarTmaForm::none;
    // Box form: only the source goes through TMA (pixels on the forward, coefficients on the
    // inverse), so its rows must be whole 16-byte units; both directions store element pairs
    // (the forward's at even block columns, w even; the inverse's at even pixel columns, W even).
    if (aligned(out, 2 * es) && ((fwd ? d.W : d.w) * es) % 16 == 0 && d.w % 2 == 0)
        return HaarTmaForm::boxes;
    // Row form: any row length; the forward votes between pair and element stores, the inverse
    // stores pixel pairs (W is even).
    return aligned(out, fwd ? es : 2 * es) ? HaarTmaForm::rows : HaarTmaForm::none;
}

tok_status haar_single_tma_launch(bool fwd, HaarTmaForm form, const void *in, void *out, tok_dtype dt,
                                  const HaarDims &d, cudaStream_t stream)
{
    const bool rows = form == HaarTmaForm::rows;
    if (dt == TOK_BF16) {
        using B16 = __nv_bfloat16;
        if (d.video)
            return fwd ? launch_single_form<B16, true, true>(rows, in, out, d, stream)
                       : launch_single_form<B16, true, false>(rows, in, out, d, stream);
        return fwd ? launch_single_form<B16, false, true>(rows, in, out, d, stream)
                   : launch_single_form<B16, false, false>(rows, in, out, d, stream);
    }
    if (d.video)
        return fwd ? launch_single_form<float, true, true>(rows, in, out, d, stream)
                   : launch_single_form<float, true, false>(rows, in, out, d, stream);
    return fwd ? launch_single_form<float, false, true>(rows, in, out, d, stream)
               : launch_single_form<float, false, false>(rows, in, out, d, stream);
}

} // namespace tok

namespace tok {
namespace {

template <typename T, bool VIDEO, int NC, bool ROWS, bool PAIRS>
tok_status launch_cl(const void *in, void *out, const HaarDims &d, cudaStream_t stream)
{
    using P = ClTiles<T, NC, ROWS>;
    constexpr int RW = TileRows<VIDEO>::RW, WT = kTileBlocks;
    const CUtensorMapDataType dt = sizeof(T) == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const uint64_t es = sizeof(T);
    CUtensorMap xm4, xm1, xt4, xt1;
    memset(&xm4, 0, sizeof xm4);
    memset(&xm1, 0, sizeof xm1);
    memset(&xt4, 0, sizeof xt4);
    memset(&xt1, 0, sizeof xt1);
    if (PAIRS) { // each frame as [H/2][2W]: rows of two pixel rows, 4W-byte strides
        const uint64_t xdims[3] = {(uint64_t)(2 * d.W), (uint64_t)(d.H / 2), (uint64_t)(d.B * d.C * d.T)};
        const uint64_t xstr[2] = {2 * d.W * es, d.H * d.W * es};
        const uint32_t box4[3] = {4u * WT, 2u, 4u}, box1[3] = {4u * WT, 2u, 1u}, tail4[3] = {8u, 2u, 4u},
                       tail1[3] = {8u, 2u, 1u};
        if (!encode_tensor_map(&xm4, dt, 3, in, xdims, xstr, box4) ||
            !encode_tensor_map(&xm1, dt, 3, in, xdims, xstr, box1) ||
            !encode_tensor_map(&xt4, dt, 3, in, xdims, xstr, tail4) ||
            !encode_tensor_map(&xt1, dt, 3, in, xdims, xstr, tail1))
            return TOK_ERR_SHAPE;
    } else if (!ROWS) { // the row form reads the pixels through their pointer (bulk copies)
        const uint64_t xdims[3] = {(uint64_t)d.W, (uint64_t)d.H, (uint64_t)(d.B * d.C * d.T)};
        const uint64_t xstr[2] = {d.W * es, d.H * d.W * es};
        const uint32_t box4[3] = {4u * WT, 4u * RW, 4u}, box1[3] = {4u * WT, 4u * RW, 1u};
        if (!encode_tensor_map(&xm1, dt, 3, in, xdims, xstr, box1) ||
            (VIDEO && !encode_tensor_map(&xm4, dt, 3, in, xdims, xstr, box4)))
            return TOK_ERR_SHAPE;
    }
    const int64_t ntx = (d.w + WT - 1) / WT, nty = (d.h + RW - 1) / RW;
    TileGrid tg{};
    tg.ntx = FastDiv((uint32_t)ntx);
    tg.nty = FastDiv((uint32_t)nty);
    tg.nq = FastDiv((uint32_t)d.Tq);
    tg.C = FastDiv((uint32_t)d.C);
    tg.T = (int)d.T;
    tg.Tq = (int)d.Tq;
    tg.H = d.H;
    tg.W = d.W;
    tg.h = d.h;
    tg.w = d.w;
    tg.ntiles = (uint32_t)(ntx * nty * d.Tq * d.B);
    tg.n_src = d.B * d.C * d.T * d.H * d.W;
    const cudaError_t attr_err = cudaFuncSetAttribute(haar_cl_kernel<T, VIDEO, NC, ROWS, PAIRS>,
                                                      cudaFuncAttributeMaxDynamicSharedMemorySize, P::SMEM);
    if (attr_err != cudaSuccess) {
        record_cuda_error(attr_err);
        return TOK_ERR_CUDA;
    }
    const unsigned grid = (unsigned)((tg.ntiles + P::KT - 1) / P::KT);
    haar_cl_kernel<T, VIDEO, NC, ROWS, PAIRS>
        <<<grid, 32, P::SMEM, stream>>>(xm4, xm1, xt4, xt1, (const T *)in, (T *)out, tg);
    return launch_status();
}

// Form per call: tensor boxes (pixel rows of whole 16-byte units), pair-row boxes (bf16 video,
// W % 8 == 4; their x coordinates, up to 2W + 508, must fit 32 bits), or row copies (bf16 images
// with W % 8 == 4, and wider video).
template <typename T, bool VIDEO, int NC>
tok_status launch_cl_form(bool rows, const void *in, void *out, const HaarDims &d, cudaStream_t stream)
{
    if (!rows)
        return launch_cl<T, VIDEO, NC, false, false>(in, out, d, stream);
    if constexpr (VIDEO && sizeof(T) == 2) {
        if (2 * d.W + 512 < ((int64_t)1 << 31))
            return launch_cl<T, VIDEO, NC, false, true>(in, out, d, stream);
    }
    return launch_cl<T, VIDEO, NC, true, false>(in, out, d, stream);
}

template <typename T, bool VIDEO>
tok_status launch_cl_c(bool rows, const void *in, void *out, const HaarDims &d, cudaStream_t stream)
{
    switch (d.C) {
    case 1:
        return launch_cl_form<T, VIDEO, 1>(rows, in, out, d, stream);
    case 2:
        return launch_cl_form<T, VIDEO, 2>(rows, in, out, d, stream);
    case 3:
        return launch_cl_form<T, VIDEO, 3>(rows, in, out, d, stream);
    default:
        return launch_cl_form<T, VIDEO, 4>(rows, in, out, d, stream);
    }
}

} // namespace

bool haar_cl_tma_eligible(const void *in, const void *out, tok_dtype dt, const HaarDims &d)
{
    // Any w: the pixel side takes the box form where its rows are whole 16-byte units and the row
    // form otherwise (bf16 with odd w); a block's G*C outputs are whole 16-byte pieces at any w.
    return d.C >= 1 && d.C <= 4 && aligned(in, 16) && aligned(out, 16) && tma_limits_ok(d) && sm_count() > 0;
}

tok_status haar_cl_tma_launch(const void *in, void *out, tok_dtype dt, const HaarDims &d, cudaStream_t stream)
{
    const bool rows = (d.W * (dt == TOK_F32 ? 4 : 2)) % 16 != 0;
    if (dt == TOK_BF16)
        return d.video ? launch_cl_c<__nv_bfloat16, true>(rows, in, out, d, stream)
                       : launch_cl_c<__nv_bfloat16, false>(rows, in, out, d, stream);
    return d.video ? launch_cl_c<float, true>(rows, in, out, d, stream)
                   : launch_cl_c<float, false>(rows, in, out, d, stream);
}

} // namespace tok

extern "C" tok_status tok_selftest_wait_timeout(uint32_t polls, cudaStream_t stream)
{
    if (polls < 1 || polls > tok::kWaitPolls)
        return TOK_ERR_SHAPE;
    tok::wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(polls);
    return tok::launch_status();
}
