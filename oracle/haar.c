/*
 * Haar patcher / unpatcher oracle.  TEST INFRASTRUCTURE ONLY: the test suite,
 * the smoke check and the benchmark's CPU-baseline leg load this file's
 * library; the product path never does.  It shares no code, header or table
 * with the CUDA library.
 *
 * Plain, slow, double-precision CPU statement of the two-level, causal,
 * full-packet, orthonormal 3D Haar wavelet patcher and of its inverse.
 *
 * What the pages fix (page title, section):
 *   - "NVIDIA Cosmos Tokenizer 完全指南", section 7.1 (Haar wavelet patching):
 *     the Haar filter taps are printed as [0.7071, 0.7071], i.e. 1/sqrt(2)
 *     (rounded in print; this file uses the exact value); one 2D DWT turns c
 *     channels into 4c and halves H and W; the docstring example
 *     [3,256,256] -> [12,128,128] -> [48,64,64] shows that the second level
 *     transforms all twelve first-level channels (full packet); the 3D patcher
 *     turns c into 8c, halves T, H and W, and repeats the first frame so the
 *     time axis stays causally aligned; patch_size=4 stacks two DWTs; the
 *     unpatchers invert the transform.
 *   - same page, sections 6.1 and 7.3: T frames give t = 1 + (T-1)/4 latent
 *     frames, the first one aligned with frame 0 alone.
 *   - "nvidia/Cosmos-Tokenize1-CV8x8x8-720p" model card, "Model Architecture":
 *     the encoder starts with a 2-level Haar transform that downsamples by 4
 *     in space and in time; the decoder ends with the inverse transform.
 *
 * Readings where the pages are silent (each one is a convention shared with
 * the CUDA path; parity unpinned by the pages for the first two -- any fixed
 * sign or subband permutation would be equally valid):
 *   - high band of a pair (a, b) is (a - b)/sqrt(2), low band (a + b)/sqrt(2);
 *   - subband s = 4*bt + 2*by + bx (bit = 1 for the high band of that axis)
 *     is written to output channel s*C + c, so after two levels channel
 *     (8*s2 + s1)*C + c; the 2D path uses s = 2*by + bx and (4*s2 + s1)*C + c;
 *   - the replicated frame is placed in front (p_0 = v_0, p_t = v_{t-1});
 *     the inverse drops the first reconstructed frame (the replica);
 *   - T == 1 takes the 2D (image) path; otherwise T % 4 == 1 is required.
 *
 * Arrays are dense, row-major, W fastest:
 *   x : [B][C][T][H][W]
 *   y : [B][64C][(T+3)/4][H/4][W/4]   (T > 1)
 *       [B][16C][1][H/4][W/4]         (T == 1)
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

#define ORACLE_OK 0
#define ORACLE_BAD_SHAPE 2
#define ORACLE_NO_MEMORY 7

/* 1/sqrt(2), the orthonormal Haar tap. */
static const double HAAR_S = 0.70710678118654752440084436210484903928;

/* One butterfly on the pair (a, b): low and high band. */
static void haar_pair(double a, double b, double *lo, double *hi)
{
    *lo = (a + b) * HAAR_S;
    *hi = (a - b) * HAAR_S;
}

/* The inverse butterfly: rebuild (a, b) from (low, high). */
static void haar_unpair(double lo, double hi, double *a, double *b)
{
    *a = (lo + hi) * HAAR_S;
    *b = (lo - hi) * HAAR_S;
}

/*
 * One level of the causal 3D DWT (Patcher3D in section 7.1 of the guide):
 * v[C][T][H][W] -> o[8C][(T+1)/2][H/2][W/2], T odd.
 *   1. The time axis is extended to T+1 frames by a copy of frame 0 in front:
 *      p_0 = v_0 and p_t = v_{t-1} for t >= 1.
 *   2. Each 2x2x2 group p[2j+dt][2i+dy][2k+dx] is paired along t, then y,
 *      then x; every pair gives a low and a high band.
 *   3. Subband s = 4*bt + 2*by + bx goes to channel s*C + c.
 */
static void level3d_fwd(const double *v, double *o, int64_t C, int64_t T, int64_t H, int64_t W)
{
    const int64_t To = (T + 1) / 2, Ho = H / 2, Wo = W / 2;
    for (int64_t c = 0; c < C; ++c)
        for (int64_t j = 0; j < To; ++j)
            for (int64_t i = 0; i < Ho; ++i)
                for (int64_t k = 0; k < Wo; ++k) {
                    double g[2][2][2]; /* [dt][dy][dx], later [bt][by][bx] */
                    for (int dt = 0; dt < 2; ++dt) {
                        const int64_t pt = 2 * j + dt;            /* frame of p */
                        const int64_t vt = (pt == 0) ? 0 : pt - 1; /* frame of v */
                        for (int dy = 0; dy < 2; ++dy)
                            for (int dx = 0; dx < 2; ++dx)
                                g[dt][dy][dx] = v[((c * T + vt) * H + (2 * i + dy)) * W + (2 * k + dx)];
                    }
                    for (int dy = 0; dy < 2; ++dy) /* along t */
                        for (int dx = 0; dx < 2; ++dx)
                            haar_pair(g[0][dy][dx], g[1][dy][dx], &g[0][dy][dx], &g[1][dy][dx]);
                    for (int bt = 0; bt < 2; ++bt) /* along y */
                        for (int dx = 0; dx < 2; ++dx)
                            haar_pair(g[bt][0][dx], g[bt][1][dx], &g[bt][0][dx], &g[bt][1][dx]);
                    for (int bt = 0; bt < 2; ++bt) /* along x */
                        for (int by = 0; by < 2; ++by)
                            haar_pair(g[bt][by][0], g[bt][by][1], &g[bt][by][0], &g[bt][by][1]);
                    for (int bt = 0; bt < 2; ++bt)
                        for (int by = 0; by < 2; ++by)
                            for (int bx = 0; bx < 2; ++bx) {
                                const int64_t s = 4 * bt + 2 * by + bx;
                                o[(((s * C + c) * To + j) * Ho + i) * Wo + k] = g[bt][by][bx];
                            }
                }
}

/*
 * Inverse of level3d_fwd: o[8C][To][Ho][Wo] -> v[C][2*To-1][2*Ho][2*Wo].
 * Each group is rebuilt by inverse butterflies along x, y and t, which gives
 * 2*To frames p_0 .. p_{2To-1}; the first one is the replicated copy of frame
 * 0 and is dropped: v_t = p_{t+1}.
 */
static void level3d_inv(const double *o, double *v, int64_t C, int64_t To, int64_t Ho, int64_t Wo)
{
    const int64_t T = 2 * To - 1, H = 2 * Ho, W = 2 * Wo;
    for (int64_t c = 0; c < C; ++c)
        for (int64_t j = 0; j < To; ++j)
            for (int64_t i = 0; i < Ho; ++i)
                for (int64_t k = 0; k < Wo; ++k) {
                    double g[2][2][2];
                    for (int bt = 0; bt < 2; ++bt)
                        for (int by = 0; by < 2; ++by)
                            for (int bx = 0; bx < 2; ++bx) {
                                const int64_t s = 4 * bt + 2 * by + bx;
                                g[bt][by][bx] = o[(((s * C + c) * To + j) * Ho + i) * Wo + k];
                            }
                    for (int bt = 0; bt < 2; ++bt) /* along x */
                        for (int by = 0; by < 2; ++by)
                            haar_unpair(g[bt][by][0], g[bt][by][1], &g[bt][by][0], &g[bt][by][1]);
                    for (int bt = 0; bt < 2; ++bt) /* along y */
                        for (int dx = 0; dx < 2; ++dx)
                            haar_unpair(g[bt][0][dx], g[bt][1][dx], &g[bt][0][dx], &g[bt][1][dx]);
                    for (int dy = 0; dy < 2; ++dy) /* along t */
                        for (int dx = 0; dx < 2; ++dx)
                            haar_unpair(g[0][dy][dx], g[1][dy][dx], &g[0][dy][dx], &g[1][dy][dx]);
                    for (int dt = 0; dt < 2; ++dt) {
                        const int64_t pt = 2 * j + dt;
                        if (pt == 0)
                            continue; /* the replica of frame 0 */
                        for (int dy = 0; dy < 2; ++dy)
                            for (int dx = 0; dx < 2; ++dx)
                                v[((c * T + (pt - 1)) * H + (2 * i + dy)) * W + (2 * k + dx)] = g[dt][dy][dx];
                    }
                }
}

/*
 * One level of the 2D DWT (Patcher in section 7.1 of the guide):
 * v[C][H][W] -> o[4C][H/2][W/2], subband s = 2*by + bx to channel s*C + c.
 */
static void level2d_fwd(const double *v, double *o, int64_t C, int64_t H, int64_t W)
{
    const int64_t Ho = H / 2, Wo = W / 2;
    for (int64_t c = 0; c < C; ++c)
        for (int64_t i = 0; i < Ho; ++i)
            for (int64_t k = 0; k < Wo; ++k) {
                double g[2][2];
                for (int dy = 0; dy < 2; ++dy)
                    for (int dx = 0; dx < 2; ++dx)
                        g[dy][dx] = v[(c * H + (2 * i + dy)) * W + (2 * k + dx)];
                for (int dx = 0; dx < 2; ++dx) /* along y */
                    haar_pair(g[0][dx], g[1][dx], &g[0][dx], &g[1][dx]);
                for (int by = 0; by < 2; ++by) /* along x */
                    haar_pair(g[by][0], g[by][1], &g[by][0], &g[by][1]);
                for (int by = 0; by < 2; ++by)
                    for (int bx = 0; bx < 2; ++bx) {
                        const int64_t s = 2 * by + bx;
                        o[((s * C + c) * Ho + i) * Wo + k] = g[by][bx];
                    }
            }
}

/* Inverse of level2d_fwd: o[4C][Ho][Wo] -> v[C][2Ho][2Wo]. */
static void level2d_inv(const double *o, double *v, int64_t C, int64_t Ho, int64_t Wo)
{
    const int64_t H = 2 * Ho, W = 2 * Wo;
    for (int64_t c = 0; c < C; ++c)
        for (int64_t i = 0; i < Ho; ++i)
            for (int64_t k = 0; k < Wo; ++k) {
                double g[2][2];
                for (int by = 0; by < 2; ++by)
                    for (int bx = 0; bx < 2; ++bx)
                        g[by][bx] = o[((((int64_t)(2 * by + bx)) * C + c) * Ho + i) * Wo + k];
                for (int by = 0; by < 2; ++by) /* along x */
                    haar_unpair(g[by][0], g[by][1], &g[by][0], &g[by][1]);
                for (int dx = 0; dx < 2; ++dx) /* along y */
                    haar_unpair(g[0][dx], g[1][dx], &g[0][dx], &g[1][dx]);
                for (int dy = 0; dy < 2; ++dy)
                    for (int dx = 0; dx < 2; ++dx)
                        v[(c * H + (2 * i + dy)) * W + (2 * k + dx)] = g[dy][dx];
            }
}

static int shape_ok(int64_t B, int64_t C, int64_t T, int64_t H, int64_t W)
{
    if (B < 0 || C < 0 || T < 1 || H < 0 || W < 0)
        return 0;
    if (H % 4 != 0 || W % 4 != 0)
        return 0;
    return T == 1 || T % 4 == 1;
}

/* Output frames of the two-level patcher: 1 + (T-1)/4 (guide, sections 6.1 and 7.3). */
int64_t oracle_haar_out_frames(int64_t T)
{
    return T == 1 ? 1 : 1 + (T - 1) / 4;
}

/*
 * Single level, exposed for the self-test: 3D if T > 1 (T odd), else 2D.
 * x: [C][T][H][W] -> y: [8C][(T+1)/2][H/2][W/2] or [4C][H/2][W/2].
 */
int oracle_haar_level_fwd(const double *x, double *y, int64_t C, int64_t T, int64_t H, int64_t W)
{
    if (C < 0 || T < 1 || H % 2 || W % 2 || (T > 1 && T % 2 == 0))
        return ORACLE_BAD_SHAPE;
    if (T == 1)
        level2d_fwd(x, y, C, H, W);
    else
        level3d_fwd(x, y, C, T, H, W);
    return ORACLE_OK;
}

/*
 * Single level inverse (the unpatcher with patch_size=2), T, H, W the pixel
 * extents: y [4C][1][H/2][W/2] (T == 1) or [8C][(T+1)/2][H/2][W/2] -> x [C][T][H][W].
 */
int oracle_haar_level_inv(const double *y, double *x, int64_t C, int64_t T, int64_t H, int64_t W)
{
    if (C < 0 || T < 1 || H % 2 || W % 2 || (T > 1 && T % 2 == 0))
        return ORACLE_BAD_SHAPE;
    if (T == 1)
        level2d_inv(y, x, C, H / 2, W / 2);
    else
        level3d_inv(y, x, C, (T + 1) / 2, H / 2, W / 2);
    return ORACLE_OK;
}

/*
 * Two-level patcher (patch_size=4): the single level applied twice, the second
 * time to all 8C (or 4C) first-level channels.
 */
int oracle_haar_fwd(const double *x, double *y, int64_t B, int64_t C, int64_t T, int64_t H, int64_t W)
{
    if (!shape_ok(B, C, T, H, W))
        return ORACLE_BAD_SHAPE;
    const int64_t nx = C * T * H * W;
    const int64_t T1 = (T == 1) ? 1 : (T + 1) / 2;
    const int64_t C1 = (T == 1) ? 4 * C : 8 * C;
    const int64_t n1 = C1 * T1 * (H / 2) * (W / 2);
    const int64_t ny = (T == 1 ? 16 * C : 64 * C) * oracle_haar_out_frames(T) * (H / 4) * (W / 4);
    if (nx == 0 || B == 0)
        return ORACLE_OK;
    double *mid = (double *)malloc((size_t)n1 * sizeof(double));
    if (!mid)
        return ORACLE_NO_MEMORY;
    for (int64_t b = 0; b < B; ++b) {
        if (T == 1) {
            level2d_fwd(x + b * nx, mid, C, H, W);
            level2d_fwd(mid, y + b * ny, C1, H / 2, W / 2);
        } else {
            level3d_fwd(x + b * nx, mid, C, T, H, W);
            level3d_fwd(mid, y + b * ny, C1, T1, H / 2, W / 2);
        }
    }
    free(mid);
    return ORACLE_OK;
}

/*
 * Two-level unpatcher: level 2 is undone first (on all 8C or 4C groups), then
 * level 1.  T, H, W are the pixel-space extents.
 */
int oracle_haar_inv(const double *y, double *x, int64_t B, int64_t C, int64_t T, int64_t H, int64_t W)
{
    if (!shape_ok(B, C, T, H, W))
        return ORACLE_BAD_SHAPE;
    const int64_t nx = C * T * H * W;
    const int64_t Tq = oracle_haar_out_frames(T);
    const int64_t T1 = (T == 1) ? 1 : 2 * Tq - 1;
    const int64_t C1 = (T == 1) ? 4 * C : 8 * C;
    const int64_t n1 = C1 * T1 * (H / 2) * (W / 2);
    const int64_t ny = (T == 1 ? 16 * C : 64 * C) * Tq * (H / 4) * (W / 4);
    if (nx == 0 || B == 0)
        return ORACLE_OK;
    double *mid = (double *)malloc((size_t)n1 * sizeof(double));
    if (!mid)
        return ORACLE_NO_MEMORY;
    for (int64_t b = 0; b < B; ++b) {
        if (T == 1) {
            level2d_inv(y + b * ny, mid, C1, H / 4, W / 4);
            level2d_inv(mid, x + b * nx, C, H / 2, W / 2);
        } else {
            level3d_inv(y + b * ny, mid, C1, Tq, H / 4, W / 4);
            level3d_inv(mid, x + b * nx, C, T1, H / 2, W / 2);
        }
    }
    free(mid);
    return ORACLE_OK;
}

/*
 * Adjoints (transposes), for gradients.  Each level of the forward is a
 * replication R (frame 0 copied in front) followed by pair butterflies P; the
 * butterfly matrix [[s, s], [s, -s]] is symmetric, so P^T = P^-1 is the inverse
 * butterfly, and R^T adds the copy's gradient into frame 0.  So the adjoint of a
 * level is the inverse level with the first reconstructed frame ADDED to frame
 * 0 instead of dropped, and the adjoint of the two-level patcher applies the
 * level-2 adjoint first.  The unpatcher is (drop the first frame) after inverse
 * butterflies, per level, level 2 first; its adjoint puts a zero frame in front
 * (the dropped frame gets no gradient) and applies the forward butterflies,
 * level 1 first.
 */
static void level3d_adj(const double *o, double *v, int64_t C, int64_t To, int64_t Ho, int64_t Wo)
{
    const int64_t T = 2 * To - 1, H = 2 * Ho, W = 2 * Wo;
    for (int64_t c = 0; c < C; ++c)
        for (int64_t j = 0; j < To; ++j)
            for (int64_t i = 0; i < Ho; ++i)
                for (int64_t k = 0; k < Wo; ++k) {
                    double g[2][2][2];
                    for (int bt = 0; bt < 2; ++bt)
                        for (int by = 0; by < 2; ++by)
                            for (int bx = 0; bx < 2; ++bx)
                                g[bt][by][bx] = o[((((int64_t)(4 * bt + 2 * by + bx) * C + c) * To + j) * Ho + i) * Wo + k];
                    for (int bt = 0; bt < 2; ++bt) /* P^T along x */
                        for (int by = 0; by < 2; ++by)
                            haar_unpair(g[bt][by][0], g[bt][by][1], &g[bt][by][0], &g[bt][by][1]);
                    for (int bt = 0; bt < 2; ++bt) /* along y */
                        for (int dx = 0; dx < 2; ++dx)
                            haar_unpair(g[bt][0][dx], g[bt][1][dx], &g[bt][0][dx], &g[bt][1][dx]);
                    for (int dy = 0; dy < 2; ++dy) /* along t */
                        for (int dx = 0; dx < 2; ++dx)
                            haar_unpair(g[0][dy][dx], g[1][dy][dx], &g[0][dy][dx], &g[1][dy][dx]);
                    for (int dt = 0; dt < 2; ++dt) {
                        const int64_t pt = 2 * j + dt;
                        const int64_t vt = (pt == 0) ? 0 : pt - 1; /* R^T: the copy lands on frame 0 */
                        for (int dy = 0; dy < 2; ++dy)
                            for (int dx = 0; dx < 2; ++dx) {
                                double *dst = &v[((c * T + vt) * H + (2 * i + dy)) * W + (2 * k + dx)];
                                if (pt == 0)
                                    *dst = g[dt][dy][dx];
                                else if (pt == 1)
                                    *dst += g[dt][dy][dx];
                                else
                                    *dst = g[dt][dy][dx];
                            }
                    }
                }
}

/* Adjoint of level3d_inv: v[C][2To-1][2Ho][2Wo] -> o[8C][To][Ho][Wo]. */
static void level3d_inv_adj(const double *v, double *o, int64_t C, int64_t To, int64_t Ho, int64_t Wo)
{
    const int64_t T = 2 * To - 1, H = 2 * Ho, W = 2 * Wo;
    for (int64_t c = 0; c < C; ++c)
        for (int64_t j = 0; j < To; ++j)
            for (int64_t i = 0; i < Ho; ++i)
                for (int64_t k = 0; k < Wo; ++k) {
                    double g[2][2][2];
                    for (int dt = 0; dt < 2; ++dt) {
                        const int64_t pt = 2 * j + dt; /* the dropped frame p_0 has no gradient */
                        for (int dy = 0; dy < 2; ++dy)
                            for (int dx = 0; dx < 2; ++dx)
                                g[dt][dy][dx] =
                                    pt == 0 ? 0.0 : v[((c * T + (pt - 1)) * H + (2 * i + dy)) * W + (2 * k + dx)];
                    }
                    for (int dy = 0; dy < 2; ++dy) /* along t: the inverse butterfly's transpose */
                        for (int dx = 0; dx < 2; ++dx)
                            haar_pair(g[0][dy][dx], g[1][dy][dx], &g[0][dy][dx], &g[1][dy][dx]);
                    for (int bt = 0; bt < 2; ++bt) /* along y */
                        for (int dx = 0; dx < 2; ++dx)
                            haar_pair(g[bt][0][dx], g[bt][1][dx], &g[bt][0][dx], &g[bt][1][dx]);
                    for (int bt = 0; bt < 2; ++bt) /* along x */
                        for (int by = 0; by < 2; ++by)
                            haar_pair(g[bt][by][0], g[bt][by][1], &g[bt][by][0], &g[bt][by][1]);
                    for (int bt = 0; bt < 2; ++bt)
                        for (int by = 0; by < 2; ++by)
                            for (int bx = 0; bx < 2; ++bx)
                                o[((((int64_t)(4 * bt + 2 * by + bx) * C + c) * To + j) * Ho + i) * Wo + k] =
                                    g[bt][by][bx];
                }
}

/* Gradient of the two-level patcher: gy (coefficient shape) -> gx (pixel shape). Video only. */
int oracle_haar_fwd_adjoint(const double *gy, double *gx, int64_t B, int64_t C, int64_t T, int64_t H, int64_t W)
{
    if (!shape_ok(B, C, T, H, W) || T == 1)
        return ORACLE_BAD_SHAPE;
    const int64_t nx = C * T * H * W, Tq = oracle_haar_out_frames(T), T1 = 2 * Tq - 1;
    const int64_t n1 = 8 * C * T1 * (H / 2) * (W / 2), ny = 64 * C * Tq * (H / 4) * (W / 4);
    if (nx == 0 || B == 0)
        return ORACLE_OK;
    double *mid = (double *)malloc((size_t)n1 * sizeof(double));
    if (!mid)
        return ORACLE_NO_MEMORY;
    for (int64_t b = 0; b < B; ++b) {
        level3d_adj(gy + b * ny, mid, 8 * C, Tq, H / 4, W / 4);
        level3d_adj(mid, gx + b * nx, C, T1, H / 2, W / 2);
    }
    free(mid);
    return ORACLE_OK;
}

/* Gradient of the two-level unpatcher: gx (pixel shape) -> gy (coefficient shape). Video only. */
int oracle_haar_inv_adjoint(const double *gx, double *gy, int64_t B, int64_t C, int64_t T, int64_t H, int64_t W)
{
    if (!shape_ok(B, C, T, H, W) || T == 1)
        return ORACLE_BAD_SHAPE;
    const int64_t nx = C * T * H * W, Tq = oracle_haar_out_frames(T), T1 = 2 * Tq - 1;
    const int64_t n1 = 8 * C * T1 * (H / 2) * (W / 2), ny = 64 * C * Tq * (H / 4) * (W / 4);
    if (nx == 0 || B == 0)
        return ORACLE_OK;
    double *mid = (double *)malloc((size_t)n1 * sizeof(double));
    if (!mid)
        return ORACLE_NO_MEMORY;
    for (int64_t b = 0; b < B; ++b) {
        level3d_inv_adj(gx + b * nx, mid, C, T1, H / 2, W / 2);
        level3d_inv_adj(mid, gy + b * ny, 8 * C, Tq, H / 4, W / 4);
    }
    free(mid);
    return ORACLE_OK;
}

/*
 * Second, independent statement of the two-level forward transform, used only
 * to pin the level-by-level form above.  It is derived from the definition:
 *   - two full-packet levels on four samples x0..x3 give the 4-point
 *     Walsh-Hadamard transform, coefficient k = 2*b2 + b1 (level-2 band bit,
 *     level-1 band bit) equal to (1/2) * sum_n (-1)^popcount(k & n) x_n;
 *   - the two frame-0 replications compose: output frame 0 reads four copies
 *     of x_0, output frame t' >= 1 reads frames 4t'-3 .. 4t'.
 * So every output is (1/8) * a signed sum over one 4x4x4 block (1/4 over a
 * 4x4 block on the 2D path), channel (8*s2 + s1)*C + c with
 * s_l = 4*bt_l + 2*by_l + bx_l.
 */
static int parity_of(int v)
{
    int p = 0;
    while (v) {
        p ^= v & 1;
        v >>= 1;
    }
    return p;
}

int oracle_haar_fwd_blockform(const double *x, double *y, int64_t B, int64_t C, int64_t T, int64_t H,
                              int64_t W)
{
    if (!shape_ok(B, C, T, H, W))
        return ORACLE_BAD_SHAPE;
    const int64_t Tq = oracle_haar_out_frames(T), h = H / 4, w = W / 4;
    const int is3d = T > 1;
    const int64_t Cout = (is3d ? 64 : 16) * C;
    const int nt = is3d ? 4 : 1;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t c = 0; c < C; ++c)
            for (int64_t tq = 0; tq < Tq; ++tq)
                for (int64_t i = 0; i < h; ++i)
                    for (int64_t j = 0; j < w; ++j)
                        for (int kt = 0; kt < nt; ++kt)
                            for (int ky = 0; ky < 4; ++ky)
                                for (int kx = 0; kx < 4; ++kx) {
                                    double acc = 0.0;
                                    for (int a = 0; a < nt; ++a) {
                                        const int64_t f = (!is3d || tq == 0) ? 0 : 4 * tq - 3 + a;
                                        for (int by = 0; by < 4; ++by)
                                            for (int bx = 0; bx < 4; ++bx) {
                                                const int sgn = parity_of(kt & a) ^ parity_of(ky & by) ^
                                                                parity_of(kx & bx);
                                                const double v =
                                                    x[(((b * C + c) * T + f) * H + 4 * i + by) * W + 4 * j + bx];
                                                acc += sgn ? -v : v;
                                            }
                                    }
                                    int64_t ch;
                                    if (is3d) {
                                        const int s2 = 4 * (kt >> 1) + 2 * (ky >> 1) + (kx >> 1);
                                        const int s1 = 4 * (kt & 1) + 2 * (ky & 1) + (kx & 1);
                                        ch = (8 * s2 + s1) * C + c;
                                    } else {
                                        const int s2 = 2 * (ky >> 1) + (kx >> 1);
                                        const int s1 = 2 * (ky & 1) + (kx & 1);
                                        ch = (4 * s2 + s1) * C + c;
                                    }
                                    y[(((b * Cout + ch) * Tq + tq) * h + i) * w + j] = acc / (is3d ? 8.0 : 4.0);
                                }
    return ORACLE_OK;
}

/*
 * Arbitrary extents and streaming time ("NVIDIA Cosmos Tokenizer 完全指南",
 * section 6.3: videos of any size are padded -- zeros in space, reflection at the
 * temporal edge -- to aligned extents before the network, and the result is
 * cropped back afterwards; long videos run window by window).
 *
 * Readings where the pages are silent (parity unpinned by the pages for the
 * choice of multiples and of the reflection form; these are conventions shared
 * with the CUDA path):
 *   - spatial padding appends zero rows at the bottom and zero columns at the
 *     right up to multiples of `ms` (a multiple of 4);
 *   - temporal padding appends frames at the end, up to the smallest Tp >= T
 *     with (Tp - 1) % mt == 0 (mt a multiple of 4), each a mirror image about
 *     the last frame without repeating it (frame T-1+k is frame T-1-k), the
 *     mirroring repeated with period 2(T-1) when more frames are needed than
 *     the clip has; images (T == 1) get no temporal padding;
 *   - the padded clip goes through the two-level patcher unchanged; the
 *     unpatcher's output is cropped to the first T frames, H rows, W columns;
 *   - a continuation chunk (streaming) is a run of 4k frames that follows
 *     earlier frames: it is transformed level by level with no frame-0
 *     replica (frames paired as they come), giving k latent frames; the first
 *     chunk (1 + 4k frames, k >= 0) is the start of a video and always takes
 *     the 3D levels, so a one-frame first chunk gives latent frame 0.
 */

/* Padded extents; returns 0 if the multiples or the shape are invalid. */
int oracle_haar_padded_extents(int64_t T, int64_t H, int64_t W, int64_t ms, int64_t mt, int64_t *Tp, int64_t *Hp,
                               int64_t *Wp)
{
    if (T < 1 || H < 0 || W < 0 || ms < 4 || ms % 4 != 0 || mt < 4 || mt % 4 != 0)
        return 0;
    *Hp = (H + ms - 1) / ms * ms;
    *Wp = (W + ms - 1) / ms * ms;
    *Tp = (T == 1) ? 1 : 1 + (T - 1 + mt - 1) / mt * mt;
    return 1;
}

/* Source frame of padded frame t (mirror about the last frame, period 2(T-1)). */
static int64_t reflect_frame(int64_t t, int64_t T)
{
    if (t < T)
        return t;
    if (T == 1)
        return 0;
    const int64_t period = 2 * (T - 1);
    const int64_t r = t % period;
    return r < T ? r : period - r;
}

/* x [B][C][T][H][W] -> xp [B][C][Tp][Hp][Wp]. */
int oracle_haar_pad(const double *x, double *xp, int64_t B, int64_t C, int64_t T, int64_t H, int64_t W, int64_t Tp,
                    int64_t Hp, int64_t Wp)
{
    if (Tp < T || Hp < H || Wp < W)
        return ORACLE_BAD_SHAPE;
    for (int64_t bc = 0; bc < B * C; ++bc)
        for (int64_t t = 0; t < Tp; ++t) {
            const int64_t ts = reflect_frame(t, T);
            for (int64_t y = 0; y < Hp; ++y)
                for (int64_t xx = 0; xx < Wp; ++xx)
                    xp[((bc * Tp + t) * Hp + y) * Wp + xx] =
                        (y < H && xx < W) ? x[((bc * T + ts) * H + y) * W + xx] : 0.0;
        }
    return ORACLE_OK;
}

/* Padded patcher: pad, then the two-level patcher on [B][C][Tp][Hp][Wp]. */
int oracle_haar_fwd_padded(const double *x, double *y, int64_t B, int64_t C, int64_t T, int64_t H, int64_t W,
                           int64_t ms, int64_t mt)
{
    int64_t Tp, Hp, Wp;
    if (B < 0 || C < 0 || !oracle_haar_padded_extents(T, H, W, ms, mt, &Tp, &Hp, &Wp))
        return ORACLE_BAD_SHAPE;
    if (B * C * Tp * Hp * Wp == 0)
        return ORACLE_OK;
    double *xp = (double *)malloc((size_t)(B * C * Tp * Hp * Wp) * sizeof(double));
    if (!xp)
        return ORACLE_NO_MEMORY;
    int rc = oracle_haar_pad(x, xp, B, C, T, H, W, Tp, Hp, Wp);
    if (rc == ORACLE_OK)
        rc = oracle_haar_fwd(xp, y, B, C, Tp, Hp, Wp);
    free(xp);
    return rc;
}

/* Cropped unpatcher: the two-level unpatcher on the padded extents, then the first
 * T frames, H rows and W columns. */
int oracle_haar_inv_cropped(const double *y, double *x, int64_t B, int64_t C, int64_t T, int64_t H, int64_t W,
                            int64_t ms, int64_t mt)
{
    int64_t Tp, Hp, Wp;
    if (B < 0 || C < 0 || !oracle_haar_padded_extents(T, H, W, ms, mt, &Tp, &Hp, &Wp))
        return ORACLE_BAD_SHAPE;
    if (B * C * Tp * Hp * Wp == 0)
        return ORACLE_OK;
    double *xp = (double *)malloc((size_t)(B * C * Tp * Hp * Wp) * sizeof(double));
    if (!xp)
        return ORACLE_NO_MEMORY;
    const int rc = oracle_haar_inv(y, xp, B, C, Tp, Hp, Wp);
    if (rc == ORACLE_OK)
        for (int64_t bc = 0; bc < B * C; ++bc)
            for (int64_t t = 0; t < T; ++t)
                for (int64_t yy = 0; yy < H; ++yy)
                    for (int64_t xx = 0; xx < W; ++xx)
                        x[((bc * T + t) * H + yy) * W + xx] = xp[((bc * Tp + t) * Hp + yy) * Wp + xx];
    free(xp);
    return rc;
}

/*
 * One level of the 3D DWT without the frame-0 replica (continuation chunks):
 * v[C][T][H][W] -> o[8C][T/2][H/2][W/2], T even; frames 2j and 2j+1 form pair j.
 * Same butterflies and subband order as level3d_fwd.
 */
static void level3d_fwd_norep(const double *v, double *o, int64_t C, int64_t T, int64_t H, int64_t W)
{
    const int64_t To = T / 2, Ho = H / 2, Wo = W / 2;
    for (int64_t c = 0; c < C; ++c)
        for (int64_t j = 0; j < To; ++j)
            for (int64_t i = 0; i < Ho; ++i)
                for (int64_t k = 0; k < Wo; ++k) {
                    double g[2][2][2];
                    for (int dt = 0; dt < 2; ++dt)
                        for (int dy = 0; dy < 2; ++dy)
                            for (int dx = 0; dx < 2; ++dx)
                                g[dt][dy][dx] = v[((c * T + 2 * j + dt) * H + (2 * i + dy)) * W + (2 * k + dx)];
                    for (int dy = 0; dy < 2; ++dy)
                        for (int dx = 0; dx < 2; ++dx)
                            haar_pair(g[0][dy][dx], g[1][dy][dx], &g[0][dy][dx], &g[1][dy][dx]);
                    for (int bt = 0; bt < 2; ++bt)
                        for (int dx = 0; dx < 2; ++dx)
                            haar_pair(g[bt][0][dx], g[bt][1][dx], &g[bt][0][dx], &g[bt][1][dx]);
                    for (int bt = 0; bt < 2; ++bt)
                        for (int by = 0; by < 2; ++by)
                            haar_pair(g[bt][by][0], g[bt][by][1], &g[bt][by][0], &g[bt][by][1]);
                    for (int bt = 0; bt < 2; ++bt)
                        for (int by = 0; by < 2; ++by)
                            for (int bx = 0; bx < 2; ++bx)
                                o[((((4 * bt + 2 * by + bx) * C + c) * To + j) * Ho + i) * Wo + k] = g[bt][by][bx];
                }
}

/* Inverse of level3d_fwd_norep: o[8C][To][Ho][Wo] -> v[C][2To][2Ho][2Wo], no frame dropped. */
static void level3d_inv_norep(const double *o, double *v, int64_t C, int64_t To, int64_t Ho, int64_t Wo)
{
    const int64_t T = 2 * To, H = 2 * Ho, W = 2 * Wo;
    for (int64_t c = 0; c < C; ++c)
        for (int64_t j = 0; j < To; ++j)
            for (int64_t i = 0; i < Ho; ++i)
                for (int64_t k = 0; k < Wo; ++k) {
                    double g[2][2][2];
                    for (int bt = 0; bt < 2; ++bt)
                        for (int by = 0; by < 2; ++by)
                            for (int bx = 0; bx < 2; ++bx)
                                g[bt][by][bx] = o[((((4 * bt + 2 * by + bx) * C + c) * To + j) * Ho + i) * Wo + k];
                    for (int bt = 0; bt < 2; ++bt)
                        for (int by = 0; by < 2; ++by)
                            haar_unpair(g[bt][by][0], g[bt][by][1], &g[bt][by][0], &g[bt][by][1]);
                    for (int bt = 0; bt < 2; ++bt)
                        for (int dx = 0; dx < 2; ++dx)
                            haar_unpair(g[bt][0][dx], g[bt][1][dx], &g[bt][0][dx], &g[bt][1][dx]);
                    for (int dy = 0; dy < 2; ++dy)
                        for (int dx = 0; dx < 2; ++dx)
                            haar_unpair(g[0][dy][dx], g[1][dy][dx], &g[0][dy][dx], &g[1][dy][dx]);
                    for (int dt = 0; dt < 2; ++dt)
                        for (int dy = 0; dy < 2; ++dy)
                            for (int dx = 0; dx < 2; ++dx)
                                v[((c * T + 2 * j + dt) * H + (2 * i + dy)) * W + (2 * k + dx)] = g[dt][dy][dx];
                }
}

/*
 * Streaming chunk of a video: first != 0 is the start of the video, T = 1 + 4k
 * frames (k >= 0), transformed by the two 3D levels with their frame-0 replicas
 * (a one-frame first chunk gives the video's latent frame 0, not the image
 * transform); first == 0 is a continuation chunk of T = 4k frames (k >= 1),
 * transformed by two levels without replicas.  Output [B][64C][(T+3)/4 or T/4][H/4][W/4].
 */
static int chunk_shape_ok(int64_t B, int64_t C, int64_t T, int64_t H, int64_t W, int first)
{
    if (B < 0 || C < 0 || H < 0 || W < 0 || H % 4 != 0 || W % 4 != 0)
        return 0;
    return first ? (T >= 1 && T % 4 == 1) : (T >= 4 && T % 4 == 0);
}

int oracle_haar_fwd_chunk(const double *x, double *y, int64_t B, int64_t C, int64_t T, int64_t H, int64_t W,
                          int first)
{
    if (!chunk_shape_ok(B, C, T, H, W, first))
        return ORACLE_BAD_SHAPE;
    const int64_t T1 = first ? (T + 1) / 2 : T / 2, Tq = first ? (T1 + 1) / 2 : T1 / 2;
    const int64_t nx = C * T * H * W, n1 = 8 * C * T1 * (H / 2) * (W / 2);
    const int64_t ny = 64 * C * Tq * (H / 4) * (W / 4);
    if (nx == 0 || B == 0)
        return ORACLE_OK;
    double *mid = (double *)malloc((size_t)n1 * sizeof(double));
    if (!mid)
        return ORACLE_NO_MEMORY;
    for (int64_t b = 0; b < B; ++b) {
        if (first) {
            level3d_fwd(x + b * nx, mid, C, T, H, W);
            level3d_fwd(mid, y + b * ny, 8 * C, T1, H / 2, W / 2);
        } else {
            level3d_fwd_norep(x + b * nx, mid, C, T, H, W);
            level3d_fwd_norep(mid, y + b * ny, 8 * C, T1, H / 2, W / 2);
        }
    }
    free(mid);
    return ORACLE_OK;
}

/* Inverse of oracle_haar_fwd_chunk (T, H, W: the chunk's pixel extents). */
int oracle_haar_inv_chunk(const double *y, double *x, int64_t B, int64_t C, int64_t T, int64_t H, int64_t W,
                          int first)
{
    if (!chunk_shape_ok(B, C, T, H, W, first))
        return ORACLE_BAD_SHAPE;
    const int64_t T1 = first ? (T + 1) / 2 : T / 2, Tq = first ? (T1 + 1) / 2 : T1 / 2;
    const int64_t nx = C * T * H * W, n1 = 8 * C * T1 * (H / 2) * (W / 2);
    const int64_t ny = 64 * C * Tq * (H / 4) * (W / 4);
    if (nx == 0 || B == 0)
        return ORACLE_OK;
    double *mid = (double *)malloc((size_t)n1 * sizeof(double));
    if (!mid)
        return ORACLE_NO_MEMORY;
    for (int64_t b = 0; b < B; ++b) {
        if (first) {
            level3d_inv(y + b * ny, mid, 8 * C, Tq, H / 4, W / 4);
            level3d_inv(mid, x + b * nx, C, T1, H / 2, W / 2);
        } else {
            level3d_inv_norep(y + b * ny, mid, 8 * C, Tq, H / 4, W / 4);
            level3d_inv_norep(mid, x + b * nx, C, T1, H / 2, W / 2);
        }
    }
    free(mid);
    return ORACLE_OK;
}
