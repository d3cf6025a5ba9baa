/*
 * FSQ (finite scalar quantization) oracle.  TEST INFRASTRUCTURE ONLY: the test
 * suite, the smoke check and the benchmark's CPU-baseline leg load this
 * file's library; the product path never does.  It shares no code, header or
 * table with the CUDA library.
 *
 * What the pages fix (page title, section):
 *   - "NVIDIA Cosmos Tokenizer 完全指南", section 7.2 (FSQ): each of the six
 *     latent channels is quantized on its own with levels [8,8,8,5,5,5]; the
 *     range is limited by a tanh-based bound and then rounded (a
 *     straight-through round in training); the implicit codebook has
 *     8*8*8*5*5*5 = 64000 entries and needs no embedding table; the index is
 *     a mixed-radix number (codes_to_indices with a basis), undone by
 *     indices_to_codes.  Section 6.2: indices have shape [B,t,h,w] and codes
 *     [B,6,t,h,w].  Section 12: the quantizer follows the conventions of the
 *     open-source FSQ code it derives from.
 *   - "Cosmos World Foundation Model Platform for Physical AI (Cosmos-Predict1)"
 *     notes, model architecture, item 1: FSQ with a 6-dim latent and levels
 *     (8,8,8,5,5,5), vocabulary 64,000.
 *
 * Readings where the pages are silent (shared with the CUDA path):
 *   - bound, as in the published FSQ method (Mentzer et al., 2023): for a
 *     channel with L levels, half = (L-1)(1+eps)/2, off = 0.5 for even L and
 *     0 for odd L, shift = atanh(off/half); v = tanh(z + shift)*half - off;
 *     q = round(v), ties to even.  eps = 1e-3.  This yields exactly L integers
 *     q in [-floor(L/2), ceil(L/2)-1] and maps z = 0 to q = 0.  Parity
 *     unpinned by the pages for eps and the even-level offset: they are pinned
 *     only through their consequences (level counts, centre code, symmetry).
 *   - digit d = q + floor(L/2) in [0, L); index = sum_i d_i * basis_i with
 *     channel 0 least significant, basis = (1, 8, 64, 512, 2560, 12800);
 *     indices are 0-based, in [0, 64000).
 *   - normalized code zhat = q / floor(L/2): what "codes" holds and what the
 *     decoder projects.
 *   - projection (not on the pages): encode z_i = sum_c W[i][c] u_c with W
 *     [6][C] row-major and no bias; decode out_c = sum_i W[i][c] zhat_i.
 *   - the quantization decision is taken on an fp32 z, the kernel's own
 *     precision: z_i is the chain z = fmaf(W[i][c], u_c, z) over c = 0..C-1
 *     starting from 0.0f (fmaf rounds once, so this value is fixed by the
 *     definition alone); the bound is then evaluated in double.
 *   - a token is "near a boundary" when some channel has |v - (floor(v)+0.5)|
 *     below 1e-5; a disagreement there is a rounding-order effect, not a bug.
 *   - decode of an index outside [0, 64000) gives NaN for every output
 *     channel of that token and is counted.
 */
#include <math.h>
#include <stdint.h>

#define FSQ_DIM 6
#define FSQ_CODEBOOK 64000
#define FSQ_EPS 1e-3
#define FSQ_NEAR 1e-5

static const int FSQ_L[FSQ_DIM] = {8, 8, 8, 5, 5, 5};

int oracle_fsq_levels(int i)
{
    return (i >= 0 && i < FSQ_DIM) ? FSQ_L[i] : 0;
}

/* Mixed-radix place value of channel i: the product of the levels below it. */
int64_t oracle_fsq_basis(int i)
{
    int64_t p = 1;
    for (int k = 0; k < i; ++k)
        p *= FSQ_L[k];
    return p;
}

/* The tanh bound of channel i, evaluated in double. */
double oracle_fsq_bound(double z, int i)
{
    const int L = FSQ_L[i];
    const double half = (L - 1) * (1.0 + FSQ_EPS) / 2.0;
    const double off = (L % 2 == 0) ? 0.5 : 0.0;
    const double shift = atanh(off / half);
    return tanh(z + shift) * half - off;
}

/* Rounded level q of channel i for an fp32 pre-quantization value z. */
int oracle_fsq_quantize(float z, int i)
{
    return (int)nearbyint(oracle_fsq_bound((double)z, i));
}

/* codes_to_indices: digits d_i in [0, L_i) -> index. */
int64_t oracle_fsq_pack(const int *digits)
{
    int64_t idx = 0;
    for (int i = 0; i < FSQ_DIM; ++i)
        idx += (int64_t)digits[i] * oracle_fsq_basis(i);
    return idx;
}

/* indices_to_codes, first half: index -> digits. */
void oracle_fsq_unpack(int64_t idx, int *digits)
{
    for (int i = 0; i < FSQ_DIM; ++i)
        digits[i] = (int)((idx / oracle_fsq_basis(i)) % FSQ_L[i]);
}

/*
 * Encode.  u: [B][C][S] fp32; w: [6][C] fp32 row-major.
 * idx: [B][S] int32.  codes: [B][6][S] double or NULL.  near: [B][S] or NULL.
 * Returns the number of near-boundary tokens.
 */
int64_t oracle_fsq_encode(const float *u, const float *w, int64_t B, int64_t C, int64_t S, int32_t *idx,
                          double *codes, uint8_t *near)
{
    int64_t n_near = 0;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t s = 0; s < S; ++s) {
            int digits[FSQ_DIM];
            int is_near = 0;
            for (int i = 0; i < FSQ_DIM; ++i) {
                float z = 0.0f;
                for (int64_t c = 0; c < C; ++c)
                    z = fmaf(w[i * C + c], u[(b * C + c) * S + s], z);
                const double v = oracle_fsq_bound((double)z, i);
                const double q = nearbyint(v);
                if (fabs(v - (floor(v) + 0.5)) < FSQ_NEAR)
                    is_near = 1;
                const int half_width = FSQ_L[i] / 2;
                digits[i] = (int)q + half_width;
                if (codes)
                    codes[(b * FSQ_DIM + i) * S + s] = q / (double)half_width;
            }
            idx[b * S + s] = (int32_t)oracle_fsq_pack(digits);
            if (near)
                near[b * S + s] = (uint8_t)is_near;
            n_near += is_near;
        }
    return n_near;
}

/*
 * Decode.  idx: [B][S] int32; w: [6][C]; out: [B][C][S] double,
 * out_c = sum_i W[i][c] * zhat_i.  Returns the number of invalid indices.
 */
int64_t oracle_fsq_decode(const int32_t *idx, const float *w, int64_t B, int64_t C, int64_t S, double *out)
{
    int64_t bad = 0;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t s = 0; s < S; ++s) {
            const int64_t id = idx[b * S + s];
            if (id < 0 || id >= FSQ_CODEBOOK) {
                ++bad;
                for (int64_t c = 0; c < C; ++c)
                    out[(b * C + c) * S + s] = NAN;
                continue;
            }
            int digits[FSQ_DIM];
            double zhat[FSQ_DIM];
            oracle_fsq_unpack(id, digits);
            for (int i = 0; i < FSQ_DIM; ++i) {
                const int half_width = FSQ_L[i] / 2;
                zhat[i] = (double)(digits[i] - half_width) / (double)half_width;
            }
            for (int64_t c = 0; c < C; ++c) {
                double acc = 0.0;
                for (int i = 0; i < FSQ_DIM; ++i)
                    acc += (double)w[i * C + c] * zhat[i];
                out[(b * C + c) * S + s] = acc;
            }
        }
    return bad;
}

/*
 * Straight-through derivative of the normalized code of channel i with respect
 * to its pre-quantization value: round_ste passes the gradient through the
 * rounding ([guide] section 7.2), so d zhat / d z = bound'(z) / floor(L/2) =
 * half * sech^2(z + shift) / floor(L/2).  Evaluated in double.
 */
double oracle_fsq_ste_slope(double z, int i)
{
    const int L = FSQ_L[i];
    const double half = (L - 1) * (1.0 + FSQ_EPS) / 2.0;
    const double off = (L % 2 == 0) ? 0.5 : 0.0;
    const double shift = atanh(off / half);
    const double c = cosh(z + shift);
    return half / (c * c) / (double)(L / 2);
}

/*
 * Encode backward (straight-through).  u: [B][C][S] fp32, w: [6][C],
 * g: [B][6][S] fp32 (gradient of the normalized codes).  With z the same fp32
 * chain as the forward and t_i = g_i * slope_i(z_i):
 *   grad_u[b][c][s] = sum_i w[i][c] t_i          (double)
 *   grad_w[i][c]    = sum_{b,s} t_i u[b][c][s]   (double, over all tokens)
 */
void oracle_fsq_encode_backward(const float *u, const float *w, const float *g, int64_t B, int64_t C, int64_t S,
                                double *grad_u, double *grad_w)
{
    for (int64_t k = 0; k < FSQ_DIM * C; ++k)
        grad_w[k] = 0.0;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t s = 0; s < S; ++s) {
            double t[FSQ_DIM];
            for (int i = 0; i < FSQ_DIM; ++i) {
                float z = 0.0f;
                for (int64_t c = 0; c < C; ++c)
                    z = fmaf(w[i * C + c], u[(b * C + c) * S + s], z);
                t[i] = (double)g[(b * FSQ_DIM + i) * S + s] * oracle_fsq_ste_slope((double)z, i);
            }
            for (int64_t c = 0; c < C; ++c) {
                const double uc = u[(b * C + c) * S + s];
                double acc = 0.0;
                for (int i = 0; i < FSQ_DIM; ++i) {
                    acc += (double)w[i * C + c] * t[i];
                    grad_w[i * C + c] += t[i] * uc;
                }
                grad_u[(b * C + c) * S + s] = acc;
            }
        }
}

/*
 * Decode backward.  idx: [B][S], w: [6][C], g: [B][C][S] fp32 (gradient of the
 * decoded latent).  With zhat the normalized code of each token:
 *   grad_codes[b][i][s] = sum_c w[i][c] g[b][c][s]      (double)
 *   grad_w[i][c]        = sum_{b,s} zhat_i g[b][c][s]   (double)
 * Tokens with an invalid index contribute nothing and get zero code gradients.
 */
void oracle_fsq_decode_backward(const int32_t *idx, const float *w, const float *g, int64_t B, int64_t C, int64_t S,
                                double *grad_codes, double *grad_w)
{
    for (int64_t k = 0; k < FSQ_DIM * C; ++k)
        grad_w[k] = 0.0;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t s = 0; s < S; ++s) {
            const int64_t id = idx[b * S + s];
            const int valid = id >= 0 && id < FSQ_CODEBOOK;
            int digits[FSQ_DIM];
            double zhat[FSQ_DIM];
            if (valid)
                oracle_fsq_unpack(id, digits);
            for (int i = 0; i < FSQ_DIM; ++i) {
                const int half_width = FSQ_L[i] / 2;
                zhat[i] = valid ? (double)(digits[i] - half_width) / (double)half_width : 0.0;
                double acc = 0.0;
                for (int64_t c = 0; c < C; ++c) {
                    const double gc = g[(b * C + c) * S + s];
                    acc += (double)w[i * C + c] * gc;
                    grad_w[i * C + c] += zhat[i] * gc;
                }
                grad_codes[(b * FSQ_DIM + i) * S + s] = valid ? acc : 0.0;
            }
        }
}
