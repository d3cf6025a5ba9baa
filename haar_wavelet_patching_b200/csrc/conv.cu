// Entry points of the first causal factorized convolution after the patcher:
// argument checks, then the hand-written tensor-core kernels of conv_tc.cu.
//
// Source: "Cosmos World Foundation Model Platform for Physical AI (Cosmos-Predict1)"
// notes, model architecture item 1: after the 2-level Haar transform the encoder's
// convolutions are factorized -- a 1 x k x k spatial convolution, then a k x 1 x 1
// temporal convolution padded by k - 1 on the past side only.
#include "tok_common.cuh"
#include "tok_internal.h"

namespace tok {
namespace {

bool fits_int(int64_t v) { return v >= 0 && v < ((int64_t)1 << 31); }

// Shared argument rules: channels-last bf16 tensors; input channels a multiple of 64
// (one 128-byte row of the MMA's K per tap and chunk), output channels a multiple of 32
// up to 256 or a multiple of 256 (the MMA's N per CTA pair); 16-byte-aligned pointers;
// 32-bit extents.
tok_status check_conv(const void *x, const void *w, const void *y, int64_t B, int64_t T, int64_t h, int64_t wd,
                      int64_t Cin, int64_t Cout, int64_t taps, int64_t *n_in, int64_t *n_out)
{
    if (B < 0 || T < 0 || h < 0 || wd < 0 || !conv_tc_eligible(Cin, Cout))
        return TOK_ERR_SHAPE;
    int64_t pos, ni, no, nw;
    if (!prod_ok({B, T, h, wd}, &pos) || !prod_ok({pos, Cin, 2}, &ni) || !prod_ok({pos, Cout, 2}, &no) ||
        !prod_ok({Cout, taps, Cin, 2}, &nw) || !fits_int(B * T) || !fits_int(pos) || !fits_int(ni / 2) ||
        !fits_int(no / 2))
        return TOK_ERR_SHAPE;
    *n_in = ni;
    *n_out = no;
    if (pos == 0)
        return TOK_OK;
    if (!x || !w || !y)
        return TOK_ERR_NULL;
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(y, 16))
        return TOK_ERR_ALIGN;
    if (overlaps(x, ni, y, no) || overlaps(w, nw, y, no))
        return TOK_ERR_ALIAS;
    return TOK_OK;
}

tok_status spatial_call(const void *x, const void *ws, void *y, int64_t B, int64_t T, int64_t h, int64_t w,
                        int64_t Cin, int64_t Cout, int64_t k, cudaStream_t stream)
{
    if (k < 1 || k % 2 == 0 || k > 15)
        return TOK_ERR_SHAPE;
    int64_t ni, no;
    const tok_status st = check_conv(x, ws, y, B, T, h, w, Cin, Cout, k * k, &ni, &no);
    if (st != TOK_OK || B * T * h * w == 0)
        return st;
    return conv_tc_spatial(x, ws, y, B, T, h, w, Cin, Cout, k, stream);
}

tok_status temporal_call(const void *x, const void *wt, void *y, int64_t B, int64_t T, int64_t h, int64_t w,
                         int64_t Cin, int64_t Cout, int64_t k, cudaStream_t stream)
{
    if (k < 1 || k > 15)
        return TOK_ERR_SHAPE;
    int64_t ni, no;
    const tok_status st = check_conv(x, wt, y, B, T, h, w, Cin, Cout, k, &ni, &no);
    if (st != TOK_OK || B * T * h * w == 0)
        return st;
    return conv_tc_temporal(x, wt, y, B, T, h, w, Cin, Cout, k, stream);
}

} // namespace
} // namespace tok

extern "C" tok_status tok_conv_spatial(const void *x, const void *ws, void *y, int64_t B, int64_t T, int64_t h,
                                       int64_t w, int64_t Cin, int64_t Cout, int64_t k, cudaStream_t stream)
{
    return tok::spatial_call(x, ws, y, B, T, h, w, Cin, Cout, k, stream);
}

extern "C" tok_status tok_conv_temporal_causal(const void *x, const void *wt, void *y, int64_t B, int64_t T,
                                               int64_t h, int64_t w, int64_t Cin, int64_t Cout, int64_t k,
                                               cudaStream_t stream)
{
    return tok::temporal_call(x, wt, y, B, T, h, w, Cin, Cout, k, stream);
}

extern "C" tok_status tok_conv_factorized(const void *x, const void *ws, const void *wt, void *mid, void *y,
                                          int64_t B, int64_t T, int64_t h, int64_t w, int64_t Cin, int64_t Cmid,
                                          int64_t Cout, int64_t k, cudaStream_t stream)
{
    int64_t ni, nm, no;
    tok_status st = tok::check_conv(x, ws, mid, B, T, h, w, Cin, Cmid, k * k, &ni, &nm);
    if (st == TOK_OK)
        st = tok::check_conv(mid, wt, y, B, T, h, w, Cmid, Cout, k, &nm, &no);
    if (st == TOK_OK && B * T * h * w > 0 && tok::overlaps(x, ni, y, no))
        st = TOK_ERR_ALIAS;
    if (st != TOK_OK)
        return st;
    st = tok::spatial_call(x, ws, mid, B, T, h, w, Cin, Cmid, k, stream);
    if (st == TOK_OK)
        st = tok::temporal_call(mid, wt, y, B, T, h, w, Cmid, Cout, k, stream);
    return st;
}
