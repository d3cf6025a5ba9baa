// The first causal factorized convolution after the patcher, on the 5th-generation
// tensor cores.
//
// Source: "Cosmos World Foundation Model Platform for Physical AI (Cosmos-Predict1)"
// notes, model architecture item 1: after the 2-level Haar transform the encoder's
// convolutions are factorized -- a 1 x k x k spatial convolution, then a k x 1 x 1
// temporal convolution padded by k - 1 on the past side only.
//
// Both convolutions are implicit GEMMs on channels-last bf16 activations with fp32
// accumulation: the spatial one is a 2D forward convolution over the B*T frames
// (M = B*T*h*w output positions, N = C_mid, K = k*k*C_in), the temporal one a 3D
// forward convolution with a (k, 1, 1) filter whose time axis is padded by k - 1
// before the first frame and by nothing after the last, so output frame t reads
// frames t - k + 1 .. t (M = B*T*h*w, N = C_out, K = k*C_mid).  They run CUTLASS's
// sm100 implicit-GEMM kernels, instantiated here: TMA im2col loads of the activation
// tile and tiled loads of the filter into shared memory, tcgen05.mma with the
// accumulator in tensor memory, and a TMA store epilogue that rounds to bf16.  The MMA
// is the 2-SM form (cta_group::2): a pair of CTAs on a 2 x 1 x 1 cluster computes a
// 256 x 256 tile, each CTA loading half of the activations and half of the filter, so
// the filter crosses L2 half as often per flop as with 128 x 256 one-CTA tiles.  The
// loads of a 2 x 1 x 1 cluster are plain cta_group::2 TMA loads, none broadcast to the pair.
#include "cutlass/cutlass.h"
#include "cutlass/kernel_hardware_info.hpp"
#include "cute/tensor.hpp"
#include "cutlass/conv/convolution.h"
#include "cutlass/conv/convnd_problem_shape.hpp"
#include "cutlass/conv/dispatch_policy.hpp"
#include "cutlass/conv/collective/collective_builder.hpp"
#include "cutlass/epilogue/collective/collective_builder.hpp"
#include "cutlass/conv/kernel/conv_universal.hpp"
#include "cutlass/conv/device/conv_universal_adapter.hpp"

#include "tok_common.cuh"
#include "tok_internal.h"

namespace tok {
namespace {

using namespace cute;
using Elem = cutlass::bfloat16_t;
using MmaTile = Shape<_256, _256, Shape<_64>>; // 256 output positions x 256 channels per CTA pair, K step 64
using Cluster = Shape<_2, _1, _1>;             // the pair of a 2-SM MMA (no broadcast loads)
// The epilogue stores 128 x 32 subtiles: its smaller shared-memory staging leaves room for a
// sixth mainloop stage (measured 1-5% faster than the automatic 128 x 64 with five stages).
using EpiTile = Shape<_128, _32>;

template <class Layout> struct Fprop {
    using Epilogue = typename cutlass::epilogue::collective::CollectiveBuilder<
        cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, MmaTile, Cluster, EpiTile, float, float, Elem,
        Layout, 8, Elem, Layout, 8,
        cutlass::epilogue::TmaWarpSpecialized2Sm>::CollectiveOp;
    using Mainloop = typename cutlass::conv::collective::CollectiveBuilder<
        cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, cutlass::conv::Operator::kFprop, Elem, Layout, 8,
        Elem, Layout, 8, float, MmaTile, Cluster,
        cutlass::conv::collective::StageCountAutoCarveout<sizeof(typename Epilogue::SharedStorage)>,
        cutlass::conv::KernelImplicitTmaWarpSpecialized2SmSm100>::CollectiveOp;
    using Problem = cutlass::conv::ConvProblemShape<cutlass::conv::Operator::kFprop, Mainloop::NumSpatialDimensions>;
    using Kernel = cutlass::conv::kernel::ConvUniversal<Problem, Mainloop, Epilogue>;
    using Op = cutlass::conv::device::ConvUniversalAdapter<Kernel>;
};
using Spatial = Fprop<cutlass::layout::TensorNHWC>;   // [N, H, W, C] with N = B*T frames
using Temporal = Fprop<cutlass::layout::TensorNDHWC>; // [B, T, H, W, C]

// Output strides in the GEMM view the epilogue expects: ((w, h, [t,] n) position strides, channel, batch).
template <class F> typename F::Epilogue::StrideD out_stride(typename F::Problem const &p)
{
    typename F::Epilogue::StrideD d{};
    constexpr int R = F::Problem::RankT;
    if constexpr (R == 4)
        get<0>(d) = make_stride(p.stride_C[2], p.stride_C[1], p.stride_C[0]);
    else
        get<0>(d) = make_stride(p.stride_C[3], p.stride_C[2], p.stride_C[1], p.stride_C[0]);
    return d;
}

template <class F> tok_status run_fprop(typename F::Problem const &p, const void *act, const void *flt, void *out,
                                        cudaStream_t stream)
{
    const auto d = out_stride<F>(p);
    typename F::Op::Arguments args{p,
                                   {static_cast<Elem const *>(act), static_cast<Elem const *>(flt)},
                                   {{1.0f, 0.0f}, static_cast<Elem const *>(out), d, static_cast<Elem *>(out), d}};
    typename F::Op op;
    if (op.can_implement(args) != cutlass::Status::kSuccess)
        return TOK_ERR_SHAPE;
    if (F::Op::get_workspace_size(args) != 0) // the library allocates nothing
        return TOK_ERR_SHAPE;
    if (op.initialize(args, nullptr, stream) != cutlass::Status::kSuccess) {
        record_cuda_error(cudaGetLastError());
        return TOK_ERR_CUDA;
    }
    if (op.run(stream) != cutlass::Status::kSuccess) {
        record_cuda_error(cudaGetLastError());
        return TOK_ERR_CUDA;
    }
    return launch_status();
}

bool fits_int(int64_t v) { return v >= 0 && v < ((int64_t)1 << 31); }

// Shared argument rules: channels-last bf16 tensors, channel counts multiples of 8
// (16-byte rows for TMA), 16-byte-aligned pointers, 32-bit extents.
tok_status check_conv(const void *x, const void *w, const void *y, int64_t B, int64_t T, int64_t h, int64_t wd,
                      int64_t Cin, int64_t Cout, int64_t taps, int64_t *n_in, int64_t *n_out)
{
    if (B < 0 || T < 0 || h < 0 || wd < 0 || Cin < 8 || Cout < 8 || Cin % 8 || Cout % 8)
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
    if (conv_tc_eligible(Cin, Cout))
        return conv_tc_spatial(x, ws, y, B, T, h, w, Cin, Cout, k, stream);
    const int pad = (int)(k - 1) / 2, kk = (int)k;
    typename Spatial::Problem p(cutlass::conv::Mode::kCrossCorrelation, {(int)(B * T), (int)h, (int)w, (int)Cin},
                                {(int)Cout, kk, kk, (int)Cin}, {pad, pad}, {pad, pad}, {1, 1}, {1, 1}, 1);
    return run_fprop<Spatial>(p, x, ws, y, stream);
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
    if (conv_tc_eligible(Cin, Cout))
        return conv_tc_temporal(x, wt, y, B, T, h, w, Cin, Cout, k, stream);
    typename Temporal::Problem p(cutlass::conv::Mode::kCrossCorrelation,
                                 {(int)B, (int)T, (int)h, (int)w, (int)Cin}, {(int)Cout, (int)k, 1, 1, (int)Cin},
                                 {(int)k - 1, 0, 0}, {0, 0, 0}, {1, 1, 1}, {1, 1, 1}, 1);
    return run_fprop<Temporal>(p, x, wt, y, stream);
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
