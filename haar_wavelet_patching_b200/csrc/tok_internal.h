// Declarations shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "tok.h"

namespace tok {

// Extents of one Haar call: pixels [B, C, T, H, W], coefficients [B, G*C, Tq, h, w];
// the call processes latent frames [tq0, tq0 + nq).
// Extended form (ext): the pixel tensor may be smaller than the 4h x 4w blocks (the
// forward pads with zeros, the inverse crops), a window tq that is not the frame-0
// replica window reads frames 4*tq + fbase .. + 3 (mirrored past frame T - 1), and
// window 0 is the replica window iff rep.  video: 3D transform (else the 2D path).
struct HaarDims {
    int64_t B, C, T, H, W;
    int64_t Tq, h, w;
    int64_t tq0, nq;
    int64_t fbase = -3;
    int rep = 1;
    bool video = true;
    bool ext = false;
};

// Which form of the TMA kernel takes a planar call in direction fwd: boxes (the source's
// rows are whole 16-byte units, and so are the destination's where it stores 16-byte rows),
// boxes_any_store (inverse: box loads, pixel-row stores of run-time width), groups (bf16
// video forward with W % 8 == 4 and an odd w: tensor boxes over pairs of pixel rows, tiles
// shifted so that coefficient pairs are stored aligned), rows (any 16-byte-aligned source,
// any row length, any element-aligned destination) or none (register kernels).
enum class HaarTmaForm { none, boxes, boxes_any_store, groups, rows };
HaarTmaForm haar_tma_form(bool fwd, const void *in, const void *out, tok_dtype dt, const HaarDims &d);
// fwd: pixels -> coefficients; adj: the adjoint variant (video only; images are orthogonal).
tok_status haar_tma_launch(bool fwd, bool adj, HaarTmaForm form, const void *in, void *out, tok_dtype dt,
                           const HaarDims &d, cudaStream_t stream);

// Single-level patcher / unpatcher (patch_size=2): pixels [B, C, T, H, W] <->
// coefficients [B, G*C, Tq, h, w] with G = 8 (video), 4 (images), Tq = (T + 1) / 2, h = H/2.
HaarTmaForm haar_single_tma_form(bool fwd, const void *in, const void *out, tok_dtype dt, const HaarDims &d);
tok_status haar_single_tma_launch(bool fwd, HaarTmaForm form, const void *in, void *out, tok_dtype dt,
                                  const HaarDims &d, cudaStream_t stream);

// Channels-last two-level patcher: pixels [B, C, T, H, W] -> [B, Tq, h, w, G*C] (1 <= C <= 4).
bool haar_cl_tma_eligible(const void *in, const void *out, tok_dtype dt, const HaarDims &d);
tok_status haar_cl_tma_launch(const void *in, void *out, tok_dtype dt, const HaarDims &d, cudaStream_t stream);

// Hand-written tensor-core convolutions (conv_tc.cu): eligible for Cin % 64 == 0 and
// Cout % 32 == 0 (Cout <= 256, or a multiple of 256); arguments checked by the caller.
bool conv_tc_eligible(int64_t Cin, int64_t Cout);
tok_status conv_tc_temporal(const void *x, const void *wt, void *y, int64_t B, int64_t T, int64_t h, int64_t w,
                            int64_t Cin, int64_t Cout, int64_t k, cudaStream_t stream);
tok_status conv_tc_spatial(const void *x, const void *ws, void *y, int64_t B, int64_t T, int64_t h, int64_t w,
                           int64_t Cin, int64_t Cout, int64_t k, cudaStream_t stream);

// Synchronize `stream`, return in *count the barrier-wait timeouts of this device's
// Haar (resp. FSQ, FSQ backward) kernels since the last call, and clear them.
tok_status read_and_clear_haar_timeouts(cudaStream_t stream, unsigned int *count);
tok_status read_and_clear_fsq_timeouts(cudaStream_t stream, unsigned int *count);
tok_status read_and_clear_fsq_bwd_timeouts(cudaStream_t stream, unsigned int *count);
tok_status read_and_clear_conv_timeouts(cudaStream_t stream, unsigned int *count);

// Remembers a CUDA error for tok_last_cuda_error().
void record_cuda_error(cudaError_t e);

} // namespace tok
