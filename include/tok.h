/*
 * tok.h -- C ABI of the B200 Haar patcher and FSQ quantizer library (libtok.so).
 *
 * Four operations of a causal image/video tokenizer's data-parallel path:
 *   tok_haar_fwd    two-level causal full-packet orthonormal Haar patcher
 *   tok_haar_inv    its inverse (the unpatcher)
 *   tok_fsq_encode  1x1 C->6 projection + FSQ bound/round + mixed-radix index
 *   tok_fsq_decode  index -> normalized codes -> 1x1 6->C projection
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers (memory the GPU can address), owned by the
 *     caller; the library allocates nothing and keeps no state between calls.
 *   - Work is enqueued on `stream` (0 = the legacy default stream) and the
 *     call returns without synchronizing.  Results are visible to later work
 *     on the same stream.
 *   - Tensors are dense and row-major with the last index fastest.
 *   - Argument errors are detected on the host and returned before anything
 *     is launched; an empty tensor (a zero extent) returns TOK_OK and touches
 *     no memory (its pointers may then be NULL).  A launch failure returns
 *     TOK_ERR_CUDA; tok_last_cuda_error() gives the CUDA error code.
 *   - Inputs and outputs must not overlap (TOK_ERR_ALIAS).
 *   - Pointers need natural alignment of their element type (TOK_ERR_ALIGN
 *     otherwise).  Every layout gives identical results; the kernel taken
 *     depends on the layout: a 16-byte-aligned source whose rows are whole
 *     16-byte units is loaded tile by tile with tensor copies; other
 *     16-byte-aligned sources row by row with bulk copies; a source that is
 *     not 16-byte aligned takes element-wise GPU kernels.  There is no CPU
 *     path.
 *
 * Sources for the operations (page title, section):
 *   [guide] "NVIDIA Cosmos Tokenizer 完全指南" (a guide to the Cosmos Tokenizer
 *           README): 6.1 and 6.2 (encode API shapes), 7.1 (Haar patching),
 *           7.2 (FSQ), 7.3 (causal time axis).
 *   [card]  "nvidia/Cosmos-Tokenize1-CV8x8x8-720p" model card: Model
 *           Architecture (2-level Haar, x4 in space and time; FSQ).
 *   [notes] "Cosmos World Foundation Model Platform for Physical AI
 *           (Cosmos-Predict1)" notes: model architecture, item 1 (FSQ levels
 *           (8,8,8,5,5,5), vocabulary 64,000).
 */
#ifndef TOK_H
#define TOK_H

#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TOK_ABI_VERSION 1

/* Exported symbols (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define TOK_API __attribute__((visibility("default")))
#else
#define TOK_API
#endif

/* Number of FSQ codes: 8*8*8*5*5*5 ([guide] 7.2, [notes]). */
#define TOK_FSQ_CODEBOOK 64000
/* FSQ channels ([guide] 6.2: codes have 6 channels). */
#define TOK_FSQ_DIM 6

typedef enum {
    TOK_OK = 0,
    TOK_ERR_NULL = 1,  /* a required pointer is NULL */
    TOK_ERR_SHAPE = 2, /* extents violate the operation's shape rule, or overflow */
    TOK_ERR_ALIGN = 3, /* a pointer is not aligned to its element size */
    TOK_ERR_DTYPE = 4, /* unknown tok_dtype */
    TOK_ERR_ALIAS = 5, /* an input buffer overlaps an output buffer */
    TOK_ERR_CUDA = 6,   /* a CUDA call or kernel launch failed; see tok_last_cuda_error() */
    TOK_ERR_TIMEOUT = 7, /* reported by tok_check_device(): a kernel stopped after a bounded wait ran out */
    TOK_ERR_TOO_LARGE = 8 /* the problem (or the device ordinal) exceeds the fixed scratch of
                             tok_fsq_encode_backward_noalloc */
} tok_status;

typedef enum {
    TOK_F32 = 0,  /* IEEE binary32 */
    TOK_BF16 = 1  /* bfloat16: fp32 accumulation inside, one round-to-nearest-even at the store */
} tok_dtype;

/* TOK_ABI_VERSION of the loaded library. */
TOK_API int tok_abi_version(void);

/* Static, NUL-terminated name of a status code. */
TOK_API const char *tok_status_str(tok_status status);

/* cudaError_t of the last call that returned TOK_ERR_CUDA on this thread (0 if none). */
TOK_API int tok_last_cuda_error(void);

/*
 * tok_check_device -- synchronize `stream` and report whether any kernel of
 * this library on the current device gave up a bounded wait since the last
 * check (TOK_ERR_TIMEOUT; that call's output is incomplete), then clear the
 * record.  The TMA-pipelined kernels wait on shared-memory barriers for their
 * copies; a wait that runs out (never expected) ends the kernel instead of
 * hanging the GPU.  Not part of the pages' method: an error channel for the
 * asynchronous calls.  Returns TOK_OK, TOK_ERR_TIMEOUT or TOK_ERR_CUDA.
 */
TOK_API tok_status tok_check_device(cudaStream_t stream);

/*
 * tok_selftest_wait_timeout -- exercise the failure channel that
 * tok_check_device reads.  Launches on `stream` one single-warp kernel whose
 * shared-memory barrier waits for 16 bytes of copy that nothing ever issues;
 * the wait gives up after `polls` polls (1 <= polls <= 2^22, the TMA kernels'
 * own limit; a few thousand end within milliseconds), counts a timeout as the
 * TMA kernels do when a wait runs out, and the kernel returns.  No copy is in
 * flight at any time, so the device stays usable.  The next
 * tok_check_device(stream) returns TOK_ERR_TIMEOUT and clears the count; the
 * one after it returns TOK_OK.  Not part of the pages' method: a test hook for
 * the error channel.  Returns TOK_ERR_SHAPE for `polls` out of range,
 * TOK_ERR_CUDA if the launch fails.
 */
TOK_API tok_status tok_selftest_wait_timeout(uint32_t polls, cudaStream_t stream);

/*
 * tok_haar_fwd -- two-level causal full-packet Haar patcher.
 * [guide] 7.1 (Patcher / Patcher3D, patch_size=4, patch_method="haar"),
 * [guide] 6.1 and 7.3 (t = 1 + (T-1)/4), [card] Model Architecture.
 *
 *   x : [B, C, T, H, W] of `dt`           (input, not modified)
 *   y : [B, 64C, T', H/4, W/4] of `dt`     T' = 1 + (T-1)/4, when T > 1
 *       [B, 16C, 1,  H/4, W/4] of `dt`     when T == 1 (images: no time axis)
 *
 * Each level pairs samples along t, y and x into a low band (a+b)/sqrt(2) and
 * a high band (a-b)/sqrt(2); on video, a copy of frame 0 is put in front of
 * the time axis first.  Level 2 transforms all 8C (2D: 4C) first-level
 * channels.  Output channel (8*s2 + s1)*C + c holds subband s1 of level 1
 * refined by subband s2 of level 2, s = 4*bt + 2*by + bx (bit 1 = high band);
 * on the 2D path (4*s2 + s1)*C + c with s = 2*by + bx.
 * Shape rule: B, C >= 0; T == 1 or T % 4 == 1; H % 4 == 0; W % 4 == 0.
 */
TOK_API tok_status tok_haar_fwd(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C, int64_t T, int64_t H,
                        int64_t W, cudaStream_t stream);

/*
 * tok_haar_inv -- the unpatcher, left inverse of tok_haar_fwd ([guide] 7.1:
 * UnPatcher / UnPatcher3D; [card] Model Architecture: the decoder ends with
 * the inverse wavelet transform).
 *
 *   y : coefficients laid out as tok_haar_fwd writes them (input)
 *   x : [B, C, T, H, W] (output); T, H, W are the pixel-space extents.
 *
 * Level 2 is undone first, then level 1, each with a = (L+H)/sqrt(2),
 * b = (L-H)/sqrt(2); after each level the first reconstructed frame (the
 * replica of frame 0) is dropped.  Same shape rule as tok_haar_fwd.
 */
TOK_API tok_status tok_haar_inv(const void *y, void *x, tok_dtype dt, int64_t B, int64_t C, int64_t T, int64_t H,
                        int64_t W, cudaStream_t stream);

/*
 * tok_haar_fwd_adjoint / tok_haar_inv_adjoint -- the gradients (transposes) of
 * the patcher and of the unpatcher, for training through them.  [guide] 7.1:
 * the patcher replicates frame 0 and pairs samples with the symmetric
 * orthonormal butterfly, so its transpose is the unpatcher's butterflies with
 * the replica's gradient ADDED to frame 0: window 0 gives frame 0 the sum of
 * its four rebuilt frames.  The unpatcher drops the replica, so its transpose
 * feeds window 0 the time samples (0, 0, 0, g_0) and applies the patcher's
 * butterflies.  On images (T == 1) both transforms are orthogonal and the
 * adjoints equal tok_haar_inv and tok_haar_fwd.  The round (straight-through)
 * has no part here: the patcher is linear.
 *
 *   tok_haar_fwd_adjoint: gy (coefficient layout, input) -> gx [B, C, T, H, W]
 *   tok_haar_inv_adjoint: gx [B, C, T, H, W] (input)    -> gy (coefficient layout)
 * Same shape rule, dtypes and errors as tok_haar_fwd.
 */
TOK_API tok_status tok_haar_fwd_adjoint(const void *gy, void *gx, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                        int64_t H, int64_t W, cudaStream_t stream);
TOK_API tok_status tok_haar_inv_adjoint(const void *gx, void *gy, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                        int64_t H, int64_t W, cudaStream_t stream);

/*
 * tok_haar_fwd_windows / tok_haar_inv_windows -- the same transforms restricted
 * to latent frames [t_begin, t_end), 0 <= t_begin <= t_end <= T' (T' = 1 on
 * images).  x and y are the full tensors with the extents above; only latent
 * frames t' in the range are written (forward: y[:, :, t']; inverse: the pixel
 * frames of window t', i.e. frame 0 for t' = 0 and frames 4t'-3 .. 4t'
 * otherwise), and only the pixel frames those windows read are read.  Windows
 * are independent (the causal structure of [guide] 7.1 and 7.3: output frame t'
 * depends on input frames 4t'-3 .. 4t' only, and frame 0 on frame 0 only), so
 * a clip can be transformed chunk by chunk as its frames arrive, and the chunks
 * compose to exactly the full call's result.  An empty range returns TOK_OK;
 * a range outside [0, T'] returns TOK_ERR_SHAPE.  Not on the pages' API: a
 * streaming form of the same operation.
 */
TOK_API tok_status tok_haar_fwd_windows(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                        int64_t H, int64_t W, int64_t t_begin, int64_t t_end, cudaStream_t stream);
TOK_API tok_status tok_haar_inv_windows(const void *y, void *x, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                        int64_t H, int64_t W, int64_t t_begin, int64_t t_end, cudaStream_t stream);

/*
 * tok_haar_fwd_channels_last -- tok_haar_fwd with a channels-last output, the
 * layout a following convolution reads its input channels from:
 *   x : [B, C, T, H, W] as tok_haar_fwd (input)
 *   y : [B, T', H/4, W/4, 64C] (video) or [B, 1, H/4, W/4, 16C] (image), element
 *       [b][t'][i][j][k] = tok_haar_fwd's y[b][k][t'][i][j] (output)
 * Not on the pages' API: a layout of the same result.  Errors as tok_haar_fwd.
 */
TOK_API tok_status tok_haar_fwd_channels_last(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                              int64_t H, int64_t W, cudaStream_t stream);

/*
 * tok_haar_fwd_single / tok_haar_inv_single -- the single-level patcher and
 * unpatcher (patch_size=2: one DWT; [guide] 7.1: one 2D DWT turns c channels into
 * 4c at half size, one 3D DWT into 8c with the first frame repeated for causal
 * alignment).  Same conventions as tok_haar_fwd for one level:
 *   x : [B, C, T, H, W], T == 1 (image) or T odd, H and W even
 *   y : [B, 8C, (T+1)/2, H/2, W/2] (video) or [B, 4C, 1, H/2, W/2] (image)
 * channel s*C + c with subband s = 4*bt + 2*by + bx (2*by + bx on images), bit 1
 * the high band (a - b)/sqrt 2 of an axis; latent frame 0 reads frame 0 twice,
 * frame t' >= 1 reads frames 2t'-1 and 2t'; the inverse keeps the later copy of
 * frame 0.  Two single levels (the second on all 8C channels) equal tok_haar_fwd.
 * Errors as tok_haar_fwd (H, W even instead of multiples of 4; T odd).
 */
TOK_API tok_status tok_haar_fwd_single(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                       int64_t H, int64_t W, cudaStream_t stream);
TOK_API tok_status tok_haar_inv_single(const void *y, void *x, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                       int64_t H, int64_t W, cudaStream_t stream);

/*
 * Clips of any extents ([guide] 6.3: before the network a clip is padded --
 * zeros in space, reflection at the temporal edge -- to aligned extents, and the
 * result is cropped back to the original size afterwards).
 *
 * tok_haar_padded_extents -- the padded extents: Hp, Wp = H, W rounded up to
 * multiples of spatial_multiple; Tp = the smallest T' >= T with
 * (T' - 1) % temporal_multiple == 0 (images, T == 1, stay at 1).  Both
 * multiples must be positive multiples of 4 (4 for the patcher alone; 8 or 16
 * to match a network's total downsampling).  TOK_ERR_SHAPE for invalid
 * arguments, TOK_ERR_NULL for a NULL output pointer.
 */
TOK_API tok_status tok_haar_padded_extents(int64_t T, int64_t H, int64_t W, int64_t spatial_multiple,
                                           int64_t temporal_multiple, int64_t *Tp, int64_t *Hp, int64_t *Wp);

/*
 * tok_haar_fwd_padded -- the patcher on a clip of any extents.
 *   x : [B, C, T, H, W] (input, any T >= 1, H, W >= 0)
 *   y : [B, 64C, 1 + (Tp-1)/4, Hp/4, Wp/4] (T > 1) or [B, 16C, 1, Hp/4, Wp/4]
 *       (T == 1), extents from tok_haar_padded_extents (output)
 * equal to tok_haar_fwd on the padded clip: rows H .. Hp-1 and columns
 * W .. Wp-1 are zero; frames T .. Tp-1 mirror the clip about its last frame
 * (frame T-1+k is frame T-1-k, repeated with period 2(T-1) if the padding is
 * longer than the clip).  The padded clip is never stored: the kernels read
 * zeros and mirrored frames in place.  Errors as tok_haar_fwd (no divisibility
 * rule on T, H, W).
 *
 * tok_haar_inv_cropped -- the unpatcher on the padded extents, keeping the
 * first T frames, H rows and W columns: y as above (input), x [B, C, T, H, W]
 * (output).  The inverse of tok_haar_fwd_padded on its output.
 */
TOK_API tok_status tok_haar_fwd_padded(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                       int64_t H, int64_t W, int64_t spatial_multiple, int64_t temporal_multiple,
                                       cudaStream_t stream);
TOK_API tok_status tok_haar_inv_cropped(const void *y, void *x, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                        int64_t H, int64_t W, int64_t spatial_multiple, int64_t temporal_multiple,
                                        cudaStream_t stream);

/*
 * Streaming chunks of a video ([guide] 6.3: long videos run window by window).
 * Unlike the windowed calls, a chunk call sees only the chunk's own frames, so
 * a long video never has to be resident in device memory at once.
 *
 * tok_haar_fwd_chunk --
 *   first != 0: the start of a video, T = 1 + 4k frames (k >= 0): the patcher
 *     with its frame-0 replicas, always the 3D transform (a one-frame first
 *     chunk gives the video's latent frame 0, not the image transform);
 *     y [B, 64C, 1 + k, H/4, W/4].
 *   first == 0: a continuation, T = 4k frames (k >= 1) that follow earlier
 *     frames; latent frame j reads frames 4j .. 4j+3 of the chunk, no replica;
 *     y [B, 64C, k, H/4, W/4].
 * Chunks of 1 + 4k0, 4k1, 4k2, ... frames give exactly the latent frames of the
 * whole video, in order.  H % 4 == 0, W % 4 == 0; other errors as tok_haar_fwd.
 *
 * tok_haar_inv_chunk -- the inverse of tok_haar_fwd_chunk (T, H, W: the chunk's
 * pixel extents): y as above (input) -> x [B, C, T, H, W] (output).
 */
TOK_API tok_status tok_haar_fwd_chunk(const void *x, void *y, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                      int64_t H, int64_t W, int first, cudaStream_t stream);
TOK_API tok_status tok_haar_inv_chunk(const void *y, void *x, tok_dtype dt, int64_t B, int64_t C, int64_t T,
                                      int64_t H, int64_t W, int first, cudaStream_t stream);

/*
 * The first causal factorized convolution after the patcher ([notes] model
 * architecture item 1: a 1 x k x k spatial convolution, then a k x 1 x 1 temporal
 * convolution padded by k - 1 on the past side only), on the tensor cores:
 * channels-last bf16 activations, bf16 weights, fp32 accumulation, bf16 results.
 * Cross-correlation (no kernel flip), no bias.  Cin (and Cmid, the temporal
 * convolution's input) is a positive multiple of 64; Cout (and Cmid, the spatial
 * convolution's output) is a multiple of 32, at most 256 or a multiple of 256;
 * k <= 15; all pointers are 16-byte aligned device memory.  Errors:
 * TOK_ERR_SHAPE (channels, k, or 32-bit extents), TOK_ERR_NULL, TOK_ERR_ALIGN,
 * TOK_ERR_ALIAS (an input overlaps the output), TOK_ERR_CUDA.  Not on the pages'
 * API: the layer the pages name, with weights the caller provides.
 *
 * tok_conv_spatial -- y[b,t,i,j,n] = sum_{dy,dx,c} ws[n][dy][dx][c] *
 *   x[b, t, i+dy-(k-1)/2, j+dx-(k-1)/2, c], zero outside the frame; k odd.
 *   x [B, T, h, w, Cin], ws [Cout, k, k, Cin], y [B, T, h, w, Cout].
 * tok_conv_temporal_causal -- y[b,t,i,j,n] = sum_{dt,c} wt[n][dt][c] *
 *   x[b, t-(k-1)+dt, i, j, c], zero before frame 0 (output frame t reads frames
 *   t-k+1 .. t).  x [B, T, h, w, Cin], wt [Cout, k, Cin], y [B, T, h, w, Cout].
 * tok_conv_factorized -- tok_conv_spatial into the caller's mid [B, T, h, w, Cmid]
 *   (overwritten), then tok_conv_temporal_causal into y.
 */
TOK_API tok_status tok_conv_spatial(const void *x, const void *ws, void *y, int64_t B, int64_t T, int64_t h,
                                    int64_t w, int64_t Cin, int64_t Cout, int64_t k, cudaStream_t stream);
TOK_API tok_status tok_conv_temporal_causal(const void *x, const void *wt, void *y, int64_t B, int64_t T, int64_t h,
                                            int64_t w, int64_t Cin, int64_t Cout, int64_t k, cudaStream_t stream);
TOK_API tok_status tok_conv_factorized(const void *x, const void *ws, const void *wt, void *mid, void *y, int64_t B,
                                       int64_t T, int64_t h, int64_t w, int64_t Cin, int64_t Cmid, int64_t Cout,
                                       int64_t k, cudaStream_t stream);

/*
 * The patcher fused into the spatial convolution after it (k = 3), one kernel:
 * [notes] model architecture item 1 (the 1 x k x k convolution right after the
 * 2-level Haar transform) on the coefficients of [guide] 7.1 (Patcher3D, two
 * levels, channel (8*s2 + s1)*C + c).  The coefficients are made in shared
 * memory as the tensor cores' operand (the patcher's own bf16 values) and never
 * reach HBM.
 *
 * tok_patch_embed_pack_weights -- reorder the spatial filter for the fused call:
 *   ws : [Cmid, 3, 3, 64C] bf16, the layout of tok_conv_spatial (input)
 *   wp : [Cmid, 9C, 64] bf16, wp[n][(c*3 + dx)*3 + dy][g] = ws[n][dy][dx][g*C + c]
 *        (output, caller-owned, 1152*C*Cmid bytes; 16-byte aligned)
 *   Run once per filter; the fused call reads wp.  Shape rule as below.
 *
 * tok_patch_embed_spatial -- y = tok_conv_spatial(channels-last patcher(x), ws)
 *   with k = 3 ('same' zero padding in space):
 *   x  : [B, C, T, H, W] bf16 pixels, video (T = 1 + 4k, T >= 5), H % 4 == 0,
 *        W % 8 == 0 (input)
 *   wp : the packed filter above (input)
 *   y  : [B, T', H/4, W/4, Cmid] bf16, T' = 1 + (T-1)/4 (output)
 *   Shape rule: 1 <= C <= 8; Cmid a multiple of 32, at most 256 or a multiple
 *   of 256; 32-bit element counts.  Pointers 16-byte aligned (TOK_ERR_ALIGN);
 *   y must not overlap x or wp (TOK_ERR_ALIAS).  fp32 accumulation, one bf16
 *   rounding.  Not on the pages' API: the layer the pages name, with weights
 *   the caller provides.
 */
TOK_API tok_status tok_patch_embed_pack_weights(const void *ws, void *wp, int64_t C, int64_t Cmid,
                                                cudaStream_t stream);
TOK_API tok_status tok_patch_embed_spatial(const void *x, const void *wp, void *y, int64_t B, int64_t C, int64_t T,
                                           int64_t H, int64_t W, int64_t Cmid, cudaStream_t stream);

/*
 * tok_fsq_encode -- fused 1x1 projection + FSQ quantization + index pack.
 * [guide] 7.2 (bound with tanh, rounding, levels [8,8,8,5,5,5], implicit
 * codebook of 64000, mixed-radix codes_to_indices), [guide] 6.2 (indices
 * [B,t,h,w], codes [B,6,t,h,w]), [notes] model architecture item 1.
 *
 *   u     : [B, C, S] fp32 latent, S = t*h*w token positions (input)
 *   w     : [6, C] fp32 projection, row-major (input, device memory)
 *   idx   : [B, S] int32 indices in [0, 64000) (output)
 *   codes : [B, 6, S] fp32 normalized codes q_i / floor(L_i/2), or NULL
 *
 * z_i = sum_c w[i][c] * u[c] is evaluated in fp32 as a chain of fused
 * multiply-adds over c = 0..C-1 from 0.  Channel i (L levels) is quantized to
 * q = round(tanh(z + shift)*half - off), half = (L-1)(1+1e-3)/2, off = 0.5
 * for even L else 0, shift = atanh(off/half); the digit q + floor(L/2) of
 * channel i has place value (1, 8, 64, 512, 2560, 12800)[i].  The kernel
 * compares z against the exact fp32 decision thresholds of that function.
 * Shape rule: B, S >= 0; 1 <= C <= 1024.
 */
TOK_API tok_status tok_fsq_encode(const float *u, const float *w, int32_t *idx, float *codes, int64_t B, int64_t C,
                          int64_t S, cudaStream_t stream);

/*
 * tok_fsq_decode -- index unpack (indices_to_codes, [guide] 7.2) + 1x1 6->C
 * projection with the transposed encode weight.
 *
 *   idx       : [B, S] int32 (input)
 *   w         : [6, C] fp32 (input; the same matrix tok_fsq_encode takes)
 *   out       : [B, C, S] fp32, out[c] = sum_i w[i][c] * zhat_i (output)
 *   bad_count : device int32 counter or NULL.  Each index outside [0, 64000)
 *               adds 1 (atomically) and its token's C outputs are NaN.
 *               The caller zeroes it; the library only adds to it.
 * Shape rule: B, S >= 0; 1 <= C <= 1024.
 */
TOK_API tok_status tok_fsq_decode(const int32_t *idx, const float *w, float *out, int32_t *bad_count, int64_t B,
                          int64_t C, int64_t S, cudaStream_t stream);

/*
 * FSQ backward (training).  [guide] 7.2: the bound uses tanh and round_ste
 * keeps a straight-through gradient -- the rounding passes the gradient
 * unchanged -- so d zhat_i / d z_i = half_i * sech^2(z_i + shift_i) / floor(L_i/2)
 * with the constants of tok_fsq_encode.  The weight gradient is a sum over all
 * tokens; it is reduced deterministically (a fixed partition of the tokens and a
 * fixed summation order, independent of the device) through a caller-provided
 * workspace of tok_fsq_backward_workspace_size() bytes, 4-byte-aligned device
 * memory that the call overwrites (nothing in it needs to be initialized).
 * grad_w is overwritten, not accumulated.  1 <= C <= 16.
 */

/* Workspace bytes for a backward call on [B, C, S]; -1 for an invalid shape. */
TOK_API int64_t tok_fsq_backward_workspace_size(int64_t B, int64_t C, int64_t S);

/*
 * tok_fsq_encode_backward -- gradients of tok_fsq_encode's codes output.
 *   u          : [B, C, S] fp32, the forward's latent (input)
 *   w          : [6, C] fp32 (input)
 *   grad_codes : [B, 6, S] fp32, gradient of the normalized codes (input)
 *   grad_u     : [B, C, S] fp32, sum_i w[i][c] * t_i (output)
 *   grad_w     : [6, C] fp32, sum over tokens of t_i * u[c] (output)
 * with t_i = grad_codes_i * d zhat_i / d z_i and z the forward's fp32 chain.
 * Errors: as tok_fsq_encode, plus TOK_ERR_SHAPE for C > 16 or a workspace that
 * is too small, TOK_ERR_ALIAS if any buffer overlaps an output or the workspace.
 */
TOK_API tok_status tok_fsq_encode_backward(const float *u, const float *w, const float *grad_codes, float *grad_u,
                                           float *grad_w, void *workspace, int64_t workspace_bytes, int64_t B,
                                           int64_t C, int64_t S, cudaStream_t stream);

/*
 * tok_fsq_encode_backward_noalloc -- tok_fsq_encode_backward without a
 * workspace argument, for callers that cannot allocate device memory when they
 * need the gradient: a host framework that owns every device allocation and
 * hands its plugins only inputs and outputs, a service that fixes its memory
 * at start-up and must not call cudaMalloc (which may synchronize the device)
 * while it serves, an embedded pipeline without an allocator.  The pages have
 * no counterpart: it is a deployment form of the same computation.
 *
 * The workspace is a fixed array compiled into the library (3 MB, held by
 * every GPU that loads the library until the process exits), so:
 *   - the workspace tok_fsq_backward_workspace_size(B, C, S) reports must fit
 *     in 3 MB: at most 8,388,608 tokens (B * S) at C = 16 when S is a multiple
 *     of 128 (each batch row's last 128-token tile counts whole; smaller C
 *     allows more); larger calls return TOK_ERR_TOO_LARGE before anything runs;
 *   - every call uses the same array: calls that may overlap on the GPU
 *     (concurrent streams, other host threads) race and must be serialized by
 *     the caller; a call overwrites whatever an earlier call left there;
 *   - the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) and caches it for the life of the process; make
 *     that first call before any stream capture, and do not reset the device
 *     (cudaDeviceReset) between calls: a reset invalidates the cached address;
 *   - the cache covers device ordinals 0 to 63: a call on a higher ordinal
 *     returns TOK_ERR_TOO_LARGE before anything runs.
 * It allocates nothing.  Arguments, outputs and results are those of
 * tok_fsq_encode_backward.
 */
TOK_API tok_status tok_fsq_encode_backward_noalloc(const float *u, const float *w, const float *grad_codes,
                                                   float *grad_u, float *grad_w, int64_t B, int64_t C, int64_t S,
                                                   cudaStream_t stream);

/*
 * tok_fsq_decode_backward -- gradients of tok_fsq_decode.
 *   idx        : [B, S] int32 (input)
 *   w          : [6, C] fp32 (input)
 *   grad_out   : [B, C, S] fp32, gradient of the decoded latent (input)
 *   grad_codes : [B, 6, S] fp32, sum_c w[i][c] * grad_out[c]; 0 for invalid indices (output)
 *   grad_w     : [6, C] fp32, sum over tokens of zhat_i * grad_out[c] (output)
 * Errors: as tok_fsq_encode_backward.
 */
TOK_API tok_status tok_fsq_decode_backward(const int32_t *idx, const float *w, const float *grad_out,
                                           float *grad_codes, float *grad_w, void *workspace,
                                           int64_t workspace_bytes, int64_t B, int64_t C, int64_t S,
                                           cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TOK_H */
