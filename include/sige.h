/*
 * sige.h -- C ABI of the B200 spatially sparse incremental convolution.
 *
 * The method (SIGE, "Efficient Spatially Sparse Inference for Conditional
 * GANs and Diffusion Models"): the activations of the original image are
 * computed once and cached; for an edited image the engine compares the
 * original and edited inputs to get a difference mask (mer.dev notes on SIGE,
 * section 3 "Method"), downsamples that mask to each scale, dilates it and
 * selects tiles (section 3.2 "Sparse Engine SIGE"), reduces it to active-block
 * indices, gathers the active blocks with their halo from the edited
 * activation, stacks them on the batch axis, runs the layer F_l on the stack
 * and scatters the output blocks back into the cached F_l(A_original)
 * (SIGE project page, "Overview").
 *
 * Conventions for every call
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates no device memory and keeps no state between calls.
 *   - Every call is asynchronous on `stream` (NULL = legacy default stream),
 *     launches exactly one kernel, and returns after enqueueing it.  Only
 *     sige_get_error() / sige_get_device_error() synchronise, and
 *     sige_reduce_mask / sige_reduce_mask_px when the caller asks for the
 *     counts on the host.
 *   - Host-side checks run before any launch: invalid arguments return
 *     SIGE_ERR_INVALID_ARG, shapes the kernels do not cover return
 *     SIGE_ERR_UNSUPPORTED, a failed launch returns SIGE_ERR_CUDA.  Nothing
 *     is enqueued in those cases.
 *   - Errors found on the device (an index list longer than its capacity, a
 *     bounded wait that expired) never trap: the kernel records the first one
 *     in the 256-byte header at the start of the call's workspace and finishes
 *     without touching memory it cannot vouch for.  sige_get_error() reads and
 *     clears that record.
 *   - Activations are NHWC.  Conv weights are [C_out][k][k][C_in] (KRSC) in
 *     the activation dtype.  Biases and GroupNorm scale/shift are float32.
 *   - Tile lists are int32 pairs (h0, w0): the output-pixel origin of each
 *     active b x b tile, in row-major tile order.  Counts live on the device,
 *     so no call needs the host to know how many tiles are active.
 */
#ifndef SIGE_H
#define SIGE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same handle as cudaStream_t. */
typedef struct CUstream_st *sige_stream_t;

typedef enum {
    SIGE_OK = 0,
    SIGE_ERR_INVALID_ARG = -1,   /* NULL pointer, bad size, inconsistent descriptors */
    SIGE_ERR_UNSUPPORTED = -2,   /* valid but not covered by the kernels (dtype, layout, C % 8) */
    SIGE_ERR_CUDA = -3,          /* no device, launch or runtime failure */
    SIGE_ERR_CAPACITY = -4,      /* device: more active tiles than the list capacity */
    SIGE_ERR_TIMEOUT = -5,       /* device: a bounded wait expired */
    SIGE_ERR_WORKSPACE = -6      /* workspace missing or smaller than required */
} sige_status;

typedef enum { SIGE_U8 = 0, SIGE_F32 = 1, SIGE_BF16 = 2 } sige_dtype;
typedef enum { SIGE_NHWC = 0, SIGE_NCHW = 1 } sige_layout;

/* A dense activation tensor.  `layout` NCHW is accepted only by
 * sige_reduce_mask (images such as 3 x H x W uint8). */
typedef struct {
    int32_t n, h, w, c;
    int32_t dtype;   /* sige_dtype */
    int32_t layout;  /* sige_layout */
} sige_tensor_desc;

/* One convolution layer F_l.  Output size Ho = (H + 2 pad - kernel)/stride + 1.
 * `block` is the output tile edge b; each gathered input block is
 * b_in = (b - 1) * stride + kernel pixels wide, so neighbouring blocks of a
 * 3x3 stride-1 conv overlap by 2 pixels (SIGE project page, "Overview").
 * Kernels and tiles are square (one `kernel`, one `block`): every layer of the
 * workloads this library serves is, and the pages describe square blocks
 * only; a k_h x k_w kernel or a b_h x b_w tile has no field here. */
typedef struct {
    int32_t kernel, stride, pad;
    int32_t c_in, c_out;
    int32_t block;
} sige_conv_desc;

/* One scale of the mask reduction: the grid (h, w) the mask is downsampled
 * to, the tile edge at that scale and the capacity (pairs) of its list. */
typedef struct {
    int32_t h, w, block, capacity;
} sige_scale_desc;

#define SIGE_MAX_SCALES 8
#define SIGE_WORKSPACE_HEADER_BYTES 256

/* Which call a workspace is sized for (sige_workspace_bytes). */
typedef enum {
    SIGE_CALL_REDUCE_MASK = 0,
    SIGE_CALL_SPARSE_CONV = 1,
    SIGE_CALL_CONV_FUSED = 2,
    SIGE_CALL_DENSE_CONV = 3,
    SIGE_CALL_RESBLOCK = 4
} sige_call;

/* ------------------------------------------------------------------ calls */

/* (1) Difference mask -> per-scale active-tile lists.
 * mer.dev notes on SIGE, section 3 "Method" (difference mask between the
 * original and edited inputs) and section 3.2 "Sparse Engine SIGE" (downsample
 * to several scales, dilate, select tiles); SIGE project page, "Overview"
 * (reduce the mask to active block indices).
 *
 * Pixel (y, x) is edited when, for some batch item, max_c |a_edit - a_orig| >
 * threshold, the difference taken in float32.  For scale s the mask is
 * OR-downsampled to (scales[s].h, scales[s].w) (in->h, in->w must be integer
 * multiples of them), dilated by `dilate` tiles of scales[s].block pixels,
 * cut into block x block tiles anchored at (0, 0) and clipped at the border;
 * every tile holding a set pixel is listed.
 *   a_orig, a_edit : device, `in` shape/dtype/layout (u8, f32 or bf16; NHWC or NCHW)
 *   idx            : device int32 pairs; scale s's list starts at pair offset
 *                    sum_{t<s} scales[t].capacity, row-major tile order
 *   counts         : device int32[n_scales], the number of active tiles (may
 *                    exceed the capacity: then only `capacity` pairs are written
 *                    and the device error SIGE_ERR_CAPACITY is recorded)
 *   host_counts    : host int32[n_scales] or NULL.  When given, the counts are
 *                    also copied there and the call synchronises `stream`
 *                    before it returns (an opt-in: the rest of the path reads
 *                    the counts on the device).  Refused with
 *                    SIGE_ERR_INVALID_ARG while `stream` is being captured.
 *   workspace      : device, >= sige_reduce_mask_workspace_bytes(), zero-filled
 *                    before its first use; each call leaves it zero-filled
 *                    apart from a recorded device error.  One workspace per
 *                    stream: calls sharing one must not overlap on the GPU.
 * One CTA of the launch waits (bounded, about 4 s) for the others to finish
 * comparing; past the bound the device error SIGE_ERR_TIMEOUT is recorded, no
 * list or count is written, and the workspace must be zero-filled again
 * before its next use. */
size_t sige_reduce_mask_workspace_bytes(const sige_tensor_desc *in, int32_t n_scales,
                                        const sige_scale_desc *scales);
int sige_reduce_mask(const void *a_orig, const void *a_edit, const sige_tensor_desc *in,
                     float threshold, int32_t dilate, int32_t n_scales,
                     const sige_scale_desc *scales, int32_t *idx, int32_t *counts,
                     int32_t *host_counts, void *workspace, size_t workspace_bytes,
                     sige_stream_t stream);

/* (1c) sige_reduce_mask with the dilation in pixels instead of tiles.
 * mer.dev notes on SIGE, section 3.2 "Sparse Engine SIGE": the mask is dilated
 * before the tiles are selected; the dilation only has to cover the layers'
 * receptive-field growth.  Per scale the OR-downsampled mask is dilated by a
 * square of `radius` pixels at that scale (clipped at the border) and every
 * b x b tile holding a set pixel is listed; no tile dilation follows.  With
 * radius = the layers' total halo (1 for one 3x3 conv, 2 for two chained ones)
 * the sparse result still equals the dense one of the edited input, on fewer
 * tiles than a one-tile dilation.  Arguments, layout, workspace and errors as
 * sige_reduce_mask; radius >= 0 (0: tiles of the raw downsampled mask). */
int sige_reduce_mask_px(const void *a_orig, const void *a_edit, const sige_tensor_desc *in,
                        float threshold, int32_t radius, int32_t n_scales,
                        const sige_scale_desc *scales, int32_t *idx, int32_t *counts,
                        int32_t *host_counts, void *workspace, size_t workspace_bytes,
                        sige_stream_t stream);

/* (1b) sige_reduce_mask without a caller workspace.  There is no counterpart
 * in the paper: this is a convenience for callers that cannot allocate device
 * memory for a workspace (a process that reserves all device memory up front,
 * a plugin interface without an allocator, a binding that only forwards the
 * tensors it was given).  The scratch lives in a 64 KB array inside the
 * library, one per GPU, held until the process exits:
 *   - requests needing more than that (256-byte header + one flag byte per
 *     tile, 16-byte padded per scale) return SIGE_ERR_WORKSPACE, nothing
 *     enqueued;
 *   - the first call on a device looks the array's address up (once, with
 *     that device current), so make that first call before any stream
 *     capture; the address is kept for the life of the process and does not
 *     survive a cudaDeviceReset of that device;
 *   - each call clears the part of the array it uses and sets counts[] to -1
 *     with two asynchronous memsets on `stream` (not kernels: they are not
 *     counted by sige_launch_count), then runs the same kernel as
 *     sige_reduce_mask;
 *   - all calls share the array: calls that overlap on the GPU (other
 *     streams, other threads) race and must be serialised by the caller;
 *   - there is no workspace header to read with sige_get_error: a list
 *     longer than its capacity shows as counts[s] > capacity, and a call that
 *     did not complete on the device (a bounded wait that expired) leaves
 *     counts[s] < 0;
 *   - every argument is checked before anything is enqueued.
 * Other arguments as in sige_reduce_mask. */
int sige_reduce_mask_static(const void *a_orig, const void *a_edit, const sige_tensor_desc *in,
                            float threshold, int32_t dilate, int32_t n_scales,
                            const sige_scale_desc *scales, int32_t *idx, int32_t *counts,
                            sige_stream_t stream);

/* (2) Gather the active blocks, with halo, from the edited activation and
 * stack them on the batch axis (SIGE project page, "Overview").
 *   blocks[t][n][hh][ww][c] = T(x[n][h0*s - p + hh][w0*s - p + ww][c]),
 *   hh, ww < b_in, zero outside the image (the conv's zero padding), with
 *   T(v) = v, or v*gn_scale[n][c] + gn_shift[n][c] when gn_scale != NULL,
 *   followed by SiLU v/(1+exp(-v)) when silu != 0; computed in float32 and
 *   stored in x's dtype.
 *   x        : device, NHWC f32 or bf16, xd->c == cd->c_in, C % 8 == 0 for bf16, % 4 for f32
 *   idx/count: the list of one scale from sige_reduce_mask; min(*count, capacity) tiles
 *   gn_scale, gn_shift : device float32 [N][C_in] or both NULL
 *   blocks   : device, [capacity][N][b_in][b_in][C_in] in x's dtype; entries
 *              past the count are left untouched. */
int sige_gather(const void *x, const sige_tensor_desc *xd, const sige_conv_desc *cd,
                const int32_t *idx, const int32_t *count, int32_t capacity,
                const float *gn_scale, const float *gn_shift, int32_t silu, void *blocks,
                sige_stream_t stream);

/* (3) Run the layer F_l on the stacked blocks: a valid convolution of each
 * block, no bias (SIGE project page, "Overview").
 *   out[t][n][i][j][o] = sum_{r,c,ci} W[o][r][c][ci] * blocks[t][n][i*s+r][j*s+c][ci]
 *   blocks     : device, [capacity][batch][b_in][b_in][C_in] in `dtype` (f32 or bf16)
 *   weight     : device, [C_out][k][k][C_in] in `dtype`
 *   out_blocks : device float32 [capacity][batch][b][b][C_out]
 *   workspace  : device, >= sige_conv_workspace_bytes(), zero-filled before
 *                first use and left zero-filled (split-K partial sums).
 * bf16 runs on the tensor cores (bf16 operands, float32 accumulation);
 * f32 runs on the CUDA cores in float32. */
int sige_sparse_conv(const void *blocks, const sige_conv_desc *cd, int32_t dtype, int32_t batch,
                     const void *weight, const int32_t *count, int32_t capacity, float *out_blocks,
                     void *workspace, size_t workspace_bytes, sige_stream_t stream);

/* (4) Scatter the output blocks into the cached output, in place (SIGE
 * project page, "Overview": scatter back into F_l(A_original)).
 *   y[n][h0+i][w0+j][o] = round(out[t][n][i][j][o] + bias[o] + residual[n][h0+i][w0+j][o])
 * for every in-image pixel of the listed tiles, rounded once to y's dtype
 * (ties to even).  Every other byte of y is left untouched.
 *   bias     : device float32 [C_out] or NULL
 *   residual : device, same shape/dtype as y, or NULL
 *   y        : device NHWC f32 or bf16 holding F_l(A_original) on entry */
int sige_scatter(const float *out_blocks, const sige_conv_desc *cd, const int32_t *idx,
                 const int32_t *count, int32_t capacity, const float *bias, const void *residual,
                 void *y, const sige_tensor_desc *yd, sige_stream_t stream);

/* (5) Gather (+GroupNorm affine +SiLU), conv and scatter (+bias +residual) of
 * one layer in a single launch; the result equals (2) -> (3) -> (4) without
 * the stacked blocks or output blocks ever reaching memory.  Arguments as in
 * those calls. */
int sige_conv_fused(const void *x, const sige_tensor_desc *xd, const void *weight,
                    const float *bias, const sige_conv_desc *cd, const int32_t *idx,
                    const int32_t *count, int32_t capacity, const float *gn_scale,
                    const float *gn_shift, int32_t silu, const void *residual, void *y,
                    const sige_tensor_desc *yd, void *workspace, size_t workspace_bytes,
                    sige_stream_t stream);

/* (6) The residual block of a diffusion UNet on the active tiles, in one
 * launch: two chained layers F_l run on the gathered active blocks, each
 * updating its cached output (SIGE project page, "Overview"; mer.dev notes on
 * SIGE, section 3 "Method": cached activations reused outside the edit):
 *   y1  = conv3x3(SiLU(x * gn1_scale + gn1_shift), w1) + b1        -> cached y1
 *   out = conv3x3(SiLU(y1 * gn2_scale + gn2_shift), w2) + b2 + x   -> cached out
 * on every in-image pixel of the first min(*count, capacity) tiles of `idx`
 * (8 x 8, stride 1, zero padding); y1 is rounded to bf16 before GroupNorm2, as
 * if stored; every other byte of y1 and out is left untouched.  conv2 reads y1
 * on the tile plus a one-pixel ring, which this call recomputes from x
 * instead of reading the cache (y1 never goes through memory on its way to
 * conv2), so the result equals sige_conv_fused for conv1 followed by
 * sige_conv_fused for conv2 on the same list whenever x differs from the
 * input the caches were computed from only at pixels whose 3 x 3 window lies
 * in listed tiles -- true for any list from sige_reduce_mask with dilate >= 1
 * (or sige_reduce_mask_px with radius >= 1) whose threshold catches every
 * change.
 *   x_edit              : device NHWC bf16 [N][H][W][128] (xd), the edited input
 *   w1, w2              : device bf16 [128][3][3][128] (KRSC)
 *   b1, b2              : device float32 [128] or NULL (no bias)
 *   gn1_scale/shift,
 *   gn2_scale/shift     : device float32 [N][128], GroupNorm folded into an
 *                         affine (sige_groupnorm_affine of the cached x and y1)
 *   block               : 8 (the tile edge; others return SIGE_ERR_UNSUPPORTED)
 *   idx, count, capacity: the tile list (as sige_conv_fused)
 *   y1, out             : device NHWC bf16, shape of x, holding the caches on
 *                         entry; must not overlap x or each other
 *   workspace           : device, >= SIGE_WORKSPACE_HEADER_BYTES (the device
 *                         error word; see sige_get_device_error), 16-byte
 *                         aligned
 * Runs on the tensor cores in clusters of two CTAs; asynchronous on `stream`,
 * one launch, nothing allocated.  Errors: SIGE_ERR_INVALID_ARG (NULL or
 * misaligned list, overlapping buffers), SIGE_ERR_UNSUPPORTED (not bf16 NHWC
 * with 128 channels and 8 x 8 tiles, misaligned tensors), SIGE_ERR_WORKSPACE,
 * SIGE_ERR_CUDA; on the device a bounded wait that expires records
 * SIGE_ERR_TIMEOUT. */
int sige_resblock_fused(const void *x_edit, const sige_tensor_desc *xd, const void *w1, const float *b1,
                        const float *gn1_scale, const float *gn1_shift, const void *w2, const float *b2,
                        const float *gn2_scale, const float *gn2_shift, int32_t block, const int32_t *idx,
                        const int32_t *count, int32_t capacity, void *y1, void *out, void *workspace,
                        size_t workspace_bytes, sige_stream_t stream);

/* Options of the GauGAN-style layers (sige_conv_fused_ext). */
typedef struct {
    int32_t transposed;       /* 1: a transposed conv (learned upsampling): input pixel (i, j) feeds
                                 output pixel (i*stride - pad + r, j*stride - pad + c) through
                                 weight[o][r][c][ci] */
    int32_t output_padding;   /* transposed only: extra output rows / columns (< stride); 0 otherwise */
    const void *spade_gamma;  /* NULL, or device NHWC map of x's shape and dtype */
    const void *spade_beta;   /* NULL (zero), or a map like spade_gamma; needs spade_gamma */
    int32_t act;              /* after the input transform: 0 none, 1 SiLU, 2 LeakyReLU(0.2) */
} sige_layer_ext;

/* (5b) sige_conv_fused for the other layer types of a GauGAN-style generator
 * (mer.dev notes on SIGE, section 5: the engine serves GauGAN's generator as
 * well as diffusion UNets): transposed convs and SPADE-style spatially
 * modulated normalisation.  The conv input is
 *   t = act((x * gn_scale[n][c] + gn_shift[n][c]) * (1 + gamma[n][y][x][c]) + beta[n][y][x][c])
 * (each factor only when given), rounded to bf16; the layer is the conv of
 * `cd` or, with ext->transposed, the transposed conv of kernel, stride and
 * pad of `cd`, output Ho = (H - 1)*stride - 2*pad + kernel + output_padding;
 * + bias (+ residual of y's shape), rounded once into y at every in-image
 * pixel of the listed tiles (tiles at the OUTPUT resolution, origins in
 * output pixels).  idx == NULL: every tile of the output grid (the dense
 * layer: the cache of the original, or the dense baseline; count and
 * capacity ignored).  Runs on the tensor cores: bf16 NHWC, C_in a multiple of
 * 64; other shapes return SIGE_ERR_UNSUPPORTED.  Arguments otherwise as
 * sige_conv_fused; the workspace is sized by sige_conv_workspace_bytes of the
 * same cd. */
int sige_conv_fused_ext(const void *x, const sige_tensor_desc *xd, const void *weight, const float *bias,
                        const sige_conv_desc *cd, const sige_layer_ext *ext, const int32_t *idx,
                        const int32_t *count, int32_t capacity, const float *gn_scale, const float *gn_shift,
                        const void *residual, void *y, const sige_tensor_desc *yd, void *workspace,
                        size_t workspace_bytes, sige_stream_t stream);

/* (6b) The whole step of an edit for one residual block, in ONE launch: the
 * difference mask of x_orig vs x_edit, its 8 x 8 tiles dilated by `dilate`
 * tiles and compacted in row-major order (as sige_reduce_mask with one
 * scale at full resolution), then sige_resblock_fused on that list (mer.dev
 * notes on SIGE, sections 3 and 3.2; SIGE project page, "Overview").  Every
 * CTA of the launch streams its share of the two inputs and marks tile
 * flags; after a grid-wide barrier each CTA derives the list itself, so no
 * second launch and no host round trip separate the mask from the convs.
 *   x_orig, x_edit : device NHWC bf16 [N][H][W][128] (xd); the mask is
 *                    OR-ed over the batch
 *   threshold      : a pixel is edited when some channel differs by more
 *                    (strict >), the difference taken in float32
 *   idx, count     : OUTPUTS: the list (int32 pairs, capacity entries) and
 *                    its length (which may exceed capacity: then only
 *                    capacity tiles are listed and processed, and the device
 *                    error SIGE_ERR_CAPACITY is recorded)
 *   workspace      : device, >= sige_resblock_step_workspace_bytes(xd, block),
 *                    zero-filled before its first use and not written by the
 *                    caller afterwards: the header holds the error word, a
 *                    grid-barrier counter that only grows (the call's
 *                    generation) and a counter that hands out the chunks of
 *                    the difference stream (it also only grows, by a fixed
 *                    amount per call), and each tile flag holds the
 *                    generation of the call that last set it, so no call has
 *                    to clear anything for the next.  After a call that
 *                    recorded SIGE_ERR_TIMEOUT, zero the workspace again.
 *                    One workspace per device and stream: calls sharing one
 *                    must not overlap.
 * Other arguments as sige_resblock_fused.  The launch keeps every CTA
 * resident at once (one pair of CTAs per two SMs); if other work holds SMs so
 * that some CTAs cannot start, the grid barrier's bounded wait (about 1 s)
 * expires and records SIGE_ERR_TIMEOUT instead of hanging.  At most 64 units
 * (tiles x batch) per CTA pair: larger capacities return
 * SIGE_ERR_UNSUPPORTED, as do tile grids beyond 16384 tiles. */
size_t sige_resblock_step_workspace_bytes(const sige_tensor_desc *xd, int32_t block);
int sige_resblock_step(const void *x_orig, const void *x_edit, const sige_tensor_desc *xd, float threshold,
                       int32_t dilate, const void *w1, const float *b1, const float *gn1_scale,
                       const float *gn1_shift, const void *w2, const float *b2, const float *gn2_scale,
                       const float *gn2_shift, int32_t block, int32_t *idx, int32_t *count, int32_t capacity,
                       void *y1, void *out, void *workspace, size_t workspace_bytes, sige_stream_t stream);

/* The same layer on every tile of the output: the dense conv that fills the
 * cache F_l(A_original) and the dense baseline the sparse path is compared
 * with.  y is fully written. */
int sige_dense_conv(const void *x, const sige_tensor_desc *xd, const void *weight,
                    const float *bias, const sige_conv_desc *cd, const float *gn_scale,
                    const float *gn_shift, int32_t silu, const void *residual, void *y,
                    const sige_tensor_desc *yd, void *workspace, size_t workspace_bytes,
                    sige_stream_t stream);

/* GroupNorm of the cached ORIGINAL activation folded into a per-channel
 * affine: scale[n][c] = gamma[c]/sqrt(var + eps), shift[n][c] = beta[c] -
 * mean*scale, mean and biased variance over H, W and the C/groups channels of
 * each group.  Computed once with the cache; the pages mention no
 * normalisation, and taking the statistics from the original keeps every op
 * of the sparse layer local.
 *   x : device NHWC f32 or bf16;  gamma, beta : device float32 [C];
 *   scale, shift : device float32 [N][C] */
int sige_groupnorm_affine(const void *x, const sige_tensor_desc *xd, int32_t groups,
                          const float *gamma, const float *beta, float eps, float *scale,
                          float *shift, sige_stream_t stream);

/* (7) Restore listed tiles from a source tensor, for sequential edits.
 * SIGE project page, "Overview", updates the cached F_l(A_original) in place
 * with the edited tiles; an interactive session applies edit after edit.  Each
 * edit's tile list comes from the mask against the ORIGINAL input, so it covers
 * every region that still differs; the tiles of the previous edit must first
 * be put back to their original values (a region the user reverted would
 * otherwise keep stale values).  This copies, for every in-image pixel of the
 * listed tiles,
 *   dst[n][h0+i][w0+j][:] = src[n][h0+i][w0+j][:]     (i, j < block)
 * where src holds the original cache (untouched) and dst the working cache.
 *   src, dst : device, NHWC, the same shape and dtype (u8, f32 or bf16), not
 *              overlapping
 *   idx      : device int32 (h0, w0) pairs; count : device int32, the number
 *              of valid pairs (only the first min(count, capacity) are used)
 * Every other byte of dst is left untouched.  Asynchronous on `stream`. */
int sige_restore_tiles(const void *src, void *dst, const sige_tensor_desc *d, int32_t block,
                       const int32_t *idx, const int32_t *count, int32_t capacity, sige_stream_t stream);

/* (7b) Incremental read-back of a layer's output to the host.  SIGE project
 * page, "Overview": only the active blocks are recomputed and scattered into
 * the cached output, so a host copy of that output, current before the edit,
 * differs from the new output only at the listed tiles.  This copies, for
 * every in-image pixel of the tiles listed in idx[0 .. min(count, capacity)),
 *   host_y[n][h0+i][w0+j][:] = y[n][h0+i][w0+j][:]     (i, j < block)
 * and leaves every other byte of host_y as it is: the device packs the tiles
 * (and a copy of the count and the list) into `staging`; one device-to-host
 * copy brings the count and the list, a second one the packed tiles of that
 * count, and the host places their rows.  Synchronous: it waits for `stream`
 * twice and returns once host_y is complete.
 *   y           : device NHWC (u8, f32 or bf16), C * element size a multiple
 *                 of 16 bytes, 16-byte aligned
 *   host_y      : host memory of y's shape (pinned or pageable)
 *   staging     : device scratch of sige_download_tiles_bytes(...) bytes,
 *                 16-byte aligned
 *   host_staging: host scratch of the same size (pinned, so that the copies
 *                 are asynchronous DMA)
 * Returns SIGE_OK, SIGE_ERR_INVALID_ARG (null or inconsistent arguments),
 * SIGE_ERR_UNSUPPORTED (layout, dtype or alignment) or SIGE_ERR_CUDA. */
size_t sige_download_tiles_bytes(const sige_tensor_desc *yd, int32_t block, int32_t capacity);
int sige_download_tiles(const void *y, const sige_tensor_desc *yd, int32_t block, const int32_t *idx,
                        const int32_t *count, int32_t capacity, void *staging, void *host_staging, void *host_y,
                        sige_stream_t stream);

/* (8) Attention step with pruned query tokens (nubint.ai review of the SIGE
 * paper, "Proposed method": attention layers by pruning the query tokens of
 * unedited regions; mer.dev notes, abstract: attention for Stable Diffusion).
 * For every token (pixel) under the first min(*count, capacity) tiles of
 * `idx` (block x block, clipped to the map), per head h:
 *   o[n][y][x][h*dvh : (h+1)*dvh] = softmax(q_h k_h^T / sqrt(dh)) v_h
 * over all `keys` keys, dh = qd->c / heads, dvh = dv / heads; float32
 * accumulation, one rounding of o to bf16.  Every other element of o is left
 * as it is.  The projections before and after are sparse 1x1 convolutions
 * (sige_conv_fused) on the same tile list.
 *   q     : device bf16 [N][H][W][D], described by qd (NHWC); read at the tokens
 *   k     : device bf16 [N][keys][D] (self-attention: the [N][H][W][D] key map)
 *   v     : device bf16 [N][keys][dv]
 *   idx, count, capacity, block : the tile list of this resolution (as (1))
 *   o     : device bf16 [N][H][W][dv], written at the tokens only; must not
 *           overlap q, k or v
 * Two kernels (sige_attention_path tells which one a layer gets):
 *   tensor cores, for dh and dvh multiples of 8 up to 64 and 16-byte aligned
 *     buffers: 128 query slots x 128-key chunks, S = q k^T and O += P v by
 *     tcgen05.mma, P = exp(S - running max) rounded to bf16 for the second
 *     product; the keys of a block are split over up to 8 CTAs of a cluster
 *     when the list is short, the partial rows merged in distributed shared
 *     memory.  A device-side wait that expires (a fault elsewhere) leaves the
 *     rows of that block unwritten;
 *   CUDA cores otherwise: fp32 scores and weights.
 * All buffers belong to the caller; nothing is allocated; asynchronous on
 * `stream`.  Errors: SIGE_ERR_INVALID_ARG (NULL pointer, non-positive size,
 * D or dv not a multiple of heads), SIGE_ERR_UNSUPPORTED (not bf16 NHWC,
 * block > 8, dh or dvh > 256), SIGE_ERR_CUDA (launch failure). */
int sige_attention_core(const void *q, const sige_tensor_desc *qd, const void *k, const void *v, int32_t keys,
                        int32_t dv, int32_t heads, const int32_t *idx, const int32_t *count, int32_t capacity,
                        int32_t block, void *o, sige_stream_t stream);

/* Which kernel sige_attention_core runs for queries described by qd, value
 * width dv and `heads` heads (16-byte aligned buffers): 1 = tcgen05 tensor
 * cores, 0 = CUDA cores; SIGE_ERR_INVALID_ARG / SIGE_ERR_UNSUPPORTED as that
 * call would return them.  Host only. */
int sige_attention_path(const sige_tensor_desc *qd, int32_t dv, int32_t heads);

/* ------------------------------------------------------------ utilities */

/* Workspace bytes for sige_sparse_conv / sige_conv_fused / sige_dense_conv
 * with this layer, batch and list capacity (capacity is ignored for the dense
 * call, which uses the full tile grid of an output of `out_h` x `out_w`).
 * With the output dimensions given (> 0), the size also covers a scratch copy
 * of the input for 3x3 layers that the tile GEMM can run: a fused or dense
 * call with GroupNorm / SiLU then transforms each input pixel once into it;
 * with a smaller workspace such a call runs on the general kernel. */
size_t sige_conv_workspace_bytes(const sige_conv_desc *cd, int32_t batch, int32_t capacity,
                                 int32_t out_h, int32_t out_w);

/* Workspace bytes of one call, by sige_call:
 *   SIGE_CALL_REDUCE_MASK : capacity = the number of tiles over all scale
 *                           grids (cd is ignored); an upper bound of
 *                           sige_reduce_mask_workspace_bytes for any split of
 *                           those tiles into at most SIGE_MAX_SCALES scales
 *   SIGE_CALL_SPARSE_CONV, SIGE_CALL_CONV_FUSED, SIGE_CALL_DENSE_CONV :
 *                           this layer, capacity = list capacity (dense: the
 *                           tiles of the output grid); the same value as
 *                           sige_conv_workspace_bytes with batch 1
 *   SIGE_CALL_RESBLOCK    : sige_resblock_fused (cd and capacity ignored)
 * 0 for an unknown call or invalid sizes. */
size_t sige_workspace_bytes(int32_t which_call, const sige_conv_desc *cd, int32_t capacity);

/* Synchronise `stream`, return the first device error recorded in the
 * workspace header (SIGE_OK if none) and clear it. */
int sige_get_error(void *workspace, sige_stream_t stream);

/* The same as sige_get_error: reads (and clears) the device error word in the
 * workspace header after synchronising `stream`. */
int sige_get_device_error(void *workspace, sige_stream_t stream);

/* Bound, in SM clock cycles, of the device-side waits that end a call with
 * SIGE_ERR_TIMEOUT when they expire, for every launch enqueued after this
 * call, process-wide; 0 restores each kernel's own bound (seconds).  Covered:
 * the wait of sige_reduce_mask's reducing CTA for the streaming CTAs, and the
 * grid barrier of sige_resblock_step (on expiry every CTA takes no tile, the
 * outputs are left as they were and the workspace stays consistent for the
 * next call; the error detail is the wait site, 111).  A test
 * of the failure path sets a bound of a few cycles so that the wait expires,
 * checks the status and restores 0.  Returns SIGE_ERR_INVALID_ARG for a
 * negative value. */
int sige_set_wait_cycles(int64_t cycles);

/* Which conv kernel the fused and dense calls (sige_conv_fused,
 * sige_dense_conv) of this layer and dtype run: 1 = tcgen05 tensor cores (the
 * general tile kernel, the 8x8-tile 3x3 kernel, or the tile GEMM for bf16
 * layers with C_in % 64 == 0 and C_out % 16 == 0 that are 1x1 stride 1, or
 * 3x3 pad 1 stride 1 or 2 on 4x4 / 8x8 tiles (any tile size for a dense call,
 * one-pixel tiles too for a sparse one; an input transform through a
 * pre-pass into the workspace when sige_conv_workspace_bytes sized it with
 * the output dimensions)), 0 = CUDA cores; negative = a
 * sige_status for an unsupported layer.  sige_sparse_conv (stacked blocks)
 * takes the general tile kernel or the CUDA cores. */
int sige_conv_path(const sige_conv_desc *cd, int32_t dtype);

/* Work decomposition of the tensor-core conv kernel for a bf16 layer, computed
 * on the host (no device work, no GPU needed): the same functions the kernel
 * runs at launch.  The active tiles are split into tile groups of T tiles
 * (slots), one unit per (tile group, 128 output channels, K split); a unit's S
 * K-splits are summed through a cluster peer (pair), by a reduce-scatter among
 * the S CTAs of one cluster, or through global memory (SIGE tile-based sparse
 * convolution, "Sparse Engine SIGE"; the split is this implementation's).
 *   tiles   : active tiles times batch (G), >= 0
 *   grid    : CTAs of the launch, a multiple of `cluster`
 *   cluster : CTAs per cluster (1 = no clusters)
 *   out     : host int32[n_out], filled with (missing entries 0):
 *             [0] B layout (0 ROW, 1 POS, 2 row-batched POS), [1] T, [2] tile
 *             groups, [3] K splits S, [4] units, [5] split sum (0 none, 1 pair,
 *             2 cluster reduce-scatter, 3 global), [6] accumulator columns of a
 *             unit, [7] weight stages, [8] halo stage bytes, [9] bytes the
 *             reduce-scatter stages (unpadded), [10] output-channel tiles,
 *             [11] 64-channel k-chunks, [12] cluster size a sparse launch asks
 *             for, [13] byte offset of the halo stages, [14] usable shared bytes
 * Returns SIGE_ERR_UNSUPPORTED for layers the tensor-core kernel does not run,
 * SIGE_ERR_INVALID_ARG for bad sizes. */
int sige_conv_schedule(const sige_conv_desc *cd, int32_t tiles, int32_t grid, int32_t cluster,
                       int32_t *out, int32_t n_out);

/* Number of kernels this library has launched in this process. */
uint64_t sige_launch_count(void);

const char *sige_status_string(int32_t status);

#ifdef __cplusplus
}
#endif

#endif /* SIGE_H */
