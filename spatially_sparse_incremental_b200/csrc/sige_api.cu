// C ABI entry points for the conv calls, host-side validation and utilities.
#include <algorithm>
#include <atomic>
#include <cmath>

#include "conv_common.cuh"
#include "conv_tc.cuh"

namespace sige {

static std::atomic<uint64_t> g_launches{0};
static std::atomic<long long> g_wait_cycles{0};   // 0: every kernel keeps its own default

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

long long wait_cycles_or(long long dflt)
{
    const long long v = g_wait_cycles.load(std::memory_order_relaxed);
    return v > 0 ? v : dflt;
}

int launch_check()
{
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? SIGE_OK : SIGE_ERR_CUDA;
}

int device_sm_count()
{
    static std::atomic<int> cache[64];   // per device, 0 = not yet queried
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64)
        return kNumSMs;
    int n = cache[d].load(std::memory_order_relaxed);
    if (!n) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, d) != cudaSuccess || n <= 0)
            n = kNumSMs;
        cache[d].store(n, std::memory_order_relaxed);
    }
    return n;
}

static int esize(int dtype) { return dtype == SIGE_BF16 ? 2 : dtype == SIGE_F32 ? 4 : 1; }

static int check_layer(const sige_conv_desc *cd, int dtype)
{
    if (!cd || cd->kernel < 1 || cd->stride < 1 || cd->pad < 0 || cd->pad >= cd->kernel ||
        cd->c_in < 1 || cd->c_out < 1 || cd->block < 1 || cd->block > 64)
        return SIGE_ERR_INVALID_ARG;
    if (dtype != SIGE_F32 && dtype != SIGE_BF16)
        return SIGE_ERR_UNSUPPORTED;
    const int bin = (cd->block - 1) * cd->stride + cd->kernel;
    if (bin * bin > 12288)
        return SIGE_ERR_UNSUPPORTED;
    return SIGE_OK;
}

// 1 = a tensor-core kernel runs the fused and dense calls of this layer,
// 0 = the CUDA-core kernel.
static int choose_path(const sige_conv_desc *cd, int dtype)
{
    return tc_supported(cd, dtype) || tile_gemm_supported(cd, dtype, false) ? 1 : 0;
}

static size_t ws_need(const sige_conv_desc *cd, int batch, int ntiles)
{
    return kWsHeader + tc_workspace_bytes(cd, batch, ntiles);
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

static int run_conv(ConvParams &p, const sige_conv_desc *cd, void *ws, size_t ws_bytes, cudaStream_t st)
{
    p.k = cd->kernel; p.s = cd->stride; p.pad = cd->pad; p.b = cd->block;
    p.bin = (cd->block - 1) * cd->stride + cd->kernel;
    p.Cin = cd->c_in; p.Cout = cd->c_out;
    p.ws = static_cast<uint8_t *>(ws);
    p.ws_bytes = ws_bytes;
    const int ntiles = p.dense ? p.tiles_total : p.cap;
    if (!ws || ws_bytes < ws_need(cd, p.N, ntiles) || !aligned16(ws))
        return SIGE_ERR_WORKSPACE;
    if (ntiles == 0)
        return SIGE_OK;
    // image to image: the 8x8-tile kernel (no GauGAN extension) or the tile
    // GEMM when they fit (a transposed conv with an input transform: the
    // general kernel)
    const bool image = p.from_image && p.to_y;
    const bool plain = image && !p.tstride && !p.sg && !p.leaky;
    const bool xform = p.gsc || p.silu || p.sg || p.leaky;
    if (plain && conv8_supported(cd, p.dtype))
        return launch_conv8(p, st);
    if (image && tile_gemm_supported(cd, p.dtype, p.dense != 0)) {
        // no transform (transposed convs included: rows copied per thread),
        // or a 1x1 layer's GroupNorm / SiLU applied in the GEMM
        if (!xform || (plain && cd->kernel == 1))
            return launch_tile_gemm(p, st);
        // a 3x3 layer with an input transform: the transform once per pixel
        // into a scratch copy in the workspace (transforming every tap's copy
        // of a row measured 1.7-3.9x slower than the general kernel), when the
        // workspace was sized by sige_conv_workspace_bytes
        const size_t base = (ws_need(cd, p.N, ntiles) + 255) & ~(size_t)255;
        if (!p.tstride && cd->kernel == 3 && ws_bytes >= base + tile_gemm_scratch_bytes(cd, p.N, p.H, p.W))
            return launch_tile_gemm_pre(p, p.ws + base, st);
    }
    if (tc_supported(cd, p.dtype))
        return launch_conv_tc(p, st);
    return launch_conv_simt(p, st);
}

} // namespace sige

using namespace sige;

extern "C" size_t sige_conv_workspace_bytes(const sige_conv_desc *cd, int32_t batch, int32_t capacity,
                                            int32_t out_h, int32_t out_w)
{
    if (!cd || cd->block < 1 || batch < 1 || capacity < 0)
        return 0;
    const int64_t dense_tiles = (int64_t)((out_h + cd->block - 1) / cd->block) * ((out_w + cd->block - 1) / cd->block);
    const int64_t nt = std::max<int64_t>(capacity, dense_tiles);
    // the same layer run as a transposed conv plans as a stride-1 conv
    sige_conv_desc v = *cd;
    v.stride = 1;
    v.pad = std::max(0, cd->kernel - 1 - cd->pad);
    const int n = (int)std::min<int64_t>(nt, INT32_MAX);
    size_t need = std::max(ws_need(cd, batch, n), ws_need(&v, batch, n));
    // the tile GEMM's scratch copy of a transformed input (3x3 layers; sized
    // from the output dimensions, so only when they are given)
    if (tile_gemm_supported(cd, SIGE_BF16, true) && cd->kernel == 3 && out_h > 0 && out_w > 0)
        need = ((ws_need(cd, batch, n) + 255) & ~(size_t)255) +
               tile_gemm_scratch_bytes(cd, batch, out_h * cd->stride + cd->kernel, out_w * cd->stride + cd->kernel);
    return std::max(need, std::max(ws_need(cd, batch, n), ws_need(&v, batch, n)));
}

extern "C" int sige_conv_path(const sige_conv_desc *cd, int32_t dtype)
{
    const int st = check_layer(cd, dtype);
    if (st != SIGE_OK)
        return st;
    return choose_path(cd, dtype);
}

extern "C" int sige_conv_schedule(const sige_conv_desc *cd, int32_t tiles, int32_t grid, int32_t cluster,
                                  int32_t *out, int32_t n_out)
{
    if (check_layer(cd, SIGE_BF16) != SIGE_OK || !tc_supported(cd, SIGE_BF16))
        return SIGE_ERR_UNSUPPORTED;
    return tc_schedule(cd, tiles, grid, cluster, out, n_out);
}

extern "C" int sige_sparse_conv(const void *blocks, const sige_conv_desc *cd, int32_t dtype, int32_t batch,
                                const void *weight, const int32_t *count, int32_t capacity,
                                float *out_blocks, void *workspace, size_t workspace_bytes,
                                sige_stream_t stream)
{
    if (!blocks || !weight || !count || !out_blocks || batch < 1 || capacity < 0)
        return SIGE_ERR_INVALID_ARG;
    const int st = check_layer(cd, dtype);
    if (st != SIGE_OK)
        return st;
    if (!aligned16(blocks) || !aligned16(weight) || !aligned16(out_blocks))
        return SIGE_ERR_UNSUPPORTED;
    ConvParams p{};
    p.src = static_cast<const uint8_t *>(blocks);
    p.N = batch; p.dtype = dtype;
    p.count = count; p.cap = capacity;
    p.w = static_cast<const uint8_t *>(weight);
    p.out_blocks = out_blocks;
    p.from_image = 0; p.to_y = 0;
    return run_conv(p, cd, workspace, workspace_bytes, (cudaStream_t)stream);
}

static int fused_common(ConvParams &p, const void *x, const sige_tensor_desc *xd, const void *weight,
                        const float *bias, const sige_conv_desc *cd, const float *gn_scale,
                        const float *gn_shift, int32_t silu, const void *residual, void *y,
                        const sige_tensor_desc *yd)
{
    if (!x || !xd || !weight || !y || !yd)
        return SIGE_ERR_INVALID_ARG;
    if ((gn_scale == nullptr) != (gn_shift == nullptr))
        return SIGE_ERR_INVALID_ARG;
    const int st = check_layer(cd, xd->dtype);
    if (st != SIGE_OK)
        return st;
    if (xd->layout != SIGE_NHWC || yd->layout != SIGE_NHWC || yd->dtype != xd->dtype)
        return SIGE_ERR_UNSUPPORTED;
    if (xd->n < 1 || xd->h < 1 || xd->w < 1 || xd->c != cd->c_in)
        return SIGE_ERR_INVALID_ARG;
    const int Ho = (xd->h + 2 * cd->pad - cd->kernel) / cd->stride + 1;
    const int Wo = (xd->w + 2 * cd->pad - cd->kernel) / cd->stride + 1;
    if (Ho < 1 || Wo < 1 || yd->n != xd->n || yd->h != Ho || yd->w != Wo || yd->c != cd->c_out)
        return SIGE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(weight) || !aligned16(y) || !aligned16(residual) ||
        !aligned16(bias) || !aligned16(gn_scale) || !aligned16(gn_shift))
        return SIGE_ERR_UNSUPPORTED;
    p.src = static_cast<const uint8_t *>(x);
    p.N = xd->n; p.H = xd->h; p.W = xd->w; p.dtype = xd->dtype;
    p.gsc = gn_scale; p.gsh = gn_shift; p.silu = silu ? 1 : 0;
    p.w = static_cast<const uint8_t *>(weight);
    p.bias = bias;
    p.residual = static_cast<const uint8_t *>(residual);
    p.y = static_cast<uint8_t *>(y);
    p.Ho = Ho; p.Wo = Wo;
    p.from_image = 1; p.to_y = 1;
    (void)esize;
    return SIGE_OK;
}

extern "C" int sige_conv_fused(const void *x, const sige_tensor_desc *xd, const void *weight,
                               const float *bias, const sige_conv_desc *cd, const int32_t *idx,
                               const int32_t *count, int32_t capacity, const float *gn_scale,
                               const float *gn_shift, int32_t silu, const void *residual, void *y,
                               const sige_tensor_desc *yd, void *workspace, size_t workspace_bytes,
                               sige_stream_t stream)
{
    if (!idx || !count || capacity < 0)
        return SIGE_ERR_INVALID_ARG;
    ConvParams p{};
    int st = fused_common(p, x, xd, weight, bias, cd, gn_scale, gn_shift, silu, residual, y, yd);
    if (st != SIGE_OK)
        return st;
    if (reinterpret_cast<uintptr_t>(idx) & 7)
        return SIGE_ERR_INVALID_ARG;
    p.idx = idx; p.count = count; p.cap = capacity; p.dense = 0;
    return run_conv(p, cd, workspace, workspace_bytes, (cudaStream_t)stream);
}

extern "C" int sige_dense_conv(const void *x, const sige_tensor_desc *xd, const void *weight,
                               const float *bias, const sige_conv_desc *cd, const float *gn_scale,
                               const float *gn_shift, int32_t silu, const void *residual, void *y,
                               const sige_tensor_desc *yd, void *workspace, size_t workspace_bytes,
                               sige_stream_t stream)
{
    ConvParams p{};
    int st = fused_common(p, x, xd, weight, bias, cd, gn_scale, gn_shift, silu, residual, y, yd);
    if (st != SIGE_OK)
        return st;
    p.dense = 1;
    p.tiles_w = (p.Wo + cd->block - 1) / cd->block;
    p.tiles_total = ((p.Ho + cd->block - 1) / cd->block) * p.tiles_w;
    p.cap = p.tiles_total;
    return run_conv(p, cd, workspace, workspace_bytes, (cudaStream_t)stream);
}

extern "C" int sige_conv_fused_ext(const void *x, const sige_tensor_desc *xd, const void *weight, const float *bias,
                                   const sige_conv_desc *cd, const sige_layer_ext *ext, const int32_t *idx,
                                   const int32_t *count, int32_t capacity, const float *gn_scale,
                                   const float *gn_shift, const void *residual, void *y,
                                   const sige_tensor_desc *yd, void *workspace, size_t workspace_bytes,
                                   sige_stream_t stream)
{
    if (!x || !xd || !weight || !y || !yd || !cd || !ext)
        return SIGE_ERR_INVALID_ARG;
    if ((gn_scale == nullptr) != (gn_shift == nullptr) || (ext->spade_beta && !ext->spade_gamma))
        return SIGE_ERR_INVALID_ARG;
    if (idx && (!count || capacity < 0 || (reinterpret_cast<uintptr_t>(idx) & 7)))
        return SIGE_ERR_INVALID_ARG;
    if (ext->act < 0 || ext->act > 2 || ext->transposed < 0 || ext->transposed > 1 || ext->output_padding < 0)
        return SIGE_ERR_INVALID_ARG;
    int st = check_layer(cd, xd->dtype);
    if (st != SIGE_OK)
        return st;
    if (xd->n < 1 || xd->h < 1 || xd->w < 1 || xd->c != cd->c_in)
        return SIGE_ERR_INVALID_ARG;
    // a transposed conv runs as a stride-1 conv over the input with stride - 1
    // zeros between pixels, padded by k - 1 - pad, with the taps reversed
    sige_conv_desc vcd = *cd;
    int Ho, Wo;
    if (ext->transposed) {
        if (ext->output_padding >= cd->stride)
            return SIGE_ERR_INVALID_ARG;
        vcd.stride = 1;
        vcd.pad = cd->kernel - 1 - cd->pad;
        Ho = (xd->h - 1) * cd->stride - 2 * cd->pad + cd->kernel + ext->output_padding;
        Wo = (xd->w - 1) * cd->stride - 2 * cd->pad + cd->kernel + ext->output_padding;
    } else {
        if (ext->output_padding != 0)
            return SIGE_ERR_INVALID_ARG;
        Ho = (xd->h + 2 * cd->pad - cd->kernel) / cd->stride + 1;
        Wo = (xd->w + 2 * cd->pad - cd->kernel) / cd->stride + 1;
    }
    if (Ho < 1 || Wo < 1 || yd->n != xd->n || yd->h != Ho || yd->w != Wo || yd->c != cd->c_out)
        return SIGE_ERR_INVALID_ARG;
    if (xd->dtype != SIGE_BF16 || xd->layout != SIGE_NHWC || yd->layout != SIGE_NHWC || yd->dtype != xd->dtype ||
        !tc_supported(&vcd, SIGE_BF16))
        return SIGE_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(weight) || !aligned16(y) || !aligned16(residual) || !aligned16(bias) ||
        !aligned16(gn_scale) || !aligned16(gn_shift) || !aligned16(ext->spade_gamma) || !aligned16(ext->spade_beta))
        return SIGE_ERR_UNSUPPORTED;
    ConvParams p{};
    p.src = static_cast<const uint8_t *>(x);
    p.N = xd->n; p.H = xd->h; p.W = xd->w; p.dtype = xd->dtype;
    p.gsc = gn_scale; p.gsh = gn_shift;
    p.silu = ext->act == 1;
    p.leaky = ext->act == 2;
    p.sg = static_cast<const uint8_t *>(ext->spade_gamma);
    p.sb = static_cast<const uint8_t *>(ext->spade_beta);
    p.tstride = ext->transposed ? cd->stride : 0;
    p.w = static_cast<const uint8_t *>(weight);
    p.bias = bias;
    p.residual = static_cast<const uint8_t *>(residual);
    p.y = static_cast<uint8_t *>(y);
    p.Ho = Ho; p.Wo = Wo;
    p.from_image = 1; p.to_y = 1;
    if (idx) {
        p.idx = idx; p.count = count; p.cap = capacity; p.dense = 0;
    } else {
        p.dense = 1;
        p.tiles_w = (Wo + cd->block - 1) / cd->block;
        p.tiles_total = ((Ho + cd->block - 1) / cd->block) * p.tiles_w;
        p.cap = p.tiles_total;
    }
    return run_conv(p, &vcd, workspace, workspace_bytes, (cudaStream_t)stream);
}

extern "C" int sige_get_error(void *workspace, sige_stream_t stream)
{
    if (!workspace)
        return SIGE_ERR_INVALID_ARG;
    int32_t h[2] = {0, 0};
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(h, workspace, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return SIGE_ERR_CUDA;
    if (h[0] != 0) {
        if (cudaMemsetAsync(workspace, 0, sizeof h, st) != cudaSuccess || cudaStreamSynchronize(st) != cudaSuccess)
            return SIGE_ERR_CUDA;
    }
    return h[0];
}

extern "C" int sige_get_device_error(void *workspace, sige_stream_t stream)
{
    return sige_get_error(workspace, stream);
}

extern "C" int sige_set_wait_cycles(int64_t cycles)
{
    if (cycles < 0)
        return SIGE_ERR_INVALID_ARG;
    g_wait_cycles.store((long long)cycles, std::memory_order_relaxed);
    return SIGE_OK;
}

extern "C" size_t sige_workspace_bytes(int32_t which_call, const sige_conv_desc *cd, int32_t capacity)
{
    if (capacity < 0)
        return 0;
    switch (which_call) {
    case SIGE_CALL_REDUCE_MASK:
        // header + one flag byte per tile of every scale, each scale padded to
        // 16 bytes (at most SIGE_MAX_SCALES of them)
        return kWsHeader + (((size_t)capacity + 15) & ~(size_t)15) + 16 * (size_t)SIGE_MAX_SCALES;
    case SIGE_CALL_SPARSE_CONV:
    case SIGE_CALL_CONV_FUSED:
    case SIGE_CALL_DENSE_CONV:
        if (!cd || cd->block < 1)
            return 0;
        return ws_need(cd, 1, capacity);
    case SIGE_CALL_RESBLOCK:
        return kWsHeader;
    default:
        return 0;
    }
}

extern "C" uint64_t sige_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

extern "C" const char *sige_status_string(int32_t status)
{
    switch (status) {
    case SIGE_OK: return "ok";
    case SIGE_ERR_INVALID_ARG: return "invalid argument";
    case SIGE_ERR_UNSUPPORTED: return "unsupported shape, dtype or layout";
    case SIGE_ERR_CUDA: return "CUDA error";
    case SIGE_ERR_CAPACITY: return "more active tiles than the list capacity";
    case SIGE_ERR_TIMEOUT: return "bounded wait expired on the device";
    case SIGE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    default: return "unknown status";
    }
}
