// Parameters shared by the conv kernels (CUDA-core and tensor-core paths).
#pragma once

#include "sige_internal.cuh"

namespace sige {

struct ConvParams {
    // source: stacked blocks [tile][n][bin][bin][Cin] (from_image == 0) or the
    // NHWC image [n][H][W][Cin] (from_image == 1)
    const uint8_t *src;
    int32_t N, H, W, Cin, Cout, dtype;
    int32_t k, s, pad, b, bin;
    // tile list (sparse) or the full tile grid of the output (dense)
    const int32_t *idx;
    const int32_t *count;
    int32_t cap;
    int32_t dense, tiles_w, tiles_total;
    // input transform (GroupNorm affine, SiLU)
    const float *gsc, *gsh;
    int32_t silu;
    // GauGAN-style layers: a per-pixel modulation of the transformed input
    // (t * (1 + sg) + sb, NHWC maps of the input's shape) and LeakyReLU(0.2)
    // instead of SiLU; tstride > 0: a transposed conv of that stride, run as a
    // stride-1 conv over the input with tstride - 1 zeros between pixels
    // (pad = k - 1 - its padding) and the taps reversed
    const uint8_t *sg, *sb;
    int32_t leaky;
    int32_t tstride;
    const uint8_t *w;  // [Cout][k][k][Cin]
    // destination: float32 output blocks (to_y == 0) or the cached output y
    float *out_blocks;
    const float *bias;
    const uint8_t *residual;
    uint8_t *y;
    int32_t Ho, Wo;
    int32_t from_image, to_y;
    // CUDA-core kernel launch shape
    int32_t ci_chunk, pg, cob;
    // workspace (tensor-core kernel)
    uint8_t *ws;
    size_t ws_bytes;
};

__device__ __forceinline__ void tile_origin(const ConvParams &p, int t, int &h0, int &w0)
{
    if (p.dense) {
        h0 = (t / p.tiles_w) * p.b;
        w0 = (t % p.tiles_w) * p.b;
    } else {
        const int2 o = __ldg(reinterpret_cast<const int2 *>(p.idx) + t);
        h0 = o.x;
        w0 = o.y;
    }
}

int launch_conv_simt(ConvParams p, cudaStream_t stream);

} // namespace sige
