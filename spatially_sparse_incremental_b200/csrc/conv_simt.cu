// Layer F_l on the CUDA cores (float32 arithmetic): the path for float32
// layers, and for bf16 layers the tensor-core kernel does not cover.
//
// One CTA works on one (tile, batch item, group of output channels) unit at a
// time.  It stages the tile's halo'd input block in shared memory (from the
// stacked blocks, or straight from the image with zero padding and the
// GroupNorm affine + SiLU applied on the way in), then each thread accumulates
// one output channel for a few of the tile's pixels.  The epilogue either
// writes float32 output blocks or scatters bias + residual + one rounding into
// the cached output.
#include <algorithm>

#include "conv_common.cuh"
#include "transform.cuh"

namespace sige {

constexpr int kSimtThreads = 256;
constexpr int kSimtMaxQ = 16;
constexpr int kSimtSmemFloats = 12288;  // 48 KB

__global__ void __launch_bounds__(kSimtThreads) k_conv_simt(const __grid_constant__ ConvParams p)
{
    extern __shared__ float sm[];
    const int ntiles = p.dense ? p.tiles_total : min(__ldg(p.count), p.cap);
    const int ncog = (p.Cout + p.cob - 1) / p.cob;
    const int units = ntiles * p.N * ncog;
    const int npx = p.b * p.b;
    const int ol = threadIdx.x % p.cob, pgi = threadIdx.x / p.cob;
    const int esz = p.dtype == SIGE_BF16 ? 2 : 4;
    const bool xform = p.gsc != nullptr || p.silu;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int cog = u % ncog;
        const int tn = u / ncog;
        const int n = tn % p.N, t = tn / p.N;
        int h0 = 0, w0 = 0;
        if (p.from_image || p.to_y)   // stacked blocks carry no tile list
            tile_origin(p, t, h0, w0);
        const int o = cog * p.cob + ol;
        float acc[kSimtMaxQ];
#pragma unroll
        for (int q = 0; q < kSimtMaxQ; ++q)
            acc[q] = 0.0f;
        for (int ci0 = 0; ci0 < p.Cin; ci0 += p.ci_chunk) {
            const int cc = min(p.ci_chunk, p.Cin - ci0);
            __syncthreads();
            for (int e = threadIdx.x; e < p.bin * p.bin * cc; e += blockDim.x) {
                const int pix = e / cc, ci = e % cc;
                const int hh = pix / p.bin, ww = pix % p.bin;
                float v = 0.0f;
                if (p.from_image) {
                    const int y = h0 * p.s - p.pad + hh, x = w0 * p.s - p.pad + ww;
                    if (y >= 0 && y < p.H && x >= 0 && x < p.W) {
                        v = load_elem(p.src, (((int64_t)n * p.H + y) * p.W + x) * p.Cin + ci0 + ci, p.dtype);
                        if (xform) {
                            v = transform1(v, p.gsc ? p.gsc + (int64_t)n * p.Cin : nullptr,
                                           p.gsc ? p.gsh + (int64_t)n * p.Cin : nullptr, ci0 + ci, p.silu);
                            if (p.dtype == SIGE_BF16)
                                v = __bfloat162float(__float2bfloat16_rn(v));
                        }
                    }
                } else {
                    v = load_elem(p.src, (((int64_t)t * p.N + n) * p.bin * p.bin + pix) * p.Cin + ci0 + ci, p.dtype);
                }
                sm[pix * cc + ci] = v;
            }
            __syncthreads();
            if (o < p.Cout) {
                for (int r = 0; r < p.k; ++r)
                    for (int c = 0; c < p.k; ++c) {
                        const int64_t wrow = (((int64_t)o * p.k + r) * p.k + c) * p.Cin + ci0;
                        for (int ci = 0; ci < cc; ++ci) {
                            const float wv = load_elem(p.w, wrow + ci, p.dtype);
#pragma unroll
                            for (int q = 0; q < kSimtMaxQ; ++q) {
                                const int pp = pgi + p.pg * q;
                                if (pp < npx) {
                                    const int i = pp / p.b, j = pp % p.b;
                                    acc[q] = fmaf(wv, sm[((i * p.s + r) * p.bin + j * p.s + c) * cc + ci], acc[q]);
                                }
                            }
                        }
                    }
            }
        }
        (void)esz;
        if (o < p.Cout) {
#pragma unroll
            for (int q = 0; q < kSimtMaxQ; ++q) {
                const int pp = pgi + p.pg * q;
                if (pp >= npx)
                    continue;
                const int i = pp / p.b, j = pp % p.b;
                if (p.to_y) {
                    const int yo = h0 + i, xo = w0 + j;
                    if (yo < p.Ho && xo < p.Wo)
                        store_out1(p.y, (((int64_t)n * p.Ho + yo) * p.Wo + xo) * p.Cout + o, p.dtype, acc[q],
                                   p.bias ? __ldg(p.bias + o) : 0.0f, p.residual);
                } else {
                    p.out_blocks[(((int64_t)t * p.N + n) * npx + pp) * p.Cout + o] = acc[q];
                }
            }
        }
    }
}

static int pow2_ceil(int v)
{
    int r = 1;
    while (r < v)
        r <<= 1;
    return r;
}

int launch_conv_simt(ConvParams p, cudaStream_t stream)
{
    const int npx = p.b * p.b;
    int pg = std::max(kSimtThreads / std::min(kSimtThreads, pow2_ceil(p.Cout)), pow2_ceil((npx + kSimtMaxQ - 1) / kSimtMaxQ));
    if (pg > kSimtThreads)
        return SIGE_ERR_UNSUPPORTED;
    p.pg = pg;
    p.cob = kSimtThreads / pg;
    const int bin2 = p.bin * p.bin;
    p.ci_chunk = std::min(p.Cin, std::max(1, kSimtSmemFloats / bin2));
    if (p.ci_chunk < 1)
        return SIGE_ERR_UNSUPPORTED;
    const size_t smem = (size_t)bin2 * p.ci_chunk * sizeof(float);
    if (smem > 48 * 1024)
        return SIGE_ERR_UNSUPPORTED;
    const int ncog = (p.Cout + p.cob - 1) / p.cob;
    const int64_t max_units = (int64_t)(p.dense ? p.tiles_total : p.cap) * p.N * ncog;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(max_units, (int64_t)device_sm_count() * 8));
    prefer_max_shared(k_conv_simt);
    k_conv_simt<<<grid, kSimtThreads, smem, stream>>>(p);
    count_launch();
    return launch_check();
}

} // namespace sige
