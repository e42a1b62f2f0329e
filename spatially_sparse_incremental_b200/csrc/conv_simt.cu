// Layer F_l on the CUDA cores (float32 arithmetic): the path for float32
// layers, and for bf16 layers the tensor-core kernel does not cover.
//
// Tiles of at most 16 pixels (b <= 4) run k_conv_simt16: a unit of 16 output
// channels x 16 pixel slots, 16 K groups of 16 threads each holding a
// 4-channel x 4-pixel block of accumulators, weights and halo staged per
// input-channel chunk in shared memory (float32: asynchronous 4-byte copies),
// the K groups summed in a fixed order at the end.  Larger tiles run
// k_conv_simt: one CTA per (tile, batch item, group of output channels), each
// thread one output channel for up to 16 of the tile's pixels.  Both stage the
// halo from the stacked blocks, or straight from the image with zero padding
// and the GroupNorm affine + SiLU applied on the way in, and end by writing
// float32 output blocks or scattering bias + residual + one rounding into the
// cached output.
#include <algorithm>
#include <atomic>

#include "conv_common.cuh"
#include "transform.cuh"

namespace sige {

constexpr int kSimtThreads = 256;
constexpr int kSimtMaxQ = 16;
constexpr int kSimtSmemFloats = 12288;  // 48 KB
constexpr int kStageBatch = 8;           // loads in flight per thread while staging

// Read-only element load (input activations and weights are never written here).
__device__ __forceinline__ float ldg_elem(const uint8_t *base, int64_t e, int dtype)
{
    if (dtype == SIGE_BF16)
        return __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(base) + e) << 16);
    return __ldg(reinterpret_cast<const float *>(base) + e);
}

// acc[q] += sum over taps and the chunk's channels of w * x, for the NQ pixels
// of this thread (NQ a compile-time count so no lane issues idle FMAs).
template <int NQ>
__device__ __forceinline__ void accumulate(float (&acc)[kSimtMaxQ], const int (&pix0)[kSimtMaxQ], const float *sm,
                                           const float *sw, int wst, int ol, int cc, int k, int bin)
{
#pragma unroll 1
    for (int r = 0; r < k; ++r)
#pragma unroll 1
        for (int c = 0; c < k; ++c) {
            const float *wrow = sw + (r * k + c) * cc * wst + ol;
            const float *xs[NQ];
#pragma unroll
            for (int q = 0; q < NQ; ++q)
                xs[q] = sm + (pix0[q] + r * bin + c) * cc;
#pragma unroll 4
            for (int ci = 0; ci < cc; ++ci) {
                const float wv = wrow[ci * wst];
#pragma unroll
                for (int q = 0; q < NQ; ++q)
                    acc[q] = fmaf(wv, xs[q][ci], acc[q]);
            }
        }
}

__global__ void __launch_bounds__(kSimtThreads) k_conv_simt(const __grid_constant__ ConvParams p)
{
    extern __shared__ float sm[];
    float *sw = sm + p.bin * p.bin * p.ci_chunk;   // weights [tap][ci][cob + 1]
    const int wst = p.cob + 1;
    const int taps = p.k * p.k;
    const int ntiles = p.dense ? p.tiles_total : min(__ldg(p.count), p.cap);
    const int ncog = (p.Cout + p.cob - 1) / p.cob;
    const int units = ntiles * p.N * ncog;
    const int npx = p.b * p.b;
    const int ol = threadIdx.x % p.cob, pgi = threadIdx.x / p.cob;
    const int nq = pgi < npx ? (npx - pgi + p.pg - 1) / p.pg : 0;   // this thread's pixels
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
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
        int pix0[kSimtMaxQ];   // halo pixel of output pixel q at tap (0, 0)
#pragma unroll
        for (int q = 0; q < kSimtMaxQ; ++q) {
            acc[q] = 0.0f;
            const int pp = min(pgi + p.pg * q, npx - 1);
            pix0[q] = (pp / p.b) * p.s * p.bin + (pp % p.b) * p.s;
        }
        for (int ci0 = 0; ci0 < p.Cin; ci0 += p.ci_chunk) {
            const int cc = min(p.ci_chunk, p.Cin - ci0);
            __syncthreads();
            // Staging: a warp takes a row (one halo pixel, or one (output
            // channel, tap) of the weights) and its lanes the row's channels, so
            // the index arithmetic is per row; each lane issues up to
            // kStageBatch loads before it stores them.
            const int npix = p.bin * p.bin;
#pragma unroll 1
            for (int r0 = warp; r0 < npix; r0 += nwarp * kStageBatch) {
                float v[kStageBatch];
#pragma unroll
                for (int k = 0; k < kStageBatch; ++k) {
                    v[k] = 0.0f;
                    const int pix = r0 + k * nwarp;
                    if (pix >= npix || lane >= cc)
                        continue;
                    const int hh = pix / p.bin, ww = pix - hh * p.bin;
                    if (p.from_image) {
                        const int y = h0 * p.s - p.pad + hh, x = w0 * p.s - p.pad + ww;
                        if (y >= 0 && y < p.H && x >= 0 && x < p.W) {
                            float xv = ldg_elem(p.src, (((int64_t)n * p.H + y) * p.W + x) * p.Cin + ci0 + lane, p.dtype);
                            if (xform) {   // padding stays zero
                                xv = transform1(xv, p.gsc ? p.gsc + (int64_t)n * p.Cin : nullptr,
                                                p.gsc ? p.gsh + (int64_t)n * p.Cin : nullptr, ci0 + lane, p.silu);
                                if (p.dtype == SIGE_BF16)
                                    xv = __bfloat162float(__float2bfloat16_rn(xv));
                            }
                            v[k] = xv;
                        }
                    } else {
                        v[k] = ldg_elem(p.src, (((int64_t)t * p.N + n) * npix + pix) * p.Cin + ci0 + lane, p.dtype);
                    }
                }
#pragma unroll
                for (int k = 0; k < kStageBatch; ++k) {
                    const int pix = r0 + k * nwarp;
                    if (pix < npix && lane < cc)
                        sm[pix * cc + lane] = v[k];
                }
            }
            // chunks of more than 32 channels: the remaining lanes' share
#pragma unroll 1
            for (int e = 32; e < cc; e += 32)
#pragma unroll 1
                for (int pix = warp; pix < npix; pix += nwarp) {
                    const int ci = e + lane;
                    if (ci >= cc)
                        continue;
                    const int hh = pix / p.bin, ww = pix - hh * p.bin;
                    float xv = 0.0f;
                    if (p.from_image) {
                        const int y = h0 * p.s - p.pad + hh, x = w0 * p.s - p.pad + ww;
                        if (y >= 0 && y < p.H && x >= 0 && x < p.W) {
                            xv = ldg_elem(p.src, (((int64_t)n * p.H + y) * p.W + x) * p.Cin + ci0 + ci, p.dtype);
                            if (xform) {
                                xv = transform1(xv, p.gsc ? p.gsc + (int64_t)n * p.Cin : nullptr,
                                                p.gsc ? p.gsh + (int64_t)n * p.Cin : nullptr, ci0 + ci, p.silu);
                                if (p.dtype == SIGE_BF16)
                                    xv = __bfloat162float(__float2bfloat16_rn(xv));
                            }
                        }
                    } else {
                        xv = ldg_elem(p.src, (((int64_t)t * p.N + n) * npix + pix) * p.Cin + ci0 + ci, p.dtype);
                    }
                    sm[pix * cc + ci] = xv;
                }
            // weights of this channel group and chunk: row (output channel, tap)
            // is contiguous over input channels in [C_out][k][k][C_in]
            const int nrow = p.cob * taps;
#pragma unroll 1
            for (int r0 = warp; r0 < nrow; r0 += nwarp * kStageBatch) {
#pragma unroll 1
                for (int e = 0; e < cc; e += 32) {
                    const int ci = e + lane;
                    float v[kStageBatch];
#pragma unroll
                    for (int k = 0; k < kStageBatch; ++k) {
                        v[k] = 0.0f;
                        const int row = r0 + k * nwarp;
                        if (row >= nrow || ci >= cc)
                            continue;
                        const int ol2 = row / taps, tap = row - ol2 * taps;
                        const int o2 = cog * p.cob + ol2;
                        if (o2 < p.Cout)
                            v[k] = ldg_elem(p.w, ((int64_t)o2 * taps + tap) * p.Cin + ci0 + ci, p.dtype);
                    }
#pragma unroll
                    for (int k = 0; k < kStageBatch; ++k) {
                        const int row = r0 + k * nwarp;
                        if (row >= nrow || ci >= cc)
                            continue;
                        const int ol2 = row / taps, tap = row - ol2 * taps;
                        sw[(tap * cc + ci) * wst + ol2] = v[k];
                    }
                }
            }
            __syncthreads();
            if (o < p.Cout) {
                // a power of two at least nq: the extra accumulators read a valid
                // (clamped) pixel and are never stored
                switch (nq <= 1 ? 1 : nq <= 2 ? 2 : nq <= 4 ? 4 : nq <= 8 ? 8 : 16) {
                case 16: accumulate<16>(acc, pix0, sm, sw, wst, ol, cc, p.k, p.bin); break;
                case 8: accumulate<8>(acc, pix0, sm, sw, wst, ol, cc, p.k, p.bin); break;
                case 4: accumulate<4>(acc, pix0, sm, sw, wst, ol, cc, p.k, p.bin); break;
                case 2: accumulate<2>(acc, pix0, sm, sw, wst, ol, cc, p.k, p.bin); break;
                default: accumulate<1>(acc, pix0, sm, sw, wst, ol, cc, p.k, p.bin); break;
                }
            }
        }
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

// Tiles of at most 16 pixels (b <= 4): register-blocked.  A unit is 16 output
// channels x 16 pixel slots of one tile; its 256 threads form 16 K groups (input
// channel ci of a chunk goes to group ci % 16) of 16 threads, and each thread
// holds a 4-channel x 4-pixel block of accumulators, so one 16-byte weight read
// and four input reads feed 16 FMAs.  The K groups are summed in a fixed order
// through shared memory at the end.
constexpr int kS16Threads = 256;
constexpr int kS16Cout = 16;            // output channels per unit (fewer per unit: more CTAs on few tiles)
constexpr int kS16Cq = kS16Cout / 4;    // 4-channel groups of a unit
constexpr int kS16Kg = kS16Threads / (kS16Cq * 4);   // K groups (a K group: kS16Cq x 4 pixel groups of threads)
static_assert(kS16Kg * kS16Cq * 4 == kS16Threads && kS16Kg * 16 * kS16Cout <= 4096, "unit shape");
constexpr int kS16WStride = kS16Cout + 4;   // weight row stride (floats): 16-byte aligned, fewer bank conflicts
constexpr int kS16SmemFloats = 24576;   // 96 KB: two CTAs per SM, fewer channel chunks

__global__ void __launch_bounds__(kS16Threads, 1) k_conv_simt16(const __grid_constant__ ConvParams p)
{
    extern __shared__ __align__(16) float s16[];
    const int taps = p.k * p.k, npix = p.bin * p.bin, npx = p.b * p.b;
    const int cmax = p.ci_chunk;
    float *sx = s16;                                            // [pixel][cc]
    float *sw = s16 + ((npix * cmax + 3) & ~3);                 // [tap][cc][kS16WStride]
    float *red = s16;                                           // [K group][16 px][64 co], after the last chunk
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarp = kS16Threads / 32;
    const int kg = tid / (kS16Cq * 4), cq = tid % kS16Cq, pq = (tid / kS16Cq) & 3;
    const int ntiles = p.dense ? p.tiles_total : min(__ldg(p.count), p.cap);
    const int ncog = (p.Cout + kS16Cout - 1) / kS16Cout;
    const int units = ntiles * p.N * ncog;
    const bool xform = p.gsc != nullptr || p.silu;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int cog = u % ncog;
        const int tn = u / ncog;
        const int n = tn % p.N, t = tn / p.N;
        int h0 = 0, w0 = 0;
        if (p.from_image || p.to_y)
            tile_origin(p, t, h0, w0);
        int pix0[4];   // halo pixel of my pixel slots at tap (0, 0); empty slots read pixel npx - 1
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int pp = min(pq * 4 + q, npx - 1);
            pix0[q] = (pp / p.b) * p.s * p.bin + (pp % p.b) * p.s;
        }
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                acc[i][j] = 0.0f;
        for (int ci0 = 0; ci0 < p.Cin; ci0 += cmax) {
            const int cc = min(cmax, p.Cin - ci0);
            __syncthreads();
            // input halo: a warp per pixel row, lanes over channels.  float32
            // images: 4-byte asynchronous copies (zero-filled padding), waited
            // for together with the weights below, then the GroupNorm affine +
            // SiLU in place
            const bool async_x = p.dtype == SIGE_F32 && p.from_image;
            if (async_x) {
                const float *xg = reinterpret_cast<const float *>(p.src);
#pragma unroll 1
                for (int pix = warp; pix < npix; pix += nwarp) {
                    const int hh = pix / p.bin, ww = pix - hh * p.bin;
                    const int y = h0 * p.s - p.pad + hh, x = w0 * p.s - p.pad + ww;
                    const bool in = y >= 0 && y < p.H && x >= 0 && x < p.W;
                    const float *row = xg + (in ? (((int64_t)n * p.H + y) * p.W + x) * p.Cin + ci0 : 0);
#pragma unroll 1
                    for (int ci = lane; ci < cc; ci += 32)
                        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(
                                         static_cast<uint32_t>(__cvta_generic_to_shared(sx + pix * cc + ci))),
                                     "l"(row + (in ? ci : 0)), "r"(in ? 4 : 0)
                                     : "memory");
                }
            } else
#pragma unroll 1
            for (int pix = warp; pix < npix; pix += nwarp) {
                const int hh = pix / p.bin, ww = pix - hh * p.bin;
#pragma unroll 1
                for (int ci = lane; ci < cc; ci += 32) {
                    float xv = 0.0f;
                    if (p.from_image) {
                        const int y = h0 * p.s - p.pad + hh, x = w0 * p.s - p.pad + ww;
                        if (y >= 0 && y < p.H && x >= 0 && x < p.W) {
                            xv = ldg_elem(p.src, (((int64_t)n * p.H + y) * p.W + x) * p.Cin + ci0 + ci, p.dtype);
                            if (xform) {   // padding stays zero
                                xv = transform1(xv, p.gsc ? p.gsc + (int64_t)n * p.Cin : nullptr,
                                                p.gsc ? p.gsh + (int64_t)n * p.Cin : nullptr, ci0 + ci, p.silu);
                                if (p.dtype == SIGE_BF16)
                                    xv = __bfloat162float(__float2bfloat16_rn(xv));
                            }
                        }
                    } else {
                        xv = ldg_elem(p.src, (((int64_t)t * p.N + n) * npix + pix) * p.Cin + ci0 + ci, p.dtype);
                    }
                    sx[pix * cc + ci] = xv;
                }
            }
            // weights: a warp per (output channel, tap) row, lanes over input
            // channels (contiguous in [C_out][k][k][C_in]).  float32: 4-byte
            // asynchronous copies, all of the chunk in flight at once; bf16
            // (converted on the way): kStageBatch rows in flight per warp.
            const int nrow = kS16Cout * taps;
            if (p.dtype == SIGE_F32) {
                // (row = col * taps + tap, stepped without a division: the
                // issue loop, not the copies, bounded this staging)
                const float *wg = reinterpret_cast<const float *>(p.w);
                int col = warp / taps, tap = warp - col * taps;
#pragma unroll 1
                for (int row = warp; row < nrow; row += nwarp) {
                    const int o2 = cog * kS16Cout + col;
                    const float *src = wg + ((int64_t)o2 * taps + tap) * p.Cin + ci0;
                    float *dst = sw + tap * cc * kS16WStride + col;
#pragma unroll 1
                    for (int ci = lane; ci < cc; ci += 32) {
                        if (o2 < p.Cout)
                            asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(
                                             static_cast<uint32_t>(__cvta_generic_to_shared(dst + ci * kS16WStride))),
                                         "l"(src + ci)
                                         : "memory");
                        else
                            dst[ci * kS16WStride] = 0.0f;
                    }
                    tap += nwarp;
                    while (tap >= taps) {
                        tap -= taps;
                        ++col;
                    }
                }
            } else
#pragma unroll 1
            for (int r0 = warp; r0 < nrow; r0 += nwarp * kStageBatch) {
#pragma unroll 1
                for (int e = 0; e < cc; e += 32) {
                    const int ci = e + lane;
                    float v[kStageBatch];
#pragma unroll
                    for (int k = 0; k < kStageBatch; ++k) {
                        v[k] = 0.0f;
                        const int row = r0 + k * nwarp;
                        if (row >= nrow || ci >= cc)
                            continue;
                        const int col = row / taps, tap = row - col * taps;
                        const int o2 = cog * kS16Cout + col;
                        if (o2 < p.Cout)
                            v[k] = ldg_elem(p.w, ((int64_t)o2 * taps + tap) * p.Cin + ci0 + ci, p.dtype);
                    }
#pragma unroll
                    for (int k = 0; k < kStageBatch; ++k) {
                        const int row = r0 + k * nwarp;
                        if (row >= nrow || ci >= cc)
                            continue;
                        const int col = row / taps, tap = row - col * taps;
                        sw[(tap * cc + ci) * kS16WStride + col] = v[k];
                    }
                }
            }
            asm volatile("cp.async.wait_all;" ::: "memory");
            if (async_x && xform) {
                __syncthreads();
#pragma unroll 1
                for (int pix = warp; pix < npix; pix += nwarp) {
                    const int hh = pix / p.bin, ww = pix - hh * p.bin;
                    const int y = h0 * p.s - p.pad + hh, x = w0 * p.s - p.pad + ww;
                    if (y < 0 || y >= p.H || x < 0 || x >= p.W)
                        continue;   // padding stays zero
#pragma unroll 1
                    for (int ci = lane; ci < cc; ci += 32)
                        sx[pix * cc + ci] = transform1(sx[pix * cc + ci], p.gsc ? p.gsc + (int64_t)n * p.Cin : nullptr,
                                                       p.gsc ? p.gsh + (int64_t)n * p.Cin : nullptr, ci0 + ci, p.silu);
                }
            }
            __syncthreads();
#pragma unroll 1
            for (int r = 0; r < p.k; ++r)
#pragma unroll 1
                for (int c = 0; c < p.k; ++c) {
                    const float *x0 = sx + (pix0[0] + r * p.bin + c) * cc;
                    const float *x1 = sx + (pix0[1] + r * p.bin + c) * cc;
                    const float *x2 = sx + (pix0[2] + r * p.bin + c) * cc;
                    const float *x3 = sx + (pix0[3] + r * p.bin + c) * cc;
                    const float *wr = sw + (r * p.k + c) * cc * kS16WStride + cq * 4;
#pragma unroll 2
                    for (int ci = kg; ci < cc; ci += kS16Kg) {
                        const float4 w4 = *reinterpret_cast<const float4 *>(wr + ci * kS16WStride);
                        const float xv[4] = {x0[ci], x1[ci], x2[ci], x3[ci]};
                        const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i)
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                acc[i][j] = fmaf(wv[i], xv[j], acc[i][j]);
                    }
                }
        }
        // sum the K groups in a fixed order and write the unit's outputs
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 4; ++j)
            *reinterpret_cast<float4 *>(red + ((kg * 16 + pq * 4 + j) * kS16Cout) + cq * 4) =
                make_float4(acc[0][j], acc[1][j], acc[2][j], acc[3][j]);
        __syncthreads();
#pragma unroll
        for (int m = 0; m < (16 * kS16Cout + kS16Threads - 1) / kS16Threads; ++m) {
            const int oi = tid + kS16Threads * m;       // [16 px][kS16Cout co]
            const int col = oi & (kS16Cout - 1), px = oi / kS16Cout;
            const int o = cog * kS16Cout + col;
            if (px >= npx || o >= p.Cout)
                continue;
            float a = 0.0f;
#pragma unroll
            for (int g = 0; g < kS16Kg; ++g)
                a += red[(g * 16 + px) * kS16Cout + col];
            const int i = px / p.b, j = px % p.b;
            if (p.to_y) {
                const int yo = h0 + i, xo = w0 + j;
                if (yo < p.Ho && xo < p.Wo)
                    store_out1(p.y, (((int64_t)n * p.Ho + yo) * p.Wo + xo) * p.Cout + o, p.dtype, a,
                               p.bias ? __ldg(p.bias + o) : 0.0f, p.residual);
            } else {
                p.out_blocks[(((int64_t)t * p.N + n) * npx + px) * p.Cout + o] = a;
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

static int launch_conv_simt16(ConvParams p, cudaStream_t stream)
{
    const int npix = p.bin * p.bin, taps = p.k * p.k;
    // one chunk of channels: halo block + weights, within 96 KB (the K-group
    // sums of the end reuse the same space)
    const int per_ci = npix + taps * kS16WStride;
    p.ci_chunk = std::min(p.Cin, (kS16SmemFloats - 4) / per_ci);
    if (p.ci_chunk < 1)
        return SIGE_ERR_UNSUPPORTED;
    const size_t smem = (size_t)kS16SmemFloats * sizeof(float);
    static std::atomic<int> attr_done[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(k_conv_simt16, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return SIGE_ERR_CUDA;
        attr_done[dev].store(1, std::memory_order_release);
    }
    const int ncog = (p.Cout + kS16Cout - 1) / kS16Cout;
    const int64_t max_units = (int64_t)(p.dense ? p.tiles_total : p.cap) * p.N * ncog;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(max_units, (int64_t)device_sm_count() * 4));
    prefer_max_shared(k_conv_simt16);
    k_conv_simt16<<<grid, kS16Threads, smem, stream>>>(p);
    count_launch();
    return launch_check();
}

int launch_conv_simt(ConvParams p, cudaStream_t stream)
{
    const int npx = p.b * p.b;
    if (npx <= 16) {
        const int st = launch_conv_simt16(p, stream);
        if (st != SIGE_ERR_UNSUPPORTED)
            return st;
    }
    int pg = std::max(kSimtThreads / std::min(kSimtThreads, pow2_ceil(p.Cout)), pow2_ceil((npx + kSimtMaxQ - 1) / kSimtMaxQ));
    if (pg > kSimtThreads)
        return SIGE_ERR_UNSUPPORTED;
    p.pg = pg;
    p.cob = kSimtThreads / pg;
    const int bin2 = p.bin * p.bin;
    // per input channel of a chunk: its halo block and the group's weights
    const int per_ci = bin2 + p.k * p.k * (p.cob + 1);
    p.ci_chunk = std::min(p.Cin, kSimtSmemFloats / per_ci);
    if (p.ci_chunk < 1)
        return SIGE_ERR_UNSUPPORTED;
    const size_t smem = (size_t)per_ci * p.ci_chunk * sizeof(float);
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
