// Gather of halo'd active blocks and scatter of output blocks into the cached
// output (SIGE project page, "Overview": gather the active blocks from the
// edited activation, stack them along the batch axis, and scatter the output
// blocks back into F_l(A_original)).  Plus the GroupNorm statistics of the
// cached original activation, folded into a per-channel affine (a cluster of
// 8 CTAs per image that combine their partial sums through distributed shared
// memory, or one CTA per (image, group) for the shapes the cluster path does
// not take), and the restore of listed tiles from a source tensor between
// sequential edits.
#include <atomic>
#include <algorithm>
#include <cstring>

#include "sige_internal.cuh"
#include "transform.cuh"

namespace sige {

// ------------------------------------------------------------------ gather

struct GatherParams {
    const uint8_t *x;
    int32_t N, H, W, C, dtype;
    int32_t s, pad, bin;
    const int32_t *idx;
    const int32_t *count;
    int32_t cap;
    const float *gsc, *gsh;
    int32_t silu;
    uint8_t *blocks;
    int32_t vpp;  // 16-byte vectors per pixel
    int32_t fast; // every vector index fits 32 bits: decompose it by the divisors below
    UDiv dvpp, dbin, dN;
};

__global__ void __launch_bounds__(256) k_gather(const __grid_constant__ GatherParams p)
{
    const int64_t ntile = min(__ldg(p.count), p.cap);
    const int64_t per_tile = (int64_t)p.N * p.bin * p.bin * p.vpp;
    const int64_t total = ntile * per_tile;
    const int esz = p.dtype == SIGE_BF16 ? 2 : 4;
    const int epv = 16 / esz;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < total;
         v += (int64_t)gridDim.x * blockDim.x) {
        int cv, ww, hh, n, t;
        if (p.fast) {
            // (multiply-high divisions: a 64-bit division per index bounded this loop)
            uint32_t r = (uint32_t)v, q = udiv(r, p.dvpp);
            cv = (int)(r - q * (uint32_t)p.vpp);
            r = q;
            q = udiv(r, p.dbin);
            ww = (int)(r - q * (uint32_t)p.bin);
            r = q;
            q = udiv(r, p.dbin);
            hh = (int)(r - q * (uint32_t)p.bin);
            r = q;
            q = p.N == 1 ? r : udiv(r, p.dN);
            n = (int)(r - q * (uint32_t)p.N);
            t = (int)q;
        } else {
            cv = (int)(v % p.vpp);
            int64_t pix = v / p.vpp;
            ww = (int)(pix % p.bin);
            pix /= p.bin;
            hh = (int)(pix % p.bin);
            pix /= p.bin;
            n = (int)(pix % p.N);
            t = (int)(pix / p.N);
        }
        const int2 o = __ldg(reinterpret_cast<const int2 *>(p.idx) + t);
        const int y = o.x * p.s - p.pad + hh, x = o.y * p.s - p.pad + ww;
        uint4 out = make_uint4(0, 0, 0, 0);
        if (y >= 0 && y < p.H && x >= 0 && x < p.W) {
            const uint4 in = ld_nc16(p.x + ((((int64_t)n * p.H + y) * p.W + x) * p.C) * esz + cv * 16);
            const int c0 = cv * epv;
            out = transform16(in, p.dtype, p.gsc ? p.gsc + (int64_t)n * p.C + c0 : nullptr,
                              p.gsc ? p.gsh + (int64_t)n * p.C + c0 : nullptr, p.silu);
        }
        reinterpret_cast<uint4 *>(p.blocks)[v] = out;
    }
}

// ------------------------------------------------------------------ scatter

struct ScatterParams {
    const float *out;
    int32_t N, Ho, Wo, Co, dtype, b;
    const int32_t *idx;
    const int32_t *count;
    int32_t cap;
    const float *bias;
    const uint8_t *residual;
    uint8_t *y;
    int32_t fast; // every vector index fits 32 bits: decompose it by the divisors below
    UDiv dc4n, db, dN;
};

__global__ void __launch_bounds__(256) k_scatter(const __grid_constant__ ScatterParams p)
{
    const int64_t ntile = min(__ldg(p.count), p.cap);
    const int c4n = p.Co / 4;
    const int64_t total = ntile * p.N * p.b * p.b * c4n;
    for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < total;
         v += (int64_t)gridDim.x * blockDim.x) {
        int c4, j, i, n, t;
        if (p.fast) {
            uint32_t r = (uint32_t)v, q = udiv(r, p.dc4n);
            c4 = (int)(r - q * (uint32_t)c4n);
            r = q;
            q = udiv(r, p.db);
            j = (int)(r - q * (uint32_t)p.b);
            r = q;
            q = udiv(r, p.db);
            i = (int)(r - q * (uint32_t)p.b);
            r = q;
            q = p.N == 1 ? r : udiv(r, p.dN);
            n = (int)(r - q * (uint32_t)p.N);
            t = (int)q;
        } else {
            c4 = (int)(v % c4n);
            int64_t pix = v / c4n;
            j = (int)(pix % p.b);
            pix /= p.b;
            i = (int)(pix % p.b);
            pix /= p.b;
            n = (int)(pix % p.N);
            t = (int)(pix / p.N);
        }
        const int2 o = __ldg(reinterpret_cast<const int2 *>(p.idx) + t);
        const int yo = o.x + i, xo = o.y + j;
        if (yo >= p.Ho || xo >= p.Wo)
            continue;
        float4 a = __ldg(reinterpret_cast<const float4 *>(p.out) + v);
        const int c = c4 * 4;
        const int64_t e = (((int64_t)n * p.Ho + yo) * p.Wo + xo) * p.Co + c;
        store_out4(p.y, e, p.dtype, a, p.bias ? p.bias + c : nullptr, p.residual);
    }
}

// ------------------------------------------------------------------ GroupNorm affine

struct GnParams {
    const uint8_t *x;
    int32_t N, HW, C, dtype, groups;
    const float *gamma, *beta;
    float eps;
    float *scale, *shift;
};

__device__ __forceinline__ double block_sum_d(double v, double *sh)
{
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0)
        sh[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < (int)(blockDim.x >> 5) ? sh[lane] : 0.0;
        for (int o = 16; o > 0; o >>= 1)
            v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
        if (lane == 0)
            sh[32] = v;
    }
    __syncthreads();
    double r = sh[32];
    __syncthreads();
    return r;
}

__device__ __forceinline__ float gn_elem(const GnParams &p, int64_t i)
{
    if (p.dtype == SIGE_BF16)
        return __uint_as_float((uint32_t)(reinterpret_cast<const uint16_t *>(p.x)[i]) << 16);
    return reinterpret_cast<const float *>(p.x)[i];
}

// One CTA per (n, group): two passes in double, fixed reduction order.
__global__ void __launch_bounds__(1024) k_gn_affine(const __grid_constant__ GnParams p)
{
    __shared__ double sh[33];
    const int n = blockIdx.x / p.groups, g = blockIdx.x % p.groups;
    const int cg = p.C / p.groups;
    const int64_t cnt = (int64_t)p.HW * cg;
    const int64_t base = (int64_t)n * p.HW * p.C + (int64_t)g * cg;
    double s = 0.0;
    for (int64_t k = threadIdx.x; k < cnt; k += blockDim.x)
        s += gn_elem(p, base + (k / cg) * p.C + (k % cg));
    const double mean = block_sum_d(s, sh) / (double)cnt;
    double v = 0.0;
    for (int64_t k = threadIdx.x; k < cnt; k += blockDim.x) {
        double d = gn_elem(p, base + (k / cg) * p.C + (k % cg)) - mean;
        v += d * d;
    }
    const double var = block_sum_d(v, sh) / (double)cnt;
    for (int c = threadIdx.x; c < cg; c += blockDim.x) {
        const int ch = g * cg + c;
        const double sc = (double)p.gamma[ch] / sqrt(var + (double)p.eps);
        p.scale[(int64_t)n * p.C + ch] = (float)sc;
        p.shift[(int64_t)n * p.C + ch] = (float)((double)p.beta[ch] - mean * sc);
    }
}

// Tile restore for sequential edits: dst[n][h0+i][w0+j][:] = src[...] for the
// in-image pixels of every listed tile.  One thread per 16-byte vector of a
// tile row (NHWC: a tile row is b * C contiguous elements), or per element when
// rows are not made of whole vectors.
struct RestoreParams {
    const uint8_t *src;
    uint8_t *dst;
    int32_t N, H, W, row_bytes;  // row_bytes = C * element size
    int32_t b, vec;              // vec: 1 = 16-byte vectors, 0 = bytes
    const int32_t *idx, *count;
    int32_t cap;
};

__global__ void __launch_bounds__(256) k_restore(const __grid_constant__ RestoreParams p)
{
    const int ntiles = min(__ldg(p.count), p.cap);
    const int unit = p.vec ? 16 : 1;
    const int per_px = p.row_bytes / unit;          // units per pixel
    const int64_t per_tile = (int64_t)p.N * p.b * p.b * per_px;
    const int64_t total = per_tile * ntiles;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int t = (int)(e / per_tile);
        int64_t r = e - (int64_t)t * per_tile;
        const int v = (int)(r % per_px);
        r /= per_px;
        const int j = (int)(r % p.b);
        r /= p.b;
        const int i = (int)(r % p.b);
        const int n = (int)(r / p.b);
        const int2 o = __ldg(reinterpret_cast<const int2 *>(p.idx) + t);
        const int y = o.x + i, x = o.y + j;
        if (y >= p.H || x >= p.W)
            continue;
        const int64_t off = (((int64_t)n * p.H + y) * p.W + x) * p.row_bytes + (int64_t)v * unit;
        if (p.vec)
            *reinterpret_cast<uint4 *>(p.dst + off) = __ldg(reinterpret_cast<const uint4 *>(p.src + off));
        else
            p.dst[off] = __ldg(p.src + off);
    }
}

// GroupNorm statistics of one image on a cluster of kGnCluster CTAs.  Each CTA
// streams a contiguous range of pixels with 16-byte loads; a thread keeps, for
// the channels of its vector column, the sums of (x - K_c) and (x - K_c)^2 in
// double, with K_c the image's first pixel (the shift keeps the one-pass
// variance exact to double rounding).  Partial sums meet in shared memory in
// a fixed order, rank 0 adds the ranks' partials through distributed shared
// memory (rank order) and turns each group's sums into scale / shift.
constexpr int kGnCluster = 8;
constexpr int kGnThreads = 512;
constexpr int kGnBatch = 8;      // independent 16-byte loads in flight per thread

__device__ __forceinline__ float gn_vec_elem(uint4 v, int k, int dtype)
{
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    if (dtype == SIGE_BF16)
        return (k & 1) ? bf16_hi(w[k >> 1]) : bf16_lo(w[k >> 1]);
    return __uint_as_float(w[k]);
}

__global__ void __cluster_dims__(kGnCluster, 1, 1) __launch_bounds__(kGnThreads)
    k_gn_stats_cluster(const __grid_constant__ GnParams p)
{
    extern __shared__ __align__(16) double gsm[];
    const int C = p.C, esz = p.dtype == SIGE_BF16 ? 2 : 4, epv = 16 / esz;
    const int vpp = C / epv;                       // vectors per pixel
    const int rows = kGnThreads / vpp;             // pixels per pass
    double *part = gsm;                            // [C][2] this CTA's sums
    double *red = gsm + 2 * C;                     // [rows][C][2]
    uint32_t rank;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    const int n = blockIdx.x / kGnCluster;
    const int t = threadIdx.x, v = t % vpp, r0 = t / vpp;
    const uint8_t *img = p.x + (size_t)n * p.HW * C * esz;
    const int64_t p0 = (int64_t)p.HW * rank / kGnCluster, p1 = (int64_t)p.HW * (rank + 1) / kGnCluster;
    double s1[8], s2[8];
    float K[8];
    const uint4 k4 = __ldg(reinterpret_cast<const uint4 *>(img) + v);   // pixel 0 of the image
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        s1[k] = 0.0;
        s2[k] = 0.0;
        K[k] = k < epv ? gn_vec_elem(k4, k, p.dtype) : 0.0f;
    }
    if (r0 < rows) {
#pragma unroll 1
        for (int64_t px0 = p0 + r0; px0 < p1; px0 += (int64_t)rows * kGnBatch) {
            uint4 x4[kGnBatch];
#pragma unroll
            for (int u = 0; u < kGnBatch; ++u) {
                const int64_t px = px0 + (int64_t)u * rows;
                x4[u] = px < p1 ? __ldg(reinterpret_cast<const uint4 *>(img + (size_t)px * C * esz) + v) : k4;
            }
#pragma unroll
            for (int u = 0; u < kGnBatch; ++u)
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    if (k >= epv)
                        break;
                    // past the range: the shift itself, which adds nothing
                    const double d = (double)gn_vec_elem(x4[u], k, p.dtype) - (double)K[k];
                    s1[k] += d;
                    s2[k] = fma(d, d, s2[k]);
                }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
            if (k < epv) {
                red[((size_t)r0 * C + v * epv + k) * 2] = s1[k];
                red[((size_t)r0 * C + v * epv + k) * 2 + 1] = s2[k];
            }
    }
    __syncthreads();
    for (int c = t; c < C; c += kGnThreads) {      // fixed row order
        double a = 0.0, b = 0.0;
        for (int rr = 0; rr < rows; ++rr) {
            a += red[((size_t)rr * C + c) * 2];
            b += red[((size_t)rr * C + c) * 2 + 1];
        }
        part[2 * c] = a;
        part[2 * c + 1] = b;
    }
    // every rank's partials are complete before rank 0 reads them
    asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (rank == 0) {
        const uint32_t local = static_cast<uint32_t>(__cvta_generic_to_shared(part));
        const int cg = C / p.groups;
        uint32_t remote[kGnCluster];
#pragma unroll
        for (int q = 0; q < kGnCluster; ++q)
            asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote[q]) : "r"(local), "r"(q));
        for (int g = t; g < p.groups; g += kGnThreads) {
            // channel sums over the ranks in rank order; two passes over the
            // group's channels: the mean, then the centred second moment
            const double cnt = (double)p.HW * cg;
            double sx = 0.0;
            for (int j = 0; j < cg; ++j) {
                const int c = g * cg + j;
                double a = 0.0;
#pragma unroll
                for (int q = 0; q < kGnCluster; ++q) {
                    double e;
                    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(e) : "r"(remote[q] + (uint32_t)(c * 16)));
                    a += e;
                }
                const double Kc = (double)gn_vec_elem(__ldg(reinterpret_cast<const uint4 *>(img) + c / epv),
                                                      c % epv, p.dtype);
                sx += a + (double)p.HW * Kc;
            }
            const double mean = sx / cnt;
            double sxx = 0.0;
            for (int j = 0; j < cg; ++j) {
                const int c = g * cg + j;
                double a = 0.0, bb = 0.0;
#pragma unroll
                for (int q = 0; q < kGnCluster; ++q) {
                    double e, f;
                    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(e) : "r"(remote[q] + (uint32_t)(c * 16)));
                    asm volatile("ld.shared::cluster.f64 %0, [%1];" : "=d"(f) : "r"(remote[q] + (uint32_t)(c * 16 + 8)));
                    a += e;
                    bb += f;
                }
                const double Kc = (double)gn_vec_elem(__ldg(reinterpret_cast<const uint4 *>(img) + c / epv),
                                                      c % epv, p.dtype);
                const double dk = Kc - mean;
                sxx += bb + 2.0 * dk * a + (double)p.HW * dk * dk;
            }
            const double var = sxx / cnt;
            for (int j = 0; j < cg; ++j) {
                const int c = g * cg + j;
                const double sc = (double)p.gamma[c] / sqrt(var + (double)p.eps);
                p.scale[(int64_t)n * C + c] = (float)sc;
                p.shift[(int64_t)n * C + c] = (float)((double)p.beta[c] - mean * sc);
            }
        }
    }
    // rank 0 has read every rank's shared memory before any CTA leaves
    asm volatile("barrier.cluster.arrive.release.aligned;\n barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

static int grid_for(int64_t work, int threads)
{
    int64_t g = (work + threads - 1) / threads;
    return (int)std::max<int64_t>(1, std::min<int64_t>(g, (int64_t)device_sm_count() * 8));
}

} // namespace sige

using namespace sige;

static bool conv_desc_ok(const sige_conv_desc *cd)
{
    return cd && cd->kernel >= 1 && cd->stride >= 1 && cd->pad >= 0 && cd->pad < cd->kernel &&
           cd->c_in >= 1 && cd->c_out >= 1 && cd->block >= 1 && cd->block <= 64;
}

extern "C" int sige_gather(const void *x, const sige_tensor_desc *xd, const sige_conv_desc *cd,
                           const int32_t *idx, const int32_t *count, int32_t capacity,
                           const float *gn_scale, const float *gn_shift, int32_t silu, void *blocks,
                           sige_stream_t stream)
{
    if (!x || !xd || !idx || !count || !blocks || capacity < 0 || !conv_desc_ok(cd))
        return SIGE_ERR_INVALID_ARG;
    if ((gn_scale == nullptr) != (gn_shift == nullptr))
        return SIGE_ERR_INVALID_ARG;
    if (xd->n < 1 || xd->h < 1 || xd->w < 1 || xd->c != cd->c_in)
        return SIGE_ERR_INVALID_ARG;
    if (xd->layout != SIGE_NHWC || (xd->dtype != SIGE_F32 && xd->dtype != SIGE_BF16))
        return SIGE_ERR_UNSUPPORTED;
    const int esz = xd->dtype == SIGE_BF16 ? 2 : 4;
    if ((xd->c * esz) % 16 || (reinterpret_cast<uintptr_t>(x) & 15) || (reinterpret_cast<uintptr_t>(blocks) & 15))
        return SIGE_ERR_UNSUPPORTED;
    if (capacity == 0)
        return SIGE_OK;
    GatherParams p{};
    p.x = static_cast<const uint8_t *>(x);
    p.N = xd->n; p.H = xd->h; p.W = xd->w; p.C = xd->c; p.dtype = xd->dtype;
    p.s = cd->stride; p.pad = cd->pad;
    p.bin = (cd->block - 1) * cd->stride + cd->kernel;
    p.idx = idx; p.count = count; p.cap = capacity;
    p.gsc = gn_scale; p.gsh = gn_shift; p.silu = silu ? 1 : 0;
    p.blocks = static_cast<uint8_t *>(blocks);
    p.vpp = xd->c * esz / 16;
    const int64_t work = (int64_t)capacity * p.N * p.bin * p.bin * p.vpp;
    p.fast = work <= 0xFFFFFFFFll ? 1 : 0;
    p.dvpp = udiv_make((uint32_t)p.vpp);
    p.dbin = udiv_make((uint32_t)p.bin);
    p.dN = udiv_make((uint32_t)p.N);
    prefer_max_shared(k_gather);
    k_gather<<<grid_for(work, 256), 256, 0, (cudaStream_t)stream>>>(p);
    count_launch();
    return launch_check();
}

extern "C" int sige_scatter(const float *out_blocks, const sige_conv_desc *cd, const int32_t *idx,
                            const int32_t *count, int32_t capacity, const float *bias,
                            const void *residual, void *y, const sige_tensor_desc *yd,
                            sige_stream_t stream)
{
    if (!out_blocks || !idx || !count || !y || !yd || capacity < 0 || !conv_desc_ok(cd))
        return SIGE_ERR_INVALID_ARG;
    if (yd->c != cd->c_out || yd->n < 1 || yd->h < 1 || yd->w < 1)
        return SIGE_ERR_INVALID_ARG;
    if (yd->layout != SIGE_NHWC || (yd->dtype != SIGE_F32 && yd->dtype != SIGE_BF16) || cd->c_out % 4)
        return SIGE_ERR_UNSUPPORTED;
    if ((reinterpret_cast<uintptr_t>(out_blocks) & 15) || (reinterpret_cast<uintptr_t>(y) & 15) ||
        (reinterpret_cast<uintptr_t>(residual) & 15))
        return SIGE_ERR_UNSUPPORTED;
    if (capacity == 0)
        return SIGE_OK;
    ScatterParams p{};
    p.out = out_blocks;
    p.N = yd->n; p.Ho = yd->h; p.Wo = yd->w; p.Co = yd->c; p.dtype = yd->dtype; p.b = cd->block;
    p.idx = idx; p.count = count; p.cap = capacity;
    p.bias = bias;
    p.residual = static_cast<const uint8_t *>(residual);
    p.y = static_cast<uint8_t *>(y);
    const int64_t work = (int64_t)capacity * p.N * p.b * p.b * (p.Co / 4);
    p.fast = work <= 0xFFFFFFFFll ? 1 : 0;
    p.dc4n = udiv_make((uint32_t)(p.Co / 4));
    p.db = udiv_make((uint32_t)p.b);
    p.dN = udiv_make((uint32_t)p.N);
    prefer_max_shared(k_scatter);
    k_scatter<<<grid_for(work, 256), 256, 0, (cudaStream_t)stream>>>(p);
    count_launch();
    return launch_check();
}

extern "C" int sige_groupnorm_affine(const void *x, const sige_tensor_desc *xd, int32_t groups,
                                     const float *gamma, const float *beta, float eps, float *scale,
                                     float *shift, sige_stream_t stream)
{
    if (!x || !xd || !gamma || !beta || !scale || !shift || groups < 1 || !(eps >= 0.0f))
        return SIGE_ERR_INVALID_ARG;
    if (xd->n < 1 || xd->h < 1 || xd->w < 1 || xd->c < 1 || xd->c % groups)
        return SIGE_ERR_INVALID_ARG;
    if (xd->layout != SIGE_NHWC || (xd->dtype != SIGE_F32 && xd->dtype != SIGE_BF16))
        return SIGE_ERR_UNSUPPORTED;
    GnParams p{};
    p.x = static_cast<const uint8_t *>(x);
    p.N = xd->n; p.HW = xd->h * xd->w; p.C = xd->c; p.dtype = xd->dtype; p.groups = groups;
    p.gamma = gamma; p.beta = beta; p.eps = eps; p.scale = scale; p.shift = shift;
    // cluster path: whole 16-byte vectors per pixel, at most 256 of them, at
    // most 64 channels per group, 16-byte aligned input
    const int esz = xd->dtype == SIGE_BF16 ? 2 : 4;
    const int vpp = (xd->c * esz) % 16 == 0 ? xd->c * esz / 16 : 0;
    if (vpp >= 1 && vpp <= kGnThreads && xd->c / groups <= 64 && (reinterpret_cast<uintptr_t>(x) & 15) == 0) {
        const int rows = kGnThreads / vpp;
        const size_t smem = (size_t)(2 * xd->c + (size_t)rows * xd->c * 2) * sizeof(double);
        static std::atomic<int> attr_done[64];
        int dev = 0;
        cudaGetDevice(&dev);
        bool ok = smem <= 200 * 1024;
        if (ok && dev >= 0 && dev < 64 && !attr_done[dev].load(std::memory_order_acquire)) {
            ok = cudaFuncSetAttribute(k_gn_stats_cluster, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      200 * 1024) == cudaSuccess;
            if (ok)
                attr_done[dev].store(1, std::memory_order_release);
            else
                cudaGetLastError();
        }
        if (ok) {
            k_gn_stats_cluster<<<xd->n * kGnCluster, kGnThreads, smem, (cudaStream_t)stream>>>(p);
            if (cudaGetLastError() == cudaSuccess) {
                count_launch();
                return SIGE_OK;
            }
        }
    }
    prefer_max_shared(k_gn_affine);
    k_gn_affine<<<xd->n * groups, 1024, 0, (cudaStream_t)stream>>>(p);
    count_launch();
    return launch_check();
}

extern "C" int sige_restore_tiles(const void *src, void *dst, const sige_tensor_desc *d, int32_t block,
                                  const int32_t *idx, const int32_t *count, int32_t capacity, sige_stream_t stream)
{
    if (!src || !dst || !d || !idx || !count || capacity < 0 || block < 1)
        return SIGE_ERR_INVALID_ARG;
    if (d->n < 1 || d->h < 1 || d->w < 1 || d->c < 1)
        return SIGE_ERR_INVALID_ARG;
    if (d->layout != SIGE_NHWC || (d->dtype != SIGE_U8 && d->dtype != SIGE_F32 && d->dtype != SIGE_BF16))
        return SIGE_ERR_UNSUPPORTED;
    if (capacity == 0)
        return SIGE_OK;
    const int esz = d->dtype == SIGE_U8 ? 1 : d->dtype == SIGE_BF16 ? 2 : 4;
    RestoreParams p{};
    p.src = static_cast<const uint8_t *>(src);
    p.dst = static_cast<uint8_t *>(dst);
    p.N = d->n; p.H = d->h; p.W = d->w;
    p.row_bytes = d->c * esz;
    p.b = block;
    p.vec = (p.row_bytes % 16 == 0 && ((reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst)) & 15) == 0)
                ? 1 : 0;
    p.idx = idx; p.count = count; p.cap = capacity;
    const int64_t work = (int64_t)capacity * p.N * block * block * (p.row_bytes / (p.vec ? 16 : 1));
    k_restore<<<grid_for(work, 256), 256, 0, (cudaStream_t)stream>>>(p);
    count_launch();
    return launch_check();
}

// ------------------------------------------------------------------ tile read-back

// Staging layout: [0, 16) the count; [16, 16 + 8 cap) the list; then, 16-byte
// aligned, the packed tiles [tile][n][i][j][C] (b x b pixels each).
static inline size_t dl_tiles_offset(int32_t capacity) { return (16 + (size_t)capacity * 8 + 15) & ~(size_t)15; }

struct PackParams {
    const uint8_t *y;
    int32_t N, H, W, vpp, b;    // vpp: 16-byte vectors per pixel
    const int32_t *idx, *count;
    int32_t cap;
    uint8_t *staging;
    size_t tiles_off;
    UDiv dvpp, db, dN;
};

__global__ void __launch_bounds__(256) k_pack_tiles(const __grid_constant__ PackParams p)
{
    const int ntile = max(0, min(__ldg(p.count), p.cap));
    if (blockIdx.x == 0) {
        if (threadIdx.x == 0)
            *reinterpret_cast<int32_t *>(p.staging) = ntile;
        for (int t = threadIdx.x; t < ntile; t += blockDim.x)
            reinterpret_cast<int2 *>(p.staging + 16)[t] = __ldg(reinterpret_cast<const int2 *>(p.idx) + t);
    }
    const uint32_t total = (uint32_t)ntile * (uint32_t)p.N * (uint32_t)(p.b * p.b) * (uint32_t)p.vpp;
    uint4 *dst = reinterpret_cast<uint4 *>(p.staging + p.tiles_off);
    for (uint32_t v = blockIdx.x * blockDim.x + threadIdx.x; v < total; v += gridDim.x * blockDim.x) {
        uint32_t q = udiv(v, p.dvpp);
        const uint32_t cv = v - q * (uint32_t)p.vpp;
        uint32_t r = q;
        q = udiv(r, p.db);
        const int j = (int)(r - q * (uint32_t)p.b);
        r = q;
        q = udiv(r, p.db);
        const int i = (int)(r - q * (uint32_t)p.b);
        r = q;
        q = p.N == 1 ? r : udiv(r, p.dN);
        const int n = (int)(r - q * (uint32_t)p.N);
        const int2 o = __ldg(reinterpret_cast<const int2 *>(p.idx) + q);
        const int yy = o.x + i, xx = o.y + j;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (yy < p.H && xx < p.W)
            val = ld_nc16(p.y + ((((int64_t)n * p.H + yy) * p.W + xx) * p.vpp + cv) * 16);
        dst[v] = val;
    }
}

static int dl_esz(int dtype) { return dtype == SIGE_U8 ? 1 : dtype == SIGE_BF16 ? 2 : dtype == SIGE_F32 ? 4 : 0; }

extern "C" size_t sige_download_tiles_bytes(const sige_tensor_desc *yd, int32_t block, int32_t capacity)
{
    if (!yd || block < 1 || capacity < 0 || yd->n < 1 || yd->c < 1 || !dl_esz(yd->dtype))
        return 0;
    const size_t tile = (size_t)yd->n * block * block * yd->c * dl_esz(yd->dtype);
    return dl_tiles_offset(capacity) + (size_t)capacity * tile;
}

extern "C" int sige_download_tiles(const void *y, const sige_tensor_desc *yd, int32_t block, const int32_t *idx,
                                   const int32_t *count, int32_t capacity, void *staging, void *host_staging,
                                   void *host_y, sige_stream_t stream)
{
    if (!y || !yd || !idx || !count || !staging || !host_staging || !host_y || block < 1 || capacity < 0)
        return SIGE_ERR_INVALID_ARG;
    if (yd->n < 1 || yd->h < 1 || yd->w < 1 || yd->c < 1)
        return SIGE_ERR_INVALID_ARG;
    const int esz = dl_esz(yd->dtype);
    if (yd->layout != SIGE_NHWC || !esz || ((size_t)yd->c * esz) % 16 ||
        ((reinterpret_cast<uintptr_t>(y) | reinterpret_cast<uintptr_t>(staging)) & 15))
        return SIGE_ERR_UNSUPPORTED;
    if (capacity == 0)
        return SIGE_OK;
    const size_t px_bytes = (size_t)yd->c * esz;
    const size_t tile_bytes = (size_t)yd->n * block * block * px_bytes;
    const int64_t vec_total = (int64_t)capacity * yd->n * block * block * (int64_t)(px_bytes / 16);
    if (vec_total > 0xFFFFFFFFll)
        return SIGE_ERR_UNSUPPORTED;
    PackParams p{};
    p.y = static_cast<const uint8_t *>(y);
    p.N = yd->n; p.H = yd->h; p.W = yd->w;
    p.vpp = (int32_t)(px_bytes / 16);
    p.b = block;
    p.idx = idx; p.count = count; p.cap = capacity;
    p.staging = static_cast<uint8_t *>(staging);
    p.tiles_off = dl_tiles_offset(capacity);
    p.dvpp = udiv_make((uint32_t)p.vpp);
    p.db = udiv_make((uint32_t)block);
    p.dN = udiv_make((uint32_t)p.N);
    const cudaStream_t st = (cudaStream_t)stream;
    k_pack_tiles<<<grid_for(vec_total, 256), 256, 0, st>>>(p);
    count_launch();
    int rc = launch_check();
    if (rc != SIGE_OK)
        return rc;
    // the count and the list, then the packed tiles of that count
    uint8_t *hs = static_cast<uint8_t *>(host_staging);
    if (cudaMemcpyAsync(hs, staging, 16 + (size_t)capacity * 8, cudaMemcpyDeviceToHost, st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return SIGE_ERR_CUDA;
    const int n = std::max(0, std::min(*reinterpret_cast<const int32_t *>(hs), capacity));
    if (n == 0)
        return SIGE_OK;
    if (cudaMemcpyAsync(hs + p.tiles_off, p.staging + p.tiles_off, (size_t)n * tile_bytes, cudaMemcpyDeviceToHost,
                        st) != cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return SIGE_ERR_CUDA;
    // place the rows (clipped at the map's edges)
    const int2 *list = reinterpret_cast<const int2 *>(hs + 16);
    uint8_t *out = static_cast<uint8_t *>(host_y);
    for (int t = 0; t < n; ++t) {
        const int h0 = list[t].x, w0 = list[t].y;
        if (h0 < 0 || w0 < 0 || h0 >= yd->h || w0 >= yd->w)
            continue;
        const int rows = std::min(block, yd->h - h0), cols = std::min(block, yd->w - w0);
        for (int nn = 0; nn < yd->n; ++nn)
            for (int i = 0; i < rows; ++i)
                memcpy(out + ((((size_t)nn * yd->h + h0 + i) * yd->w + w0) * px_bytes),
                       hs + p.tiles_off + (size_t)t * tile_bytes + (((size_t)nn * block + i) * block) * px_bytes,
                       (size_t)cols * px_bytes);
    }
    return SIGE_OK;
}
