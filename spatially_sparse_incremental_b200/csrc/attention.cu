// Attention step of a layer whose unedited query tokens are pruned: for every
// token under the active-tile list, per head, o = softmax(q K^T / sqrt(d_head)) V
// over all keys, written at that token; every other token of o is left as it is.
// (The nubint.ai review of "Efficient Spatially Sparse Inference for
// Conditional GANs and Diffusion Models", "Proposed method": attention layers
// by pruning the query tokens of unedited regions; the mer.dev notes on the
// same paper, abstract: attention layers for Stable Diffusion.)
//
// The projections around this step are sparse 1x1 convolutions on the same
// tile list (the fused conv of this library): q of the active tokens, the
// cached k / v updated at the active tokens (self-attention) or computed once
// from the context (cross-attention), and the output projection with bias and
// residual scattered into the cached output.
//
// Kernel: one CTA per (active tile, batch item, head), persistent over that
// list (the tile count is read on the device).  The CTA stages the tile's b*b
// queries, then walks the keys in chunks of 32 staged in shared memory; a warp
// owns up to 8 queries, lane j scores key j of the chunk, and an online
// softmax (running maximum and sum per query, fp32) rescales the per-lane
// accumulators of the output columns d = lane + 32 c.  One rounding to bf16 at
// the end.  CUDA cores: a first, plain form of the step.
#include "sige_internal.cuh"

#include <algorithm>
#include <atomic>
#include <math.h>

namespace sige {

constexpr int kAttnThreads = 256;   // 8 warps
constexpr int kAttnWarps = kAttnThreads / 32;
constexpr int kAttnKeys = 32;       // keys per staged chunk (one per lane)
constexpr int kAttnMaxBlock = 8;    // queries per tile <= 64 = 8 per warp
constexpr int kAttnQPerWarp = kAttnMaxBlock * kAttnMaxBlock / kAttnWarps;
constexpr int kAttnMaxHead = 256;   // per-head width of q / k and of v
constexpr int kAttnCols = kAttnMaxHead / 32;

struct AttnParams {
    const __nv_bfloat16 *q;   // [N][H][W][D]
    const __nv_bfloat16 *k;   // [N][Lk][D]
    const __nv_bfloat16 *v;   // [N][Lk][Dv]
    __nv_bfloat16 *o;         // [N][H][W][Dv]
    const int32_t *idx;       // [cap][2] tile origins (h0, w0)
    const int32_t *count;
    int32_t N, H, W, D, Dv, Lk, heads, dh, dvh, b, cap;
    float scale;              // 1 / sqrt(dh)
};

// Shared floats of one CTA: queries [b*b][dh], keys [32][dh + 1] (padded so
// that the 32 lanes reading one column of different rows hit different
// banks), values [32][dvh], softmax weights [8 warps][32].
static size_t attn_smem_bytes(int b, int dh, int dvh)
{
    return sizeof(float) * ((size_t)b * b * dh + (size_t)kAttnKeys * (dh + 1) + (size_t)kAttnKeys * dvh +
                            (size_t)kAttnWarps * kAttnKeys);
}

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(kAttnThreads) k_attention(const __grid_constant__ AttnParams p)
{
    extern __shared__ float attn_smem[];
    const int dh = p.dh, dvh = p.dvh, dhp = p.dh + 1;
    float *Qs = attn_smem;                          // [b*b][dh]
    float *Ks = Qs + p.b * p.b * dh;                // [32][dh + 1]
    float *Vs = Ks + kAttnKeys * dhp;               // [32][dvh]
    float *Ps = Vs + kAttnKeys * dvh;               // [8][32]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntile = min(__ldg(p.count), p.cap);
    const int units = ntile * p.N * p.heads;

#pragma unroll 1
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int head = u % p.heads;
        const int rest = u / p.heads;
        const int n = rest % p.N;
        const int t = rest / p.N;
        const int2 org = __ldg(reinterpret_cast<const int2 *>(p.idx) + t);
        // the tile's queries, clipped to the map: query qi is pixel
        // (org.x + qi / wb, org.y + qi % wb)
        const int hb = min(p.b, p.H - org.x), wb = min(p.b, p.W - org.y);
        const int nq = (hb > 0 && wb > 0 && org.x >= 0 && org.y >= 0) ? hb * wb : 0;
        __syncthreads();   // the previous unit has finished with the staged queries
#pragma unroll 1
        for (int e = threadIdx.x; e < nq * dh; e += kAttnThreads) {
            const int qi = e / dh, d = e - qi * dh;
            const int y = org.x + qi / wb, x = org.y + qi % wb;
            Qs[qi * dh + d] = __bfloat162float(p.q[(((int64_t)n * p.H + y) * p.W + x) * p.D + head * dh + d]);
        }
        float m[kAttnQPerWarp], l[kAttnQPerWarp], acc[kAttnQPerWarp][kAttnCols];
#pragma unroll
        for (int s = 0; s < kAttnQPerWarp; ++s) {
            m[s] = -INFINITY;
            l[s] = 0.0f;
#pragma unroll
            for (int c = 0; c < kAttnCols; ++c)
                acc[s][c] = 0.0f;
        }
        const int64_t kbase = (int64_t)n * p.Lk;
#pragma unroll 1
        for (int k0 = 0; k0 < p.Lk; k0 += kAttnKeys) {
            const int nk = min(kAttnKeys, p.Lk - k0);
            __syncthreads();   // queries staged; the previous chunk consumed
#pragma unroll 1
            for (int e = threadIdx.x; e < kAttnKeys * dh; e += kAttnThreads) {
                const int j = e / dh, d = e - j * dh;
                Ks[j * dhp + d] = j < nk ? __bfloat162float(p.k[(kbase + k0 + j) * p.D + head * dh + d]) : 0.0f;
            }
#pragma unroll 1
            for (int e = threadIdx.x; e < kAttnKeys * dvh; e += kAttnThreads) {
                const int j = e / dvh, d = e - j * dvh;
                Vs[j * dvh + d] = j < nk ? __bfloat162float(p.v[(kbase + k0 + j) * p.Dv + head * dvh + d]) : 0.0f;
            }
            __syncthreads();
#pragma unroll
            for (int s = 0; s < kAttnQPerWarp; ++s) {
                const int qi = warp + kAttnWarps * s;
                if (qi >= nq)   // the same for the whole warp
                    break;
                float sc = 0.0f;
                const float *qr = Qs + qi * dh, *kr = Ks + lane * dhp;
#pragma unroll 4
                for (int d = 0; d < dh; ++d)
                    sc = fmaf(qr[d], kr[d], sc);
                sc = lane < nk ? sc * p.scale : -INFINITY;
                const float mn = fmaxf(m[s], warp_max(sc));   // finite: the chunk holds >= 1 key
                const float pj = lane < nk ? expf(sc - mn) : 0.0f;
                const float corr = expf(m[s] - mn);            // 0 on the first chunk (m = -inf)
                l[s] = l[s] * corr + warp_sum(pj);
                Ps[warp * kAttnKeys + lane] = pj;
                __syncwarp();
#pragma unroll
                for (int c = 0; c < kAttnCols; ++c) {
                    const int d = c * 32 + lane;
                    if (c * 32 < dvh) {
                        float a = acc[s][c] * corr;
                        if (d < dvh) {
#pragma unroll 4
                            for (int j = 0; j < nk; ++j)
                                a = fmaf(Ps[warp * kAttnKeys + j], Vs[j * dvh + d], a);
                        }
                        acc[s][c] = a;
                    }
                }
                __syncwarp();
                m[s] = mn;
            }
        }
#pragma unroll
        for (int s = 0; s < kAttnQPerWarp; ++s) {
            const int qi = warp + kAttnWarps * s;
            if (qi >= nq)
                break;
            const int y = org.x + qi / wb, x = org.y + qi % wb;
            __nv_bfloat16 *orow = p.o + (((int64_t)n * p.H + y) * p.W + x) * p.Dv + head * dvh;
            const float inv = 1.0f / l[s];
#pragma unroll
            for (int c = 0; c < kAttnCols; ++c) {
                const int d = c * 32 + lane;
                if (d < dvh)
                    orow[d] = __float2bfloat16_rn(acc[s][c] * inv);
            }
        }
    }
}

} // namespace sige

using namespace sige;

extern "C" int sige_attention_core(const void *q, const sige_tensor_desc *qd, const void *k, const void *v,
                                   int32_t keys, int32_t dv, int32_t heads, const int32_t *idx,
                                   const int32_t *count, int32_t capacity, int32_t block, void *o,
                                   sige_stream_t stream)
{
    if (!q || !qd || !k || !v || !o || !idx || !count || capacity < 0 || keys < 1 || dv < 1 || heads < 1)
        return SIGE_ERR_INVALID_ARG;
    // the device indexes keys and units in 32 bits
    if ((int64_t)qd->n * keys > INT32_MAX)
        return SIGE_ERR_INVALID_ARG;
    if (qd->n < 1 || qd->h < 1 || qd->w < 1 || qd->c < 1 || block < 1)
        return SIGE_ERR_INVALID_ARG;
    if (qd->c % heads || dv % heads)
        return SIGE_ERR_INVALID_ARG;
    if (qd->dtype != SIGE_BF16 || qd->layout != SIGE_NHWC || block > kAttnMaxBlock || qd->c / heads > kAttnMaxHead ||
        dv / heads > kAttnMaxHead)
        return SIGE_ERR_UNSUPPORTED;
    if (capacity == 0)
        return SIGE_OK;
    const int tc = attention_core_tc(q, k, v, o, idx, count, qd->n, qd->h, qd->w, qd->c, dv, keys, heads, block,
                                     capacity, (cudaStream_t)stream);
    if (tc != 1)
        return tc;
    AttnParams p{};
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k = static_cast<const __nv_bfloat16 *>(k);
    p.v = static_cast<const __nv_bfloat16 *>(v);
    p.o = static_cast<__nv_bfloat16 *>(o);
    p.idx = idx;
    p.count = count;
    p.N = qd->n; p.H = qd->h; p.W = qd->w; p.D = qd->c; p.Dv = dv; p.Lk = keys; p.heads = heads;
    p.dh = qd->c / heads; p.dvh = dv / heads; p.b = block; p.cap = capacity;
    p.scale = 1.0f / sqrtf((float)p.dh);
    const size_t smem = attn_smem_bytes(block, p.dh, p.dvh);
    static std::atomic<int> smem_set[64];   // per device: the opt-in of the largest request
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64)
        dev = 0;
    if ((int)smem > smem_set[dev].load(std::memory_order_acquire)) {
        const size_t most = attn_smem_bytes(kAttnMaxBlock, kAttnMaxHead, kAttnMaxHead);
        if (cudaFuncSetAttribute(k_attention, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)most) != cudaSuccess)
            return SIGE_ERR_CUDA;
        smem_set[dev].store((int)most, std::memory_order_release);
    }
    const int64_t units = (int64_t)capacity * p.N * p.heads;
    if (units > INT32_MAX)
        return SIGE_ERR_INVALID_ARG;
    const int grid = (int)std::min<int64_t>(units, (int64_t)device_sm_count() * 4);
    k_attention<<<grid, kAttnThreads, smem, (cudaStream_t)stream>>>(p);
    count_launch();
    return launch_check();
}

extern "C" int sige_attention_path(const sige_tensor_desc *qd, int32_t dv, int32_t heads)
{
    if (!qd || dv < 1 || heads < 1 || qd->c < 1)
        return SIGE_ERR_INVALID_ARG;
    if (qd->c % heads || dv % heads)
        return SIGE_ERR_INVALID_ARG;
    if (qd->dtype != SIGE_BF16 || qd->layout != SIGE_NHWC || qd->c / heads > kAttnMaxHead || dv / heads > kAttnMaxHead)
        return SIGE_ERR_UNSUPPORTED;
    return attention_tc_scope(qd->c / heads, dv / heads) ? 1 : 0;
}
