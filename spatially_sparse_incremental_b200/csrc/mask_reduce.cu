// Difference mask -> multi-scale active-tile lists, one launch.
//
// mer.dev notes on SIGE, section 3 "Method": the edited region is located by
// comparing the original and edited inputs.  Section 3.2 "Sparse Engine
// SIGE": the difference mask is downsampled to several scales, dilated, and
// used to select tiles.  SIGE project page, "Overview": the mask is reduced to
// active block indices.
//
// Layout of the work:
//   phase 1 (all CTAs, HBM-bound): stream both inputs once with 16-byte
//     loads; an element whose |edit - orig| > threshold marks, at every
//     scale, the tile its pixel falls in.  Downsampling by an integer factor f
//     followed by b x b tiles is the same as tiles of b*f input pixels, so the
//     OR-downsample and the tile OR collapse into one flag store per scale.
//   phase 2 (the last CTA to arrive): per scale, dilate the tile flags by
//     `dilate` tiles (equal to dilating the scale's mask by dilate*b pixels
//     before tiling), compact the active tiles in row-major order with a
//     block-wide prefix sum, write the (h0, w0) list and the count, then clear
//     the flags and the arrival counter so the workspace is ready for the next
//     call.
#include <algorithm>

#include "sige_internal.cuh"

namespace sige {

struct ScaleParams {
    int32_t tile_h, tile_w;  // tile edge in input pixels (block * downsample factor)
    int32_t th, tw;          // tile grid at this scale
    int32_t block;           // tile edge at this scale; origins are (i*block, j*block)
    int32_t capacity;        // pairs
    int32_t flag_off;        // byte offset of this scale's flags
    int32_t idx_off;         // pair offset of this scale's list
};

struct MaskParams {
    const uint8_t *a;  // original
    const uint8_t *b;  // edited
    int32_t N, H, W, C, dtype, layout;
    float thr;
    int32_t dilate;
    int32_t n_scales;
    ScaleParams sc[kMaxScales];
    int32_t *idx;
    int32_t *counts;
    WsHeader *hdr;
    uint8_t *flags;
    int32_t flag_bytes;  // multiple of 16
    int64_t nwork;       // vectors (modes 0, 1) or elements (mode 2)
    int32_t mode;        // 0 = NHWC 16-byte vectors, 1 = NCHW 16-byte vectors, 2 = scalar
    int32_t vpp;         // mode 0: vectors per pixel
    int32_t epv;         // elements per vector
};

constexpr int kMaskThreads = 256;
constexpr int kMaskUnroll = 8;
constexpr int kFlagSmem = 16384;

__device__ __forceinline__ float elem_as_float(uint32_t word, int k, int dtype)
{
    if (dtype == SIGE_U8)
        return (float)((word >> (8 * k)) & 0xFFu);
    if (dtype == SIGE_BF16)
        return k ? bf16_hi(word) : bf16_lo(word);
    return __uint_as_float(word);
}

// Bit e set <=> element e of the 16-byte vector differs by more than thr.
__device__ __forceinline__ uint32_t diff_bits16(uint4 a, uint4 b, int dtype, float thr)
{
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
    const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
    uint32_t bits = 0;
    if (dtype == SIGE_U8) {
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int k = 0; k < 4; ++k)
                if (fabsf(elem_as_float(bw[w], k, SIGE_U8) - elem_as_float(aw[w], k, SIGE_U8)) > thr)
                    bits |= 1u << (4 * w + k);
    } else if (dtype == SIGE_BF16) {
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int k = 0; k < 2; ++k)
                if (fabsf(elem_as_float(bw[w], k, SIGE_BF16) - elem_as_float(aw[w], k, SIGE_BF16)) > thr)
                    bits |= 1u << (2 * w + k);
    } else {
#pragma unroll
        for (int w = 0; w < 4; ++w)
            if (fabsf(__uint_as_float(bw[w]) - __uint_as_float(aw[w])) > thr)
                bits |= 1u << w;
    }
    return bits;
}

// The scale table is indexed with a runtime scale number; kernel parameters
// read that way go through generic loads, so every CTA first copies the table
// into shared memory.
__device__ __forceinline__ void mark(const ScaleParams *sc, int n_scales, uint8_t *flags, int y, int x)
{
    for (int s = 0; s < n_scales; ++s) {
        const ScaleParams q = sc[s];
        flags[q.flag_off + (y / q.tile_h) * q.tw + (x / q.tile_w)] = 1;
    }
}

__device__ __forceinline__ float scalar_elem(const uint8_t *base, int64_t i, int dtype)
{
    if (dtype == SIGE_U8)
        return (float)base[i];
    if (dtype == SIGE_BF16)
        return __uint_as_float((uint32_t)(reinterpret_cast<const uint16_t *>(base)[i]) << 16);
    return reinterpret_cast<const float *>(base)[i];
}

__device__ __forceinline__ bool phase1(const MaskParams &p, const ScaleParams *sc)
{
    bool wrote = false;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t HW = (int64_t)p.H * p.W;
    const int n_scales = p.n_scales, mode = p.mode, dtype = p.dtype, W = p.W, H = p.H, C = p.C;
    const int vpp = p.vpp, epv = p.epv, layout = p.layout;
    const float thr = p.thr;
    const int64_t nwork = p.nwork;
    const uint8_t *a = p.a, *b = p.b;
    uint8_t *flags = p.flags;
    for (int64_t v0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v0 < nwork;
         v0 += stride * kMaskUnroll) {
        if (mode == 2) {
#pragma unroll
            for (int u = 0; u < kMaskUnroll; ++u) {
                int64_t i = v0 + u * stride;
                if (i >= nwork)
                    break;
                float d = fabsf(scalar_elem(b, i, dtype) - scalar_elem(a, i, dtype));
                if (d > thr) {
                    wrote = true;
                    int y, x;
                    if (layout == SIGE_NHWC) {
                        int64_t pix = i / C;
                        y = (int)((pix % HW) / W);
                        x = (int)(pix % W);
                    } else {
                        y = (int)((i / W) % H);
                        x = (int)(i % W);
                    }
                    mark(sc, n_scales, flags, y, x);
                }
            }
            continue;
        }
        uint4 av[kMaskUnroll], bv[kMaskUnroll];
#pragma unroll
        for (int u = 0; u < kMaskUnroll; ++u) {
            int64_t v = v0 + u * stride;
            if (v < nwork) {
                av[u] = ld_stream16(a + v * 16);
                bv[u] = ld_stream16(b + v * 16);
            }
        }
#pragma unroll
        for (int u = 0; u < kMaskUnroll; ++u) {
            int64_t v = v0 + u * stride;
            if (v >= nwork)
                break;
            uint32_t bits = diff_bits16(av[u], bv[u], dtype, thr);
            if (!bits)
                continue;
            wrote = true;
            if (mode == 0) {
                int64_t pix = v / vpp;
                mark(sc, n_scales, flags, (int)((pix % HW) / W), (int)(pix % W));
            } else {
                int64_t e0 = v * epv;
                int y = (int)((e0 / W) % H);
                int x0 = (int)(e0 % W);
                while (bits) {
                    int k = __ffs(bits) - 1;
                    bits &= bits - 1;
                    mark(sc, n_scales, flags, y, x0 + k);
                }
            }
        }
    }
    return wrote;
}

// Block-wide exclusive prefix sum of one int per thread; *total gets the sum.
__device__ __forceinline__ int block_scan(int v, int *warp_sums, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o)
            incl += t;
    }
    if (lane == 31)
        warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < nw ? warp_sums[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xFFFFFFFFu, wi, o);
            if (lane >= o)
                wi += t;
        }
        if (lane < nw)
            warp_sums[lane] = wi - w;
        if (lane == 31)
            warp_sums[32] = wi;
    }
    __syncthreads();
    const int off = warp_sums[warp] + incl - v;
    *total = warp_sums[32];
    __syncthreads();
    return off;
}

constexpr int kTilesPerThread = 4;

__device__ __forceinline__ void phase2(const MaskParams &p, const ScaleParams *sc)
{
    __shared__ uint8_t sflag[kFlagSmem];
    __shared__ int warp_sums[33];
    const int n_scales = p.n_scales, dilate = p.dilate;
    for (int s = 0; s < n_scales; ++s) {
        const ScaleParams q = sc[s];
        const int nt = q.th * q.tw;
        const uint8_t *g = p.flags + q.flag_off;
        const bool in_smem = nt <= kFlagSmem;
        if (in_smem) {
            // flag_off is 16-byte aligned and the flag area is padded to 16
            // bytes, so these 16-byte reads stay inside it
            for (int t = threadIdx.x * 16; t < nt; t += blockDim.x * 16) {
                const uint4 w = __ldcg(reinterpret_cast<const uint4 *>(g + t));
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    if (t + k < nt)
                        sflag[t + k] = (uint8_t)((ws[k >> 2] >> (8 * (k & 3))) & 0xFF);
            }
            __syncthreads();
        }
        int base = 0;
        const int chunk = blockDim.x * kTilesPerThread;
        for (int t0 = 0; t0 < nt; t0 += chunk) {
            const int tb = t0 + threadIdx.x * kTilesPerThread;
            uint32_t bits = 0;
#pragma unroll
            for (int k = 0; k < kTilesPerThread; ++k) {
                const int t = tb + k;
                if (t >= nt)
                    break;
                const int i = t / q.tw, j = t - i * q.tw;
                const int i0 = max(0, i - dilate), i1 = min(q.th - 1, i + dilate);
                const int j0 = max(0, j - dilate), j1 = min(q.tw - 1, j + dilate);
                int act = 0;
                for (int ii = i0; ii <= i1 && !act; ++ii)
                    for (int jj = j0; jj <= j1; ++jj) {
                        const uint8_t f = in_smem ? sflag[ii * q.tw + jj] : __ldcg(g + ii * q.tw + jj);
                        if (f) {
                            act = 1;
                            break;
                        }
                    }
                bits |= (uint32_t)act << k;
            }
            int chunk_total;
            int pos = base + block_scan(__popc(bits), warp_sums, &chunk_total);
            while (bits) {
                const int k = __ffs(bits) - 1;
                bits &= bits - 1;
                if (pos < q.capacity) {
                    const int t = tb + k;
                    const int i = t / q.tw, j = t - i * q.tw;
                    reinterpret_cast<int2 *>(p.idx)[q.idx_off + pos] = make_int2(i * q.block, j * q.block);
                }
                ++pos;
            }
            base += chunk_total;
        }
        if (threadIdx.x == 0) {
            p.counts[s] = base;
            if (base > q.capacity)
                record_error(p.hdr, SIGE_ERR_CAPACITY, s);
        }
        __syncthreads();
    }
    // leave the workspace zero-filled for the next call
    const uint4 z = make_uint4(0, 0, 0, 0);
    for (int k = threadIdx.x; k < p.flag_bytes / 16; k += blockDim.x)
        reinterpret_cast<uint4 *>(p.flags)[k] = z;
    if (threadIdx.x == 0)
        p.hdr->arrive = 0;
}

__global__ void __launch_bounds__(kMaskThreads) k_mask_reduce(const __grid_constant__ MaskParams p)
{
    __shared__ ScaleParams s_sc[kMaxScales];
    if (threadIdx.x < kMaxScales)
        s_sc[threadIdx.x] = p.sc[threadIdx.x];
    __syncthreads();
    if (phase1(p, s_sc))
        __threadfence();   // flags stored by this thread are visible before the arrival below
    __syncthreads();
    __shared__ int is_last;
    if (threadIdx.x == 0) {
        unsigned prev = atomicAdd(&p.hdr->arrive, 1u);
        is_last = (prev == gridDim.x - 1);
    }
    __syncthreads();
    if (!is_last)
        return;
    __threadfence();
    phase2(p, s_sc);
}

// ------------------------------------------------------------------ host

static size_t align16(size_t v) { return (v + 15) & ~(size_t)15; }

static bool scales_ok(const sige_tensor_desc *in, int32_t n_scales, const sige_scale_desc *scales)
{
    if (!in || !scales || n_scales < 1 || n_scales > kMaxScales)
        return false;
    for (int s = 0; s < n_scales; ++s) {
        const sige_scale_desc &q = scales[s];
        if (q.h < 1 || q.w < 1 || q.block < 1 || q.capacity < 0)
            return false;
        if (in->h % q.h || in->w % q.w)
            return false;
    }
    return true;
}

static size_t flag_bytes_of(int32_t n_scales, const sige_scale_desc *scales)
{
    size_t tot = 0;
    for (int s = 0; s < n_scales; ++s) {
        size_t th = (scales[s].h + scales[s].block - 1) / scales[s].block;
        size_t tw = (scales[s].w + scales[s].block - 1) / scales[s].block;
        tot += align16(th * tw);
    }
    return tot;
}

} // namespace sige

using namespace sige;

extern "C" size_t sige_reduce_mask_workspace_bytes(const sige_tensor_desc *in, int32_t n_scales,
                                                   const sige_scale_desc *scales)
{
    if (!scales_ok(in, n_scales, scales))
        return 0;
    return kWsHeader + flag_bytes_of(n_scales, scales);
}

extern "C" int sige_reduce_mask(const void *a_orig, const void *a_edit, const sige_tensor_desc *in,
                                float threshold, int32_t dilate, int32_t n_scales,
                                const sige_scale_desc *scales, int32_t *idx, int32_t *counts,
                                void *workspace, size_t workspace_bytes, sige_stream_t stream)
{
    if (!a_orig || !a_edit || !in || !idx || !counts)
        return SIGE_ERR_INVALID_ARG;
    if (in->n < 1 || in->h < 1 || in->w < 1 || in->c < 1)
        return SIGE_ERR_INVALID_ARG;
    if (in->dtype != SIGE_U8 && in->dtype != SIGE_F32 && in->dtype != SIGE_BF16)
        return SIGE_ERR_UNSUPPORTED;
    if (in->layout != SIGE_NHWC && in->layout != SIGE_NCHW)
        return SIGE_ERR_UNSUPPORTED;
    if (!(threshold >= 0.0f) || threshold != threshold || dilate < 0)
        return SIGE_ERR_INVALID_ARG;
    if (!scales_ok(in, n_scales, scales))
        return SIGE_ERR_INVALID_ARG;
    const size_t need = kWsHeader + flag_bytes_of(n_scales, scales);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15))
        return SIGE_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(idx) & 7))
        return SIGE_ERR_INVALID_ARG;

    MaskParams p{};
    p.a = static_cast<const uint8_t *>(a_orig);
    p.b = static_cast<const uint8_t *>(a_edit);
    p.N = in->n; p.H = in->h; p.W = in->w; p.C = in->c;
    p.dtype = in->dtype; p.layout = in->layout;
    p.thr = threshold;
    p.dilate = dilate;
    p.n_scales = n_scales;
    int32_t foff = 0, ioff = 0;
    for (int s = 0; s < n_scales; ++s) {
        const sige_scale_desc &q = scales[s];
        ScaleParams &o = p.sc[s];
        o.block = q.block;
        o.tile_h = q.block * (in->h / q.h);
        o.tile_w = q.block * (in->w / q.w);
        o.th = (q.h + q.block - 1) / q.block;
        o.tw = (q.w + q.block - 1) / q.block;
        o.capacity = q.capacity;
        o.flag_off = foff;
        o.idx_off = ioff;
        foff += (int32_t)align16((size_t)o.th * o.tw);
        ioff += q.capacity;
    }
    p.idx = idx;
    p.counts = counts;
    p.hdr = static_cast<WsHeader *>(workspace);
    p.flags = static_cast<uint8_t *>(workspace) + kWsHeader;
    p.flag_bytes = foff;

    const int esz = in->dtype == SIGE_U8 ? 1 : in->dtype == SIGE_BF16 ? 2 : 4;
    const int64_t nelem = (int64_t)in->n * in->h * in->w * in->c;
    const bool aligned = ((reinterpret_cast<uintptr_t>(a_orig) | reinterpret_cast<uintptr_t>(a_edit)) & 15) == 0;
    p.epv = 16 / esz;
    if (aligned && in->layout == SIGE_NHWC && ((int64_t)in->c * esz) % 16 == 0) {
        p.mode = 0;
        p.vpp = (int32_t)(((int64_t)in->c * esz) / 16);
        p.nwork = nelem * esz / 16;
    } else if (aligned && in->layout == SIGE_NCHW && ((int64_t)in->w * esz) % 16 == 0) {
        p.mode = 1;
        p.nwork = nelem * esz / 16;
    } else {
        p.mode = 2;
        p.nwork = nelem;
    }
    static int occ[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64)
        dev = 0;
    if (!occ[dev]) {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_mask_reduce, kMaskThreads, 0) != cudaSuccess || n < 1)
            n = 1;
        occ[dev] = n;
    }
    int64_t per_cta = (int64_t)kMaskThreads * kMaskUnroll;
    int grid = (int)std::min<int64_t>((p.nwork + per_cta - 1) / per_cta, (int64_t)device_sm_count() * occ[dev]);
    grid = std::max(grid, 1);
    k_mask_reduce<<<grid, kMaskThreads, 0, (cudaStream_t)stream>>>(p);
    count_launch();
    return launch_check();
}
