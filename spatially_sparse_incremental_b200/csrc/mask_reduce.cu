// Difference mask -> multi-scale active-tile lists, one launch.
//
// mer.dev notes on SIGE, section 3 "Method": the edited region is located by
// comparing the original and edited inputs.  Section 3.2 "Sparse Engine
// SIGE": the difference mask is downsampled to several scales, dilated, and
// used to select tiles.  SIGE project page, "Overview": the mask is reduced to
// active block indices.
//
// Layout of the work:
//   phase 1 (every CTA but CTA 0, HBM-bound): stream both inputs once.  The
//     inputs are cut into chunks (up to 16 KB of each input); every streaming
//     CTA keeps four in flight with bulk asynchronous copies into shared
//     memory.  The first four of each CTA are fixed (chunk worker + k *
//     workers); the rest are handed out by a counter in the workspace header,
//     one at a time as a stage frees, so CTAs whose copies land late take
//     fewer chunks and all finish together (with a fixed split the last CTA
//     finished ~4 us after the median one).  An element whose |edit - orig| >
//     threshold marks, at every scale, the tile its pixel falls in (with a
//     pixel radius R, every tile within R pixels of it at that scale).
//     Downsampling by an integer factor f followed by b x b tiles is the same
//     as tiles of b*f input pixels, so the OR-downsample and the tile OR
//     collapse into one flag store per scale.
//   phase 2 (CTA 0, which takes no part in phase 1): per scale, dilate the
//     tile flags by `dilate` tiles (equal to dilating the scale's mask by
//     dilate*b pixels before tiling), compact the active tiles in row-major
//     order, write the (h0, w0) list and the count, then clear the flags and
//     the arrival counter so the workspace is ready for the next call.  Grids
//     of at most 32 x 32 tiles take one warp per scale (rows as 32-bit words,
//     dilation by shifts and shuffles, a warp prefix sum); larger grids use
//     the block-wide bit-word path.
//
// Phase 2 runs once per call on one CTA, so its cost is latency: each of its
// instructions is fetched cold.  CTA 0 therefore runs it once without storing
// anything while the other CTAs stream the inputs, which leaves its code in
// this SM's instruction cache, then waits (bounded) for the last arrival and
// runs it for real.  CTA 0 is the only CTA that waits on others, and the
// others wait on nothing, so any scheduling order of the CTAs completes.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "sige_internal.cuh"

namespace sige {

struct ScaleParams {
    int32_t tile_h, tile_w;  // tile edge in input pixels (block * downsample factor)
    int32_t th, tw;          // tile grid at this scale
    int32_t block;           // tile edge at this scale; origins are (i*block, j*block)
    int32_t capacity;        // pairs
    int32_t flag_off;        // byte offset of this scale's flags
    int32_t idx_off;         // pair offset of this scale's list
    int32_t log_h, log_w;    // log2 of tile_h / tile_w when powers of two, else -1
    int32_t fy, fx;          // downsample factors (input pixels per scale pixel)
    int32_t hs, ws;          // the scale's grid
};

struct __align__(16) MaskParams {
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
    int32_t pow2;        // vpp, H and W are powers of two: index math by shifts
    int32_t log_vpp, log_w, log_epv;
    int32_t chunk;       // modes 0, 1: vectors per chunk of each input (multiple of 256)
    int32_t nchunks;     // modes 0, 1: chunks of each input
    int32_t radius;      // pixel dilation at each scale before tiling (0: none)
    int64_t wait_cycles; // bound of CTA 0's wait for the streaming CTAs, in SM clock cycles
};

// Copy the parameter block into shared memory, one 16-byte piece per lane of
// warp 0: a single round of loads, whose latency the streaming CTAs overlap
// with their first copies in flight.
__device__ __forceinline__ void copy_params(MaskParams *dst, const MaskParams &src)
{
    constexpr int kPieces = (int)(sizeof(MaskParams) / 16);
    static_assert(sizeof(MaskParams) % 16 == 0, "parameter block is copied in 16-byte pieces");
    const int lane = threadIdx.x & 31;
    static_assert(kPieces <= 64, "two pieces per lane at most");
    if (lane < kPieces)
        reinterpret_cast<uint4 *>(dst)[lane] = reinterpret_cast<const uint4 *>(&src)[lane];
    if (lane + 32 < kPieces)
        reinterpret_cast<uint4 *>(dst)[lane + 32] = reinterpret_cast<const uint4 *>(&src)[lane + 32];
}

constexpr int kMaskThreads = 256;
constexpr int kScalarPerThread = 8;   // mode 2: elements per thread of the grid size

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

// Kernel parameters read through a pointer or with a runtime index go through
// generic loads, which cost about a global-memory round trip each.  Every CTA
// therefore copies the parameter block into shared memory once, and the
// out-of-line functions below read that copy.
__device__ __forceinline__ void mark(const ScaleParams *sc, int n_scales, uint8_t *flags, int y, int x, int R)
{
    for (int s = 0; s < n_scales; ++s) {
        const ScaleParams q = sc[s];
        if (R == 0) {
            const int ty = q.log_h >= 0 ? y >> q.log_h : y / q.tile_h;
            const int tx = q.log_w >= 0 ? x >> q.log_w : x / q.tile_w;
            flags[q.flag_off + ty * q.tw + tx] = 1;
            continue;
        }
        // pixel dilation: every tile the (2R+1)^2 square around the pixel's
        // scale position touches (clipped at the border)
        const int Y = y / q.fy, X = x / q.fx;
        const int t0 = max(0, Y - R) / q.block, t1 = min(q.hs - 1, Y + R) / q.block;
        const int u0 = max(0, X - R) / q.block, u1 = min(q.ws - 1, X + R) / q.block;
        for (int ty = t0; ty <= t1; ++ty)
            for (int tx = u0; tx <= u1; ++tx)
                flags[q.flag_off + ty * q.tw + tx] = 1;
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

// Mark the tiles of the elements set in `bits` (the exact test of vector v);
// out of line, since only vectors inside the edit reach it.
__device__ __noinline__ void mark_bits(const MaskParams &p, const ScaleParams *sc, int64_t v, uint32_t bits)
{
    if (p.mode == 0) {
        if (p.pow2) {
            const int64_t pix = v >> p.log_vpp;
            mark(sc, p.n_scales, p.flags, (int)(pix >> p.log_w) & (p.H - 1), (int)pix & (p.W - 1), p.radius);
        } else {
            const int64_t HW = (int64_t)p.H * p.W;
            const int64_t pix = v / p.vpp;
            mark(sc, p.n_scales, p.flags, (int)((pix % HW) / p.W), (int)(pix % p.W), p.radius);
        }
    } else {
        const int64_t e0 = v * p.epv;
        const int y = p.pow2 ? (int)(e0 >> p.log_w) & (p.H - 1) : (int)((e0 / p.W) % p.H);
        const int x0 = p.pow2 ? (int)e0 & (p.W - 1) : (int)(e0 % p.W);
        while (bits) {
            const int k = __ffs(bits) - 1;
            bits &= bits - 1;
            mark(sc, p.n_scales, p.flags, y, x0 + k, p.radius);
        }
    }
}

__device__ __noinline__ bool scalar_pass(const MaskParams &p, const ScaleParams *sc, int worker, int nworkers)
{
    bool wrote = false;
    const int64_t stride = (int64_t)nworkers * blockDim.x;
    const int64_t HW = (int64_t)p.H * p.W;
    for (int64_t i = (int64_t)worker * blockDim.x + threadIdx.x; i < p.nwork; i += stride) {
        const float d = fabsf(scalar_elem(p.b, i, p.dtype) - scalar_elem(p.a, i, p.dtype));
        if (d > p.thr) {
            wrote = true;
            int y, x;
            if (p.layout == SIGE_NHWC) {
                const int64_t pix = i / p.C;
                y = (int)((pix % HW) / p.W);
                x = (int)(pix % p.W);
            } else {
                y = (int)((i / p.W) % p.H);
                x = (int)(i % p.W);
            }
            mark(sc, p.n_scales, p.flags, y, x, p.radius);
        }
    }
    return wrote;
}

constexpr int kMaskStages = 4;          // chunks in flight per streaming CTA
constexpr int kMaskChunkMax = 1024;     // vectors (16 KB) per chunk and input
constexpr size_t kMaskStreamSmem = (size_t)kMaskStages * 2 * kMaskChunkMax * 16;   // 128 KB
constexpr long long kMaskCopyWait = 1ll << 31;   // bound of one chunk wait (about 1 s)

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ bool mbar_try_parity(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n .reg .pred q;\n mbarrier.try_wait.parity.shared::cta.b64 q, [%1], %2;\n selp.u32 %0, 1, 0, q;\n}\n"
                 : "=r"(ok)
                 : "r"(bar), "r"(parity)
                 : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity)
{
    if (mbar_try_parity(bar, parity))
        return true;
    const long long t0 = clock64();
    while (!mbar_try_parity(bar, parity))
        if (clock64() - t0 > kMaskCopyWait)
            return false;
    return true;
}

// Chunk c of both inputs into stage st; one thread issues it.
__device__ __forceinline__ void issue_chunk(const MaskParams &p, uint8_t *stages, uint64_t *full, int64_t c, int st)
{
    const int64_t v0 = c * p.chunk;
    const uint32_t bytes = (uint32_t)(min((int64_t)p.chunk, p.nwork - v0) * 16);
    uint8_t *da = stages + (size_t)st * 2 * kMaskChunkMax * 16;
    uint8_t *db = da + (size_t)kMaskChunkMax * 16;
    const uint32_t bar = smem_addr(&full[st]);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(2 * bytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(da)),
                 "l"(p.a + v0 * 16), "r"(bytes), "r"(bar)
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_addr(db)),
                 "l"(p.b + v0 * 16), "r"(bytes), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ int64_t chunk_count(const MaskParams &p) { return p.nchunks; }

// The fixed first round of a streaming CTA (one thread; barriers
// initialised): chunk worker + k * nworkers into stage k, -1 past the end.
__device__ __forceinline__ void issue_first_chunks(const MaskParams &p, uint8_t *stages, uint64_t *full,
                                                   int64_t *s_chunk, int worker, int nworkers)
{
    const int64_t n = chunk_count(p);
    for (int k = 0; k < kMaskStages; ++k) {
        const int64_t c = worker + (int64_t)k * nworkers;
        s_chunk[k] = c < n ? c : -1;
        if (c < n)
            issue_chunk(p, stages, full, c, k);
    }
}

// Every streaming CTA takes from the work counter until a take returns a
// chunk past the end, so a call makes exactly (chunks - dyn0) + workers takes
// when dyn0 < chunks, none otherwise.  CTA 0 subtracts that number after the
// last arrival instead of storing 0: a take still on its way to memory then
// cannot leave the counter non-zero for the next call (subtraction and
// addition commute), and the streaming CTAs need no fence for it.
__device__ __forceinline__ void release_work_counter(const MaskParams &p, int nworkers)
{
    const int64_t n = chunk_count(p), dyn0 = (int64_t)kMaskStages * nworkers;
    if (p.mode != 2 && dyn0 < n)
        atomicSub(&p.hdr->next, (uint32_t)(n - dyn0 + nworkers));
}

// Stream chunks through the stage ring and compare them: stage i mod 4 holds
// chunk s_chunk[i mod 4] (-1: none; chunks are taken in increasing order, so
// the first empty stage ends the stream).  Thread 0 refills a stage from the
// counter once every thread is done with it, and asks for the index of the
// refill after that right away, so the counter's round trip overlaps a
// chunk's comparison.
// Bitwise-equal 16-byte vectors cannot differ by more than a non-negative
// threshold, so only vectors whose bytes differ get the exact float32 test.  Returns
// whether this thread stored a flag; *ok turns false if a copy never landed
// (then every copy still in flight has been waited for, boundedly).
__device__ __forceinline__ bool phase1_bulk(const MaskParams &p, const MaskParams &sp, uint8_t *stages,
                                            uint64_t *full, int64_t *s_chunk, int nworkers, bool *ok)
{
    const int64_t n = chunk_count(p), dyn0 = (int64_t)kMaskStages * nworkers;
    int64_t pend = n;
    if (threadIdx.x == 0 && dyn0 < n)
        pend = dyn0 + (int64_t)atomicAdd(&p.hdr->next, 1u);
    bool wrote = false;
    *ok = true;
    int64_t i = 0;
    for (;; ++i) {
        const int st = (int)(i % kMaskStages);
        const int64_t c = s_chunk[st];
        if (c < 0)
            break;
        const bool landed = mbar_wait_bounded(smem_addr(&full[st]), (uint32_t)((i / kMaskStages) & 1));
        if (landed) {
            const int64_t v0 = c * (int64_t)p.chunk;
            const int nv = (int)min((int64_t)p.chunk, p.nwork - v0);
            const uint4 *sa = reinterpret_cast<const uint4 *>(stages + (size_t)st * 2 * kMaskChunkMax * 16);
            const uint4 *sb = sa + kMaskChunkMax;
#pragma unroll 4
            for (int j = threadIdx.x; j < nv; j += blockDim.x) {
                const uint4 a = sa[j], b = sb[j];
                if ((a.x ^ b.x) | (a.y ^ b.y) | (a.z ^ b.z) | (a.w ^ b.w)) {
                    const uint32_t bits = diff_bits16(a, b, p.dtype, p.thr);
                    if (bits) {
                        mark_bits(sp, sp.sc, v0 + j, bits);
                        wrote = true;
                    }
                }
            }
        }
        // every thread is done with the stage (and has read s_chunk) before
        // it is refilled; the refill's s_chunk entry is read S iterations on,
        // after at least one more of these barriers
        if (!__syncthreads_and(landed)) {
            *ok = false;
            break;
        }
        if (threadIdx.x == 0) {
            if (pend < n) {
                s_chunk[st] = pend;
                issue_chunk(p, stages, full, pend, st);
                pend = dyn0 + (int64_t)atomicAdd(&p.hdr->next, 1u);
            } else {
                s_chunk[st] = -1;
            }
        }
    }
    if (!*ok && threadIdx.x == 0) {
        // no copy may still be writing this CTA's shared memory when it exits
        for (int64_t k = i; k < i + kMaskStages; ++k)
            if (s_chunk[k % kMaskStages] >= 0)
                mbar_wait_bounded(smem_addr(&full[k % kMaskStages]), (uint32_t)((k / kMaskStages) & 1));
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

// Phase 2 works on bit rows: word (i, w) holds the flags of tiles
// (i, 32w .. 32w+31).  Dilation by D tiles is then an OR of the D rows above and
// below followed by shifts of +-1..D bits (with carries from the neighbouring
// words), and the row-major compaction is a prefix sum of popcounts.
constexpr int kMaxWords = 4096;          // bit words per scale held in shared memory (131072 tiles)

__device__ __forceinline__ uint32_t row_word(const uint32_t *bits, int wpr, int th, int i, int w, int D)
{
    uint32_t v = 0;
    const int i0 = max(0, i - D), i1 = min(th - 1, i + D);
#pragma unroll 1
    for (int ii = i0; ii <= i1; ++ii)
        v |= bits[ii * wpr + w];
    return v;
}

// Tile grids of at most 32 x 32 (every grid of the SIGE workloads): one warp
// per scale, lane i holding tile row i as a bit word.  The scale's flags (at
// most 1 KB) come into shared memory with two 16-byte loads per lane (many
// small loads per thread do not overlap well); dilation is shuffles and
// shifts, the row-major prefix sum a warp scan, so no block barrier is on the
// path.
__device__ __forceinline__ void scale_small(const MaskParams &p, const ScaleParams &qs, int s, bool commit,
                                            uint8_t *stage)
{
    const ScaleParams q = qs;   // registers: stores below must not force re-reads
    const int lane = threadIdx.x & 31, D = p.dilate;
    const int nb = (q.th * q.tw + 15) & ~15;
    const uint4 *g = reinterpret_cast<const uint4 *>(p.flags + q.flag_off);
    uint4 *st = reinterpret_cast<uint4 *>(stage);
    const uint4 g0 = lane * 16 < nb ? __ldcg(g + lane) : make_uint4(0, 0, 0, 0);
    const uint4 g1 = (lane + 32) * 16 < nb ? __ldcg(g + lane + 32) : make_uint4(0, 0, 0, 0);
    st[lane] = g0;
    st[lane + 32] = g1;
    __syncwarp();
    // lane i assembles tile row i: bit j = flag (i, j)
    uint32_t mine = 0;
    if (lane < q.th) {
        const uint8_t *row = stage + lane * q.tw;
        if ((q.tw & 3) == 0) {
            uint32_t w[8];
#pragma unroll
            for (int k = 0; k < 8; ++k)
                w[k] = 4 * k < q.tw ? *reinterpret_cast<const uint32_t *>(row + 4 * k) : 0u;
#pragma unroll
            for (int k = 0; k < 8; ++k)
#pragma unroll
                for (int b = 0; b < 4; ++b)
                    mine |= (uint32_t)(((w[k] >> (8 * b)) & 0xFFu) != 0) << (4 * k + b);
        } else {
#pragma unroll 4
            for (int j = 0; j < q.tw; ++j)
                mine |= (uint32_t)(row[j] != 0) << j;
        }
    }
    uint32_t v = mine;
#pragma unroll 1
    for (int d = 1; d <= D; ++d) {
        const uint32_t up = __shfl_up_sync(0xFFFFFFFFu, mine, d);
        const uint32_t dn = __shfl_down_sync(0xFFFFFFFFu, mine, d);
        if (lane >= d)
            v |= up;
        if (lane + d < 32)
            v |= dn;
    }
    uint32_t h = v;
#pragma unroll 1
    for (int d = 1; d <= D; ++d)
        h |= (v << d) | (v >> d);
    h &= q.tw == 32 ? 0xFFFFFFFFu : ((1u << q.tw) - 1u);
    if (lane >= q.th)
        h = 0;
    const int c = __popc(h);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o)
            incl += t;
    }
    const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    if (!commit)
        return;
    int pos = incl - c;
    int2 *out = reinterpret_cast<int2 *>(p.idx) + q.idx_off;
    while (h) {
        const int k = __ffs(h) - 1;
        h &= h - 1;
        if (pos < q.capacity)
            out[pos] = make_int2(lane * q.block, k * q.block);
        ++pos;
    }
    if (lane == 0) {
        p.counts[s] = total;
        if (total > q.capacity)
            record_error(p.hdr, SIGE_ERR_CAPACITY, s);
    }
    // leave this scale's flags zero-filled for the next call
#pragma unroll 1
    for (int o = lane * 16; o < nb; o += 32 * 16)
        *reinterpret_cast<uint4 *>(p.flags + q.flag_off + o) = make_uint4(0, 0, 0, 0);
}

// commit = false: the same work with every global store left out (the warm-up
// pass of CTA 0, which may read flags that other CTAs are still writing).
// sbits, sdil: kMaxWords words each of shared memory (CTA 0 streams nothing, so
// its dynamic shared memory is free for them).
__device__ __noinline__ void phase2(const MaskParams &p, const ScaleParams *sc, bool commit, uint32_t *sbits,
                                   uint32_t *sdil)
{
    __shared__ int warp_sums[33];
    bool small = p.dilate < 32;
    for (int s = 0; s < p.n_scales; ++s)
        small = small && sc[s].th <= 32 && sc[s].tw <= 32;
    if (small) {
        const int warp = threadIdx.x >> 5;
        if (warp < p.n_scales)
            scale_small(p, sc[warp], warp, commit, reinterpret_cast<uint8_t *>(sdil) + warp * 1024);
        if (commit && threadIdx.x == 0) {
            p.hdr->arrive = 0;
            release_work_counter(p, gridDim.x - 1);
        }
        return;
    }
    const int n_scales = p.n_scales, D = p.dilate;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
#pragma unroll 1
    for (int s = 0; s < n_scales; ++s) {
        const ScaleParams q = sc[s];
        const int wpr = (q.tw + 31) >> 5;
        const int nw = q.th * wpr;
        const uint8_t *g = p.flags + q.flag_off;
        int base = 0;
        if (nw <= kMaxWords && D < 32) {
            // flag bytes -> shared memory in one round of 16-byte loads (the
            // flag area of a scale is 16-byte aligned and padded), then one
            // ballot per bit word
            const int nt = q.th * q.tw;
            uint8_t *sflag = reinterpret_cast<uint8_t *>(sdil);   // free until the dilation pass
            if (nt <= (int)(kMaxWords * sizeof(uint32_t))) {
#pragma unroll 1
                for (int t = threadIdx.x * 16; t < nt; t += blockDim.x * 16)
                    *reinterpret_cast<uint4 *>(sflag + t) = __ldcg(reinterpret_cast<const uint4 *>(g + t));
                __syncthreads();
            }
            const bool in_smem = nt <= (int)(kMaxWords * sizeof(uint32_t));
#pragma unroll 1
            for (int wi = warp; wi < nw; wi += nwarps) {
                const int i = wi / wpr, j = (wi - i * wpr) * 32 + lane;
                const int f = j < q.tw ? (in_smem ? sflag[i * q.tw + j] : __ldcg(g + i * q.tw + j)) : 0;
                const uint32_t word = __ballot_sync(0xFFFFFFFFu, f != 0);
                if (lane == 0)
                    sbits[wi] = word;
            }
            __syncthreads();
            // dilation: vertical OR, then horizontal shifts with carries
            const uint32_t last_mask = (q.tw & 31) ? ((1u << (q.tw & 31)) - 1u) : 0xFFFFFFFFu;
#pragma unroll 1
            for (int wi = threadIdx.x; wi < nw; wi += blockDim.x) {
                const int i = wi / wpr, w = wi - i * wpr;
                const uint32_t v = row_word(sbits, wpr, q.th, i, w, D);
                const uint32_t prev = w > 0 ? row_word(sbits, wpr, q.th, i, w - 1, D) : 0u;
                const uint32_t next = w + 1 < wpr ? row_word(sbits, wpr, q.th, i, w + 1, D) : 0u;
                uint32_t h = v;
#pragma unroll 1
                for (int d = 1; d <= D; ++d)
                    h |= (v << d) | (v >> d) | (prev >> (32 - d)) | (next << (32 - d));
                sdil[wi] = (w == wpr - 1) ? (h & last_mask) : h;
            }
            __syncthreads();
            // compaction: each thread takes a contiguous run of words
            const int per = (nw + blockDim.x - 1) / blockDim.x;
            const int w0 = min(nw, (int)threadIdx.x * per), w1 = min(nw, w0 + per);
            int cnt = 0;
#pragma unroll 1
            for (int wi = w0; wi < w1; ++wi)
                cnt += __popc(sdil[wi]);
            int total;
            int pos = block_scan(cnt, warp_sums, &total);
#pragma unroll 1
            for (int wi = w0; wi < w1; ++wi) {
                uint32_t m = sdil[wi];
                const int i = wi / wpr, jb = (wi - i * wpr) * 32;
                while (m) {
                    const int k = __ffs(m) - 1;
                    m &= m - 1;
                    if (commit && pos < q.capacity)
                        reinterpret_cast<int2 *>(p.idx)[q.idx_off + pos] = make_int2(i * q.block, (jb + k) * q.block);
                    ++pos;
                }
            }
            base = total;
        } else {
            // very large grids: byte flags straight from global memory
            const int nt = q.th * q.tw;
            const int chunk = blockDim.x;
#pragma unroll 1
            for (int t0 = 0; t0 < nt; t0 += chunk) {
                const int t = t0 + threadIdx.x;
                int act = 0;
                if (t < nt) {
                    const int i = t / q.tw, j = t - i * q.tw;
                    const int i0 = max(0, i - D), i1 = min(q.th - 1, i + D);
                    const int j0 = max(0, j - D), j1 = min(q.tw - 1, j + D);
#pragma unroll 1
                    for (int ii = i0; ii <= i1 && !act; ++ii)
#pragma unroll 1
                        for (int jj = j0; jj <= j1 && !act; ++jj)
                            act = __ldcg(g + ii * q.tw + jj) != 0;
                }
                int chunk_total;
                const int pos = base + block_scan(act, warp_sums, &chunk_total);
                if (commit && act && pos < q.capacity) {
                    const int i = t / q.tw, j = t - i * q.tw;
                    reinterpret_cast<int2 *>(p.idx)[q.idx_off + pos] = make_int2(i * q.block, j * q.block);
                }
                base += chunk_total;
            }
        }
        if (commit && threadIdx.x == 0) {
            p.counts[s] = base;
            if (base > q.capacity)
                record_error(p.hdr, SIGE_ERR_CAPACITY, s);
        }
        __syncthreads();
    }
    if (!commit)
        return;
    // leave the workspace zero-filled for the next call
    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll 1
    for (int k = threadIdx.x; k < p.flag_bytes / 16; k += blockDim.x)
        reinterpret_cast<uint4 *>(p.flags)[k] = z;
    if (threadIdx.x == 0) {
        p.hdr->arrive = 0;
        release_work_counter(p, gridDim.x - 1);
    }
}

// Default bound of CTA 0's wait for the streaming CTAs (about 4 s at 2 GHz);
// past it the call records SIGE_ERR_TIMEOUT and leaves its workspace as it
// is.  sige_set_wait_cycles() replaces it for later launches (a test of the
// failure path shortens it until it expires).
constexpr long long kMaskWaitCycles = 1ll << 33;

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t *ptr)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

__global__ void __launch_bounds__(kMaskThreads) k_mask_reduce(const __grid_constant__ MaskParams p)
{
    extern __shared__ __align__(128) uint8_t dyn[];
    __shared__ MaskParams s_p;
    __shared__ __align__(8) uint64_t full[kMaskStages];
    __shared__ int64_t s_chunk[kMaskStages];
    __shared__ int s_go;
    pdl_trigger();
    pdl_wait();   // the inputs, lists and workspace may come from the kernel before
    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaskStages; ++i)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&full[i])));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        if (blockIdx.x != 0 && p.mode != 2)
            issue_first_chunks(p, dyn, full, s_chunk, blockIdx.x - 1, gridDim.x - 1);
    }
    if (threadIdx.x < 32)
        copy_params(&s_p, p);
    __syncthreads();
    const ScaleParams *s_sc = s_p.sc;
    if (blockIdx.x == 0) {
        uint32_t *sbits = reinterpret_cast<uint32_t *>(dyn);
        uint32_t *sdil = sbits + kMaxWords;
        phase2(s_p, s_sc, false, sbits, sdil);
        // lane 0 of each warp polls the arrival counter, so the last arrival
        // is seen within an eighth of a load round trip; the first to see it
        // (or the first to give up) tells the others through shared memory
        if (threadIdx.x == 0)
            s_go = -1;
        __syncthreads();
        if ((threadIdx.x & 31) == 0) {
            volatile int *go = &s_go;
            const uint32_t want = gridDim.x - 1;
            const long long t0 = clock64();
            while (*go < 0) {
                if (ld_acquire_u32(&p.hdr->arrive) == want) {
                    *go = 1;
                    break;
                }
                if (clock64() - t0 > p.wait_cycles) {
                    if (atomicCAS(&s_go, -1, 0) == -1)
                        record_error(p.hdr, SIGE_ERR_TIMEOUT, -1);
                    break;
                }
            }
        }
        __syncthreads();
        if (s_go == 1)
            phase2(s_p, s_sc, true, sbits, sdil);
        return;
    }
    bool wrote, ok = true;
    if (p.mode == 2)
        wrote = scalar_pass(s_p, s_sc, blockIdx.x - 1, gridDim.x - 1);
    else
        wrote = phase1_bulk(p, s_p, dyn, full, s_chunk, gridDim.x - 1, &ok);
    if (!ok && threadIdx.x == 0)
        record_error(p.hdr, SIGE_ERR_TIMEOUT, -2);
    // The barrier orders every thread's flag stores before thread 0's fence,
    // and the fence (cumulative) makes them visible before the arrival.
    const bool any = __syncthreads_or(wrote);
    if (threadIdx.x == 0) {
        if (any)
            __threadfence();
        atomicAdd(&p.hdr->arrive, 1u);
    }
}

// ------------------------------------------------------------------ host

static size_t align16(size_t v) { return (v + 15) & ~(size_t)15; }

static int32_t log2_exact(int64_t v)
{
    if (v < 1 || (v & (v - 1)))
        return -1;
    int32_t l = 0;
    while ((int64_t)1 << l < v)
        ++l;
    return l;
}

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

// Host-side checks of a mask-reduction call that need no workspace; both
// entry points run them before anything is enqueued.
static int validate_mask_args(const void *a_orig, const void *a_edit, const sige_tensor_desc *in, float threshold,
                              int32_t dilate, int32_t radius, int32_t n_scales, const sige_scale_desc *scales,
                              const int32_t *idx, const int32_t *counts)
{
    if (!a_orig || !a_edit || !in || !idx || !counts)
        return SIGE_ERR_INVALID_ARG;
    if (in->n < 1 || in->h < 1 || in->w < 1 || in->c < 1)
        return SIGE_ERR_INVALID_ARG;
    if (in->dtype != SIGE_U8 && in->dtype != SIGE_F32 && in->dtype != SIGE_BF16)
        return SIGE_ERR_UNSUPPORTED;
    if (in->layout != SIGE_NHWC && in->layout != SIGE_NCHW)
        return SIGE_ERR_UNSUPPORTED;
    if (!(threshold >= 0.0f) || threshold != threshold || dilate < 0 || radius < 0)
        return SIGE_ERR_INVALID_ARG;
    if (!scales_ok(in, n_scales, scales))
        return SIGE_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(idx) & 7))
        return SIGE_ERR_INVALID_ARG;
    return SIGE_OK;
}

// The opt-in host copy of the counts: enqueued after the kernel, then the
// stream is synchronised.  A capturing stream cannot be synchronised, so a
// request during capture is refused before anything is enqueued.
static int check_host_counts(const int32_t *host_counts, sige_stream_t stream)
{
    if (!host_counts)
        return SIGE_OK;
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing((cudaStream_t)stream, &cs) != cudaSuccess)
        return SIGE_ERR_CUDA;
    return cs == cudaStreamCaptureStatusNone ? SIGE_OK : SIGE_ERR_INVALID_ARG;
}

static int copy_host_counts(int st, int32_t *host_counts, const int32_t *counts, int32_t n_scales,
                            sige_stream_t stream)
{
    if (st != SIGE_OK || !host_counts)
        return st;
    if (cudaMemcpyAsync(host_counts, counts, sizeof(int32_t) * (size_t)n_scales, cudaMemcpyDeviceToHost,
                        (cudaStream_t)stream) != cudaSuccess ||
        cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess)
        return SIGE_ERR_CUDA;
    return SIGE_OK;
}

static int reduce_mask_impl(const void *a_orig, const void *a_edit, const sige_tensor_desc *in, float threshold,
                            int32_t dilate, int32_t radius, int32_t n_scales, const sige_scale_desc *scales,
                            int32_t *idx, int32_t *counts, int32_t *host_counts, void *workspace,
                            size_t workspace_bytes, sige_stream_t stream)
{
    int vs = validate_mask_args(a_orig, a_edit, in, threshold, dilate, radius, n_scales, scales, idx, counts);
    if (vs != SIGE_OK)
        return vs;
    const size_t need = kWsHeader + flag_bytes_of(n_scales, scales);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 15))
        return SIGE_ERR_WORKSPACE;
    vs = check_host_counts(host_counts, stream);
    if (vs != SIGE_OK)
        return vs;

    MaskParams p{};
    p.a = static_cast<const uint8_t *>(a_orig);
    p.b = static_cast<const uint8_t *>(a_edit);
    p.N = in->n; p.H = in->h; p.W = in->w; p.C = in->c;
    p.dtype = in->dtype; p.layout = in->layout;
    p.thr = threshold;
    p.dilate = dilate;
    p.radius = radius;
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
        o.log_h = log2_exact(o.tile_h);
        o.log_w = log2_exact(o.tile_w);
        o.fy = in->h / q.h;
        o.fx = in->w / q.w;
        o.hs = q.h;
        o.ws = q.w;
        foff += (int32_t)align16((size_t)o.th * o.tw);
        ioff += q.capacity;
    }
    p.idx = idx;
    p.counts = counts;
    p.hdr = static_cast<WsHeader *>(workspace);
    p.flags = static_cast<uint8_t *>(workspace) + kWsHeader;
    p.flag_bytes = foff;
    p.wait_cycles = wait_cycles_or(kMaskWaitCycles);

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
    p.log_vpp = p.mode == 0 ? log2_exact(p.vpp) : 0;
    p.log_w = log2_exact(in->w);
    p.log_epv = log2_exact(p.epv);
    p.pow2 = p.log_vpp >= 0 && p.log_w >= 0 && log2_exact(in->h) >= 0;
    // CTA 0 reduces; the others stream the inputs, one per SM
    const int workers_max = std::max(1, device_sm_count() - 1);
    int grid;
    size_t smem;
    if (p.mode == 2) {
        grid = 1 + (int)std::min<int64_t>((p.nwork + kMaskThreads * kScalarPerThread - 1) / (kMaskThreads * kScalarPerThread), workers_max);
        smem = 2 * kMaxWords * sizeof(uint32_t);
    } else {
        // chunks of 256..1024 vectors, about four per streaming CTA
        int64_t chunk = (p.nwork / ((int64_t)workers_max * 4) + 255) / 256 * 256;
        chunk = std::max<int64_t>(256, std::min<int64_t>(kMaskChunkMax, chunk));
        p.chunk = (int32_t)chunk;
        const int64_t nchunks = (p.nwork + chunk - 1) / chunk;
        p.nchunks = (int32_t)nchunks;
        grid = 1 + (int)std::min<int64_t>(nchunks, workers_max);
        smem = std::max(kMaskStreamSmem, 2 * kMaxWords * sizeof(uint32_t));
    }
    static std::atomic<int> attr_done[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(k_mask_reduce, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaskStreamSmem) !=
            cudaSuccess)
            return SIGE_ERR_CUDA;
        attr_done[dev].store(1, std::memory_order_release);
    }
    prefer_max_shared(k_mask_reduce);
    const cudaError_t e = launch_pdl(k_mask_reduce, dim3(grid), dim3(kMaskThreads), smem, (cudaStream_t)stream, p);
    count_launch();
    if (e != cudaSuccess)
        return SIGE_ERR_CUDA;
    return copy_host_counts(launch_check(), host_counts, counts, n_scales, stream);
}

extern "C" int sige_reduce_mask(const void *a_orig, const void *a_edit, const sige_tensor_desc *in,
                                float threshold, int32_t dilate, int32_t n_scales,
                                const sige_scale_desc *scales, int32_t *idx, int32_t *counts,
                                int32_t *host_counts, void *workspace, size_t workspace_bytes,
                                sige_stream_t stream)
{
    return reduce_mask_impl(a_orig, a_edit, in, threshold, dilate, 0, n_scales, scales, idx, counts, host_counts,
                            workspace, workspace_bytes, stream);
}

extern "C" int sige_reduce_mask_px(const void *a_orig, const void *a_edit, const sige_tensor_desc *in,
                                   float threshold, int32_t radius, int32_t n_scales,
                                   const sige_scale_desc *scales, int32_t *idx, int32_t *counts,
                                   int32_t *host_counts, void *workspace, size_t workspace_bytes,
                                   sige_stream_t stream)
{
    return reduce_mask_impl(a_orig, a_edit, in, threshold, 0, radius, n_scales, scales, idx, counts, host_counts,
                            workspace, workspace_bytes, stream);
}

// ------------------------------------------------------------------ variant without a workspace
//
// The same reduction for callers that cannot hand the library a device
// workspace: processes that reserve all device memory up front and allow no
// further allocation, plugin interfaces that expose no allocator, or bindings
// that only forward the tensors they were given.  Its scratch (the header and
// the per-scale tile flags) lives in this file-scope array instead.  Every
// GPU that loads the library holds the array until the process exits, and
// every call on a device shares it.

namespace sige {

constexpr size_t kStaticScratchBytes = 64 * 1024;
static __device__ __align__(256) uint8_t g_mask_scratch[kStaticScratchBytes];

// The array's name is only a host-side stand-in; its device address is looked
// up once per device, with that device current, and kept for the life of the
// process (it does not survive a cudaDeviceReset of that device).
static void *static_scratch_address(int &status)
{
    static std::mutex mu;
    static void *addr[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        status = SIGE_ERR_CUDA;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_mask_scratch) != cudaSuccess || !p) {
            status = SIGE_ERR_CUDA;
            return nullptr;
        }
        addr[dev] = p;
    }
    status = SIGE_OK;
    return addr[dev];
}

} // namespace sige

extern "C" int sige_reduce_mask_static(const void *a_orig, const void *a_edit, const sige_tensor_desc *in,
                                       float threshold, int32_t dilate, int32_t n_scales,
                                       const sige_scale_desc *scales, int32_t *idx, int32_t *counts,
                                       sige_stream_t stream)
{
    // every argument check first: nothing is enqueued for an invalid call
    int st = validate_mask_args(a_orig, a_edit, in, threshold, dilate, 0, n_scales, scales, idx, counts);
    if (st != SIGE_OK)
        return st;
    const size_t need = kWsHeader + flag_bytes_of(n_scales, scales);
    if (need > kStaticScratchBytes)
        return SIGE_ERR_WORKSPACE;   // more tiles than the built-in scratch holds
    void *scratch = static_scratch_address(st);
    if (!scratch)
        return st;
    // The kernel needs its flags and arrival counter at zero on entry (an
    // earlier call that failed part-way could have left them otherwise).  The
    // counts start at -1: the kernel overwrites them only when the reduction
    // completes, so a call that recorded a device error (which no caller can
    // read here: the header lives in the shared array and the next call clears
    // it) leaves negative counts behind.
    if (cudaMemsetAsync(scratch, 0, need, (cudaStream_t)stream) != cudaSuccess ||
        cudaMemsetAsync(counts, 0xFF, sizeof(int32_t) * (size_t)n_scales, (cudaStream_t)stream) != cudaSuccess)
        return SIGE_ERR_CUDA;
    return reduce_mask_impl(a_orig, a_edit, in, threshold, dilate, 0, n_scales, scales, idx, counts, nullptr,
                            scratch, need, stream);
}
