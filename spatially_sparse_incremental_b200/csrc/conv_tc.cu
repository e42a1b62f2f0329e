// Layer F_l on the 5th-generation tensor cores (tcgen05, bf16 operands,
// float32 accumulation in tensor memory) for the stacked halo'd blocks of the
// SIGE tile-based sparse convolution (SIGE project page, "Overview": gather the
// active blocks with their halo, stack them on the batch axis, run F_l,
// scatter the output blocks into the cached F_l(A_original)).
//
// The conv is an implicit GEMM D[c_out][pixel] = sum_K W[c_out][K] * X[pixel][K]
// with K = (tap, c_in):
//   * A = the weights, [C_out][k*k*C_in] K-major, 128 output channels per
//     tile, moved by TMA into 128-byte-swizzled shared memory, 64 input
//     channels (one "k-chunk" = one tap x 64 channels) per pipeline stage;
//   * B = the pixels.  Each B stage holds, for 64 input channels, the whole
//     halo'd input block of every tile of the work unit, in the no-swizzle
//     K-major core-matrix layout (8 rows x 16 bytes).  The tap (r, c) of the
//     3x3 (or k x k) window is then only an offset of the B descriptor's start
//     address: the halo is read from global memory once per 64 channels and
//     reused by all k*k taps inside shared memory;
//   * D lives in tensor memory: lane = output channel, column = pixel.
// Three B layouts:
//   ROW (b = 8, stride 1): an N-group of 8 rows is one output row of a tile,
//     i.e. 8 consecutive halo pixels; one MMA per (tile, tap, 16 channels),
//     N = 64 (the tile's 8 x 8 pixels).
//   Row-batched POS (even b otherwise): units of 8 tiles stored
//     [halo row][halo col][channel group][slot]; an N-group of 8 rows is the 8
//     tiles at one halo pixel, the next N-group the next output pixel of the
//     row (s halo columns on), so one MMA covers an output row of all 8 tiles,
//     N = 8 b.
//   POS (odd b): an N-group of 8 rows is 8 tiles at the same halo position;
//     one MMA per (output position (i, j), tap, 16 channels), N = the number
//     of tiles of the unit (16..256).
// The producers apply the GroupNorm affine + SiLU (and the zero padding
// outside the image) while moving the halo into shared memory; the epilogue
// adds bias and residual and rounds once into the cached output, or writes
// float32 output blocks.  When the active tiles are too few to fill the GPU,
// the K loop is split over several CTAs.  The kernel is launched in clusters
// of two CTAs, or of four where one tile would split K at least 4 ways (the
// split is then a power of two dividing 4).  A 2-way split of a unit of at
// most 64 columns in clusters of two is summed through the peer's shared
// memory (rank 1 sends its partial to rank 0, which adds its own and runs the
// epilogue).  A split that divides the cluster size reduce-scatters inside
// the cluster: member q of the tile group receives column slice q of every
// member's partial in its freed halo stages, sums them in member order and
// writes that slice.  Any other split ends with the last CTA of a tile group
// summing the partials from global memory in a fixed order.  The sums are
// deterministic in every case.
//
// Warp roles (320 threads): warp 0 issues the weight TMA, warp 1 allocates
// tensor memory and issues the MMAs, warps 2-9 stage the halo and run the
// epilogue.  Warps 0 and 1 run warp-uniform loops and one lane, chosen by
// elect.sync, issues each TMA / MMA / commit.  Every mbarrier wait is bounded;
// on expiry the kernel records SIGE_ERR_TIMEOUT in the workspace header and
// unwinds.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "conv_tc.cuh"
#include "tc_ptx.cuh"
#include "transform.cuh"

namespace sige {

constexpr int kTcThreads = 320;              // warp 0 TMA, warp 1 MMA, warps 2-9 halo + epilogue
constexpr int kProd = 256;                    // halo / epilogue threads
constexpr uint32_t kAStageBytes = 128 * 64 * 2;
constexpr int kMaxSplit = 32;
constexpr int kSmemLimit = 232448;             // 227 KB opt-in per CTA
constexpr int kMaxSA = 16;                     // weight stages at most
constexpr uint32_t kCtrlBytes = 4096;          // barriers, flags, tile origins
constexpr uint32_t kRedBytes = 64 * 128 * 4;   // split-K partial of one unit received from the cluster peer

// Flat argument block.  The kernel copies it into a local at entry: fields of
// a kernel parameter read through a reference (non-inlined helpers, or after an
// asm "memory" clobber) become slow generic loads, a local copy stays in
// registers.
struct TcArgs {
    // layer
    const uint8_t *src;       // stacked blocks (from_image == 0) or NHWC image
    const int32_t *idx;
    const int32_t *count;
    const float *gsc, *gsh;
    const float *bias;
    const uint8_t *residual;
    uint8_t *y;
    float *out_blocks;
    uint8_t *ws;
    uint32_t *counters;       // per tile group arrival counters (split K)
    float *partials;          // [slab][ncols][128] float32
    int32_t N, H, W, Cin, Cout, dtype;
    int32_t k, s, pad, b, bin, Ho, Wo;
    int32_t cap, dense, tiles_w, tiles_total;
    int32_t silu, from_image, to_y;
    const uint8_t *sg, *sb;   // per-pixel modulation maps (NHWC, input shape) or null
    int32_t leaky;            // LeakyReLU(0.2) after the transform
    int32_t tstride;          // > 0: transposed conv of this stride (virtual zero-inserted input, taps reversed)
    // schedule / shared-memory plan
    int32_t mode;             // 0 = ROW, 1 = POS, 2 = POS with 8 slots and one MMA per output row
    int32_t taps, kci;        // k*k, C_in / 64
    int32_t MT;               // output-channel tiles of 128
    int32_t T_max;            // ROW: tiles per unit; POS: slots (multiple of 16)
    int32_t SB;               // halo stages (the weight stage count is set per launch from the unit size)
    uint32_t per_slot;        // bytes of one tile (ROW) or slot (POS) per halo stage
    uint32_t smem_bytes;      // dynamic shared memory of the launch
    int32_t ncols;            // tensor-memory columns allocated (power of 2)
    int32_t num_sms;
    int32_t halo_tma;         // 1: ROW-mode halo rows come by TMA (tmx), 0: per-thread cp.async
    int32_t pair;             // 1: launched in clusters (of csize CTAs)
    UDiv dN, dbin, db;        // division by N, bin and b in the per-element loops
    int32_t csize;            // CTAs per cluster (1: no clusters).  csize 2: a 2-way K split of
                              // a unit of <= 64 columns is summed through the peer's shared
                              // memory; other splits that divide csize reduce-scatter within
                              // the cluster; the rest go through global memory
};

__device__ __forceinline__ void tile_origin_a(const TcArgs &a, int t, int &h0, int &w0)
{
    if (a.dense) {
        h0 = (t / a.tiles_w) * a.b;
        w0 = (t % a.tiles_w) * a.b;
    } else {
        const int2 o = __ldg(reinterpret_cast<const int2 *>(a.idx) + t);
        h0 = o.x;
        w0 = o.y;
    }
}

// ------------------------------------------------------------------ schedule

struct Sched {
    UDiv dT;    // division by T
    int T;      // tiles per unit (POS: slots, multiple of 16)
    int TB;     // tile groups
    int S;      // K splits
    int units;
};

// Units of work for G tiles: tile groups of T tiles (slots) x output-channel
// tiles x K splits.  In clusters of csize >= 4 the split is a power of two that
// divides csize, so that all splits of a tile group sit in one cluster.
__host__ __device__ inline Sched make_sched_for(int mode, int T_max, int MT, int KC, int num_sms, int csize, int G)
{
    Sched s;
    const int want = max(1, (G * MT + num_sms - 1) / num_sms);
    if (mode == 0)
        s.T = min(T_max, want);
    else if (mode == 2)
        s.T = 8;
    else
        s.T = min(T_max, ((want + 15) / 16) * 16);
    s.TB = (G + s.T - 1) / s.T;
    s.dT = udiv_make((uint32_t)s.T);
    // split K only where each split keeps a long K loop: below that the extra
    // round trip of the partial sums costs more than the shorter loop saves
    s.S = max(1, min(num_sms / max(1, s.TB * MT), min(KC / 8, kMaxSplit)));
    if (csize >= 4) {
        int q = 1;
        while (2 * q <= min(s.S, csize))
            q *= 2;
        s.S = q;
    }
    s.units = s.TB * MT * s.S;
    return s;
}

__device__ __forceinline__ Sched make_sched(const TcArgs &p, int G)
{
    return make_sched_for(p.mode, p.T_max, p.MT, p.taps * p.kci, p.num_sms, p.csize, G);
}

struct Unit {
    int tb, mt, split, kb, ke;
};

__device__ __forceinline__ Unit decode_unit(const TcArgs &p, const Sched &s, int u)
{
    Unit r;
    r.split = u % s.S;
    const int tm = u / s.S;
    r.mt = tm % p.MT;
    r.tb = tm / p.MT;
    const int KC = p.taps * p.kci;   // small: 32-bit products
    r.kb = r.split * KC / s.S;
    r.ke = (r.split + 1) * KC / s.S;
    return r;
}

// ------------------------------------------------------------------ shared-memory carve-up
//
//   [0, 1024)        mbarriers and control words
//   [1024, 3072)     tile origins of the current unit (256 x int2)
//   [4096, ...)      weight stages, 16 KB each, as many as fit (<= 16)
//   [.., b_base)     clusters of two only: the 32 KB receive buffer of the
//                    split-K partial sent by the cluster peer
//   [b_base, end)    SB halo stages of T slots each; reused as the epilogue's
//                    staging buffer, or as the reduce-scatter's receive area,
//                    once the unit's MMAs are complete

// Accumulator columns of a unit of T tiles (ROW) or T slots (POS).
__host__ __device__ inline int unit_cols(const TcArgs &p, int T)
{
    return p.mode == 0 ? T * 64 : p.b * p.b * T;
}

struct Carve {
    uint32_t a_base;    // byte offset of weight stage 0
    uint32_t b_base;    // byte offset of halo stage 0
    uint32_t stage_b;   // bytes per halo stage
    uint32_t red_base;  // receive buffer of the peer's partial (kRedBytes), when red
    bool red;           // clusters of two, unit of <= 64 columns, and two weight stages still fit
    int SA;             // weight stages
};

__host__ __device__ inline Carve carve(const TcArgs &p, int T)
{
    Carve c;
    c.stage_b = (uint32_t)T * p.per_slot;
    c.b_base = (p.smem_bytes - 1024 - p.SB * c.stage_b) & ~15u;
    c.a_base = kCtrlBytes;
    c.red_base = c.b_base;
    c.red = false;
    if (p.csize == 2 && unit_cols(p, T) * 512 <= (int)kRedBytes && c.b_base >= kRedBytes + 1024) {
        const uint32_t rb = (c.b_base - kRedBytes) & ~1023u;
        if (rb >= c.a_base + 2 * kAStageBytes) {
            c.red_base = rb;
            c.red = true;
        }
    }
    c.SA = min(kMaxSA, (int)((c.red_base - c.a_base) / kAStageBytes));
    return c;
}

// How the K splits of a unit are summed (the same for every CTA of a launch).
enum : int { kSplitNone = 0, kSplitPair = 1, kSplitCluster = 2, kSplitGlobal = 3 };

__host__ __device__ inline int split_kind(const TcArgs &p, const Sched &sc, const Carve &cv)
{
    const int ncols = unit_cols(p, sc.T);
    if (sc.S == 1)
        return kSplitNone;
    // 2-way split through the cluster peer's receive buffer
    if (cv.red && sc.S == 2)
        return kSplitPair;
    // reduce-scatter among the S CTAs of the tile group (consecutive ranks of
    // one cluster), the slices staged in the halo stages, which are free by then
    if (p.csize >= 2 && p.csize % sc.S == 0 && (ncols / sc.S) % 4 == 0 &&
        (uint32_t)ncols * 512u <= (uint32_t)p.SB * cv.stage_b)
        return kSplitCluster;
    return kSplitGlobal;
}

// ------------------------------------------------------------------ B staging

// Byte offset of (tile slot, halo row, halo col, 16-byte channel group) in a B stage.
__device__ __forceinline__ uint32_t b_offset(const TcArgs &p, int slots, int slot, int hh, int ww, int kc)
{
    const int bin = p.bin;
    if (p.mode == 0)  // [slot][hh][kc][ww][16 B]
        return (uint32_t)((((slot * bin + hh) * 8 + kc) * bin + ww) * 16);
    // [hh][ww][kc][slot][16 B]
    return (uint32_t)((((hh * bin + ww) * 8 + kc) * slots + slot) * 16);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Batch item of stacked item g (tile-major, item-minor).
__device__ __forceinline__ int item_of(const TcArgs &c, int g)
{
    return c.N == 1 ? 0 : g - (int)udiv((uint32_t)g, c.dN) * c.N;
}

// Source of one 16-byte halo chunk, or nullptr where the conv's zero padding
// (or a tile past the list) applies.
__device__ __forceinline__ const uint8_t *halo_src(const TcArgs &c, const int2 *s_orig, int T, int tb, int G, int slot,
                                                   int hh, int ww, int pix, int ch)
{
    const int g = tb * T + slot;
    if (g >= G)
        return nullptr;
    if (!c.from_image)
        return c.src + (((int64_t)g * c.bin * c.bin + pix) * c.Cin + ch) * 2;
    const int2 o = s_orig[slot];
    int y = o.x * c.s - c.pad + hh, x = o.y * c.s - c.pad + ww;
    if (c.tstride > 0) {
        // transposed conv: pixel (y, x) of the virtual input holds x[y / t][x / t]
        // where both are multiples of t, and zero elsewhere
        if (y < 0 || x < 0 || y % c.tstride || x % c.tstride)
            return nullptr;
        y /= c.tstride;
        x /= c.tstride;
    }
    if (y < 0 || y >= c.H || x < 0 || x >= c.W)
        return nullptr;
    return c.src + ((((int64_t)item_of(c, g) * c.H + y) * c.W + x) * c.Cin + ch) * 2;
}

// The input transform of the GauGAN-style layers, for 8 bf16 channels of one
// pixel whose bytes sit at `off` in the input: GroupNorm-style affine of batch
// item n (when set), the per-pixel modulation t * (1 + sg) + sb (when set),
// then SiLU or LeakyReLU(0.2); one rounding to bf16.
__device__ __noinline__ uint4 transform16_ext(const TcArgs &c, uint4 in, int64_t off, int n, int ch)
{
    const uint32_t *w = reinterpret_cast<const uint32_t *>(&in);
    const uint4 z = make_uint4(0, 0, 0, 0);
    const uint4 gv = c.sg ? __ldg(reinterpret_cast<const uint4 *>(c.sg + off)) : z;
    const uint4 bv = c.sb ? __ldg(reinterpret_cast<const uint4 *>(c.sb + off)) : z;
    const uint32_t *g = reinterpret_cast<const uint32_t *>(&gv);
    const uint32_t *b = reinterpret_cast<const uint32_t *>(&bv);
    uint4 out;
    uint32_t *o = reinterpret_cast<uint32_t *>(&out);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float v[2] = {bf16_lo(w[q]), bf16_hi(w[q])};
        const float gg[2] = {bf16_lo(g[q]), bf16_hi(g[q])};
        const float bb[2] = {bf16_lo(b[q]), bf16_hi(b[q])};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int k = ch + 2 * q + e;
            if (c.gsc)
                v[e] = __fmaf_rn(v[e], __ldg(c.gsc + (int64_t)n * c.Cin + k), __ldg(c.gsh + (int64_t)n * c.Cin + k));
            if (c.sg)
                v[e] = __fmaf_rn(v[e], 1.0f + gg[e], bb[e]);
            if (c.silu)
                v[e] = silu_f(v[e]);
            else if (c.leaky)
                v[e] = v[e] >= 0.0f ? v[e] : 0.2f * v[e];
        }
        o[q] = pack_bf16x2(v[0], v[1]);
    }
    return out;
}

// Fill one B stage: 64 input channels (chunk q) of the halo of every tile of
// the unit, in the core-matrix layout.  Every chunk is one 16-byte cp.async
// (zero-filled for padding), all in flight at once; then the GroupNorm affine
// and SiLU are applied in place.  Thread et always handles channel group
// kc = et & 7 and pixels (et >> 3) + (kProd / 8) k, walked incrementally.
__device__ __forceinline__ void fill_b(const TcArgs &c, int T, int tb, int q, int G, uint8_t *stage, int et,
                                       const int2 *s_orig)
{
    const int bin = c.bin, bin2 = bin * bin;
    const int kc = et & 7;
    const int ch = q * 64 + kc * 8;
    const uint32_t sbase = smem_u32(stage);
    const int lin0 = et >> 3;
    const int slot0 = lin0 / bin2, pix0 = lin0 - slot0 * bin2;
    const int hh0 = pix0 / bin, ww0 = pix0 - hh0 * bin;
    {
        int slot = slot0, hh = hh0, ww = ww0;
#pragma unroll 1
        while (slot < T) {
            const uint8_t *src = halo_src(c, s_orig, T, tb, G, slot, hh, ww, hh * bin + ww, ch);
            cp_async16(sbase + b_offset(c, T, slot, hh, ww, kc), src ? src : c.src, src ? 16u : 0u);
            ww += kProd / 8;
            while (ww >= bin) {
                ww -= bin;
                if (++hh == bin) {
                    hh = 0;
                    ++slot;
                }
            }
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (c.gsc == nullptr && !c.silu && !c.sg && !c.leaky)
        return;
    const bool ext = c.sg != nullptr || c.leaky;
    float gsc[8], gsh[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        gsc[k] = 1.0f;
        gsh[k] = 0.0f;
    }
    const bool affine = c.gsc != nullptr;
    if (affine && c.N == 1) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            gsc[k] = __ldg(c.gsc + ch + k);
            gsh[k] = __ldg(c.gsh + ch + k);
        }
    }
    int slot = slot0, hh = hh0, ww = ww0;
#pragma unroll 1
    while (slot < T) {
        if (const uint8_t *src = halo_src(c, s_orig, T, tb, G, slot, hh, ww, hh * bin + ww, ch)) {
            uint4 *d = reinterpret_cast<uint4 *>(stage + b_offset(c, T, slot, hh, ww, kc));
            if (ext) {
                *d = transform16_ext(c, *d, src - c.src, item_of(c, tb * T + slot), ch);
            } else if (affine && c.N > 1) {
                const int n = item_of(c, tb * T + slot);
                *d = transform16(*d, SIGE_BF16, c.gsc + (int64_t)n * c.Cin + ch, c.gsh + (int64_t)n * c.Cin + ch,
                                 c.silu);
            } else {
                *d = transform16_bf16_reg(*d, gsc, gsh, affine, c.silu);
            }
        }
        ww += kProd / 8;
        while (ww >= bin) {
            ww -= bin;
            if (++hh == bin) {
                hh = 0;
                ++slot;
            }
        }
    }
}

// Fill one B stage of the slot layouts (POS and row-batched POS), whose bytes
// run [halo pixel][channel group][slot]: 16-byte chunk `lin` of the stage sits
// at byte 16 lin, so thread et copies chunks et, et + 256, ...  A warp then
// writes 512 contiguous bytes of shared memory (no bank conflicts) and reads
// 64 contiguous bytes from each of 8 tiles.  Then the GroupNorm affine and
// SiLU are applied in place, in the same order.
__device__ __forceinline__ void fill_b_slots(const TcArgs &c, int T, UDiv dT, int tb, int q, int G, uint8_t *stage,
                                             int et, const int2 *s_orig)
{
    const int bin = c.bin;
    const int total = bin * bin * 8 * T;
    const uint32_t sbase = smem_u32(stage);
#pragma unroll 1
    for (int lin = et; lin < total; lin += kProd) {
        const int r = (int)udiv((uint32_t)lin, dT), slot = lin - r * T;
        const int kc = r & 7, pix = r >> 3;
        const int hh = (int)udiv((uint32_t)pix, c.dbin), ww = pix - hh * bin;
        const uint8_t *src = halo_src(c, s_orig, T, tb, G, slot, hh, ww, pix, q * 64 + kc * 8);
        cp_async16(sbase + (uint32_t)lin * 16u, src ? src : c.src, src ? 16u : 0u);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (c.gsc == nullptr && !c.silu && !c.sg && !c.leaky)
        return;
    const bool affine = c.gsc != nullptr;
    const bool ext = c.sg != nullptr || c.leaky;
#pragma unroll 1
    for (int lin = et; lin < total; lin += kProd) {
        const int r = (int)udiv((uint32_t)lin, dT), slot = lin - r * T;
        const int kc = r & 7, pix = r >> 3;
        const int hh = (int)udiv((uint32_t)pix, c.dbin), ww = pix - hh * bin;
        const int ch = q * 64 + kc * 8;
        const uint8_t *src = halo_src(c, s_orig, T, tb, G, slot, hh, ww, pix, ch);
        if (!src)
            continue;   // zero padding stays zero
        uint4 *d = reinterpret_cast<uint4 *>(stage + (size_t)lin * 16);
        const int n = (affine || ext) ? item_of(c, tb * T + slot) : 0;
        if (ext)
            *d = transform16_ext(c, *d, src - c.src, n, ch);
        else
            *d = transform16(*d, SIGE_BF16, affine ? c.gsc + (int64_t)n * c.Cin + ch : nullptr,
                             affine ? c.gsh + (int64_t)n * c.Cin + ch : nullptr, c.silu);
    }
}

// GroupNorm scale / shift of this thread's 8 channels of chunk q (batch 1);
// loaded before the halo wait so that their latency overlaps the copy.
__device__ __forceinline__ void load_gn8(const TcArgs &c, int q, int et, float (&gsc)[8], float (&gsh)[8])
{
    const int ch = q * 64 + (et & 7) * 8;
    const bool affine = c.gsc != nullptr && c.N == 1;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        gsc[k] = affine ? __ldg(c.gsc + ch + k) : 1.0f;
        gsh[k] = affine ? __ldg(c.gsh + ch + k) : 0.0f;
    }
}

// In-place GroupNorm affine + SiLU of a B stage whose raw halo arrived by TMA
// (zero-filled outside the image); padding entries are left at zero.  gsc /
// gsh come from load_gn8 (batch 1; larger batches read theirs per tile).
__device__ __forceinline__ void transform_b(const TcArgs &c, int T, int tb, int q, int G, uint8_t *stage, int et,
                                            const int2 *s_orig, const float (&gsc)[8], const float (&gsh)[8])
{
    if (c.gsc == nullptr && !c.silu)
        return;
    const int bin = c.bin, bin2 = bin * bin;
    const int kc = et & 7;
    const int ch = q * 64 + kc * 8;
    const bool affine = c.gsc != nullptr;
    const int lin0 = et >> 3;
    int slot = lin0 / bin2, pix = lin0 - slot * bin2;
    int hh = pix / bin, ww = pix - hh * bin;
#pragma unroll 1
    while (slot < T) {
        if (halo_src(c, s_orig, T, tb, G, slot, hh, ww, hh * bin + ww, ch)) {
            uint4 *d = reinterpret_cast<uint4 *>(stage + b_offset(c, T, slot, hh, ww, kc));
            if (affine && c.N > 1) {
                const int n = item_of(c, tb * T + slot);
                *d = transform16(*d, SIGE_BF16, c.gsc + (int64_t)n * c.Cin + ch, c.gsh + (int64_t)n * c.Cin + ch,
                                 c.silu);
            } else {
                *d = transform16_bf16_reg(*d, gsc, gsh, affine, c.silu);
            }
        }
        ww += kProd / 8;
        while (ww >= bin) {
            ww -= bin;
            if (++hh == bin) {
                hh = 0;
                ++slot;
            }
        }
    }
}

// ------------------------------------------------------------------ epilogue


// Pixel of accumulator column `col`: returns the flat element index of its
// first channel `co0` in the destination, or -1 when the column is not a
// pixel to write (past the list, outside the image).
__device__ __forceinline__ int64_t col_target(const TcArgs &c, const int2 *s_orig, const Sched &sc, int tb, int G,
                                              int col, int co0)
{
    const int T = sc.T;
    int slot, i, j;
    if (c.mode == 0) {
        slot = col >> 6;
        i = (col >> 3) & 7;
        j = col & 7;
    } else {
        const int pos = (int)udiv((uint32_t)col, sc.dT);
        slot = col - pos * T;
        i = (int)udiv((uint32_t)pos, c.db);
        j = pos - i * c.b;
    }
    const int g = tb * T + slot;
    if (g >= G)
        return -1;
    if (c.to_y) {
        const int2 o = s_orig[slot];
        const int yo = o.x + i, xo = o.y + j;
        if (yo >= c.Ho || xo >= c.Wo)
            return -1;
        return (((int64_t)item_of(c, g) * c.Ho + yo) * c.Wo + xo) * c.Cout + co0;
    }
    return (((int64_t)g * c.b + i) * c.b + j) * c.Cout + co0;
}

// Write 8 (bf16) or 4 (float32) consecutive channels of one pixel: bias,
// residual (already loaded: rw), one rounding, one 16-byte store.
__device__ __forceinline__ void store_vec(const TcArgs &c, int64_t e, const float *v, const float *bias8, uint4 rw)
{
    if (!c.to_y) {
        *reinterpret_cast<float4 *>(c.out_blocks + e) = make_float4(v[0], v[1], v[2], v[3]);
        return;
    }
    if (c.dtype == SIGE_BF16) {
        const float r[8] = {bf16_lo(rw.x), bf16_hi(rw.x), bf16_lo(rw.y), bf16_hi(rw.y),
                            bf16_lo(rw.z), bf16_hi(rw.z), bf16_lo(rw.w), bf16_hi(rw.w)};
        uint4 o;
        o.x = pack_bf16x2((v[0] + bias8[0]) + r[0], (v[1] + bias8[1]) + r[1]);
        o.y = pack_bf16x2((v[2] + bias8[2]) + r[2], (v[3] + bias8[3]) + r[3]);
        o.z = pack_bf16x2((v[4] + bias8[4]) + r[4], (v[5] + bias8[5]) + r[5]);
        o.w = pack_bf16x2((v[6] + bias8[6]) + r[6], (v[7] + bias8[7]) + r[7]);
        *reinterpret_cast<uint4 *>(c.y + e * 2) = o;
    }
}

// ------------------------------------------------------------------ kernel

__global__ void __launch_bounds__(kTcThreads, 1)
    k_conv_tc(const __grid_constant__ TcArgs args, const __grid_constant__ CUtensorMap tmw,
              const __grid_constant__ CUtensorMap tmx)
{
    const TcArgs p = args;   // registers, see TcArgs
    const TcArgs &c = p;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw_addr + 1023) & ~1023u) - raw_addr);
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase;
    auto a_full = [&](int i) { return bar0 + 8u * i; };
    auto a_empty = [&](int i) { return bar0 + 8u * (kMaxSA + i); };
    auto b_full = [&](int i) { return bar0 + 8u * (2 * kMaxSA + i); };
    auto b_empty = [&](int i) { return bar0 + 8u * (2 * kMaxSA + 2 + i); };
    const uint32_t acc_full = bar0 + 8u * (2 * kMaxSA + 4);
    const uint32_t acc_empty = acc_full + 8u;
    const uint32_t drain = acc_full + 16u;
    auto b_load = [&](int i) { return acc_full + 24u + 8u * i; };   // halo TMA arrivals
    const uint32_t red_full = acc_full + 40u;   // pair launches, rank 0: the peer's partial has arrived
    const uint32_t red_free = acc_full + 48u;   // pair launches, rank 1: the peer has consumed it
    const uint32_t rs_ready = acc_full + 56u;   // reduce-scatter: every member of the group may be written
    const uint32_t rs_full = acc_full + 64u;    // reduce-scatter: every member's slice for this CTA has landed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + 512);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + 516);
    volatile int *bcast = abort_flag + 1;
    volatile int *group_ok = abort_flag + 2;
    int2 *s_orig = reinterpret_cast<int2 *>(smem + 1024);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaxSA; ++i) {
            mbar_init(a_full(i), 1);
            mbar_init(a_empty(i), 1);
        }
        for (int i = 0; i < p.SB; ++i) {
            mbar_init(b_full(i), kProd);
            mbar_init(b_empty(i), 1);
            mbar_init(b_load(i), 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, kProd);
        mbar_init(drain, 1);
        mbar_init(red_full, 1);
        mbar_init(red_free, 1);
        // reduce-scatter: each of the S members arrives with weight csize / S
        mbar_init(rs_ready, max(1, p.csize));
        mbar_init(rs_full, max(1, p.csize));
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmw)) : "memory");
        if (args.halo_tma)
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmx)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(p.ncols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // the barriers of both CTAs of a pair are initialised before either side's
    // first remote access (each waits on this cluster barrier before it)
    bool cwaited = false;
    if (p.pair)
        cluster_arrive();
    // everything above touches only this CTA's own resources; the tile list,
    // the activations and the output may come from the kernel before
    pdl_trigger();
    pdl_wait();
    if (threadIdx.x == 64 && !c.dense) {
        // the tile origins this CTA reads first, for K split in 1 or 2
        const int32_t *i0 = c.idx + 2 * min(c.cap - 1, (int)blockIdx.x);
        const int32_t *i1 = c.idx + 2 * min(c.cap - 1, (int)blockIdx.x / 2);
        if (c.cap > 0) {
            asm volatile("prefetch.global.L1 [%0];" ::"l"(i0));
            asm volatile("prefetch.global.L1 [%0];" ::"l"(i1));
        }
    }

    const int ntile = c.dense ? c.tiles_total : min(__ldg(c.count), c.cap);
    const int G = ntile * c.N;
    const Sched sc = make_sched(p, G);
    const Carve cv = carve(p, sc.T);

    if (warp == 0) {
        // ---------------- weight producer (TMA), whole warp, one issuing lane
        // stage index and phase advance incrementally: a runtime division per
        // k-chunk costs more than the TMA issue itself
        int s = 0;
        uint32_t ph = 1, issued = 0;
        bool ok = true;
#pragma unroll 1
        for (int u = blockIdx.x; u < sc.units && ok; u += gridDim.x) {
            const Unit un = decode_unit(p, sc, u);
            int q = un.kb / p.taps, tap = un.kb - q * p.taps;
            const int y0 = un.mt * 128;
#pragma unroll 1
            for (int kc = un.kb; kc < un.ke; ++kc) {
                if (!mbar_wait_w(a_empty(s), ph, abort_flag, hdr, 1)) {
                    ok = false;
                    break;
                }
                // a transposed conv reads its taps in reverse order
                const int wtap = c.tstride > 0 ? p.taps - 1 - tap : tap;
                tma_load_2d_w(sbase + cv.a_base + s * kAStageBytes, &tmw, a_full(s), kAStageBytes,
                              wtap * c.Cin + q * 64, y0);
                ++issued;
                if (++s == cv.SA) {
                    s = 0;
                    ph ^= 1;
                }
                if (++tap == p.taps) {
                    tap = 0;
                    ++q;
                }
            }
        }
        // every issued load must land before the CTA may exit: wait for the
        // last use of each stage
#pragma unroll 1
        for (uint32_t k = 0; k < (uint32_t)cv.SA && k < issued; ++k) {
            // the use of stage st waited on a_empty with parity w, so its
            // a_full completion has parity w ^ 1; w is ph for stages used in
            // the current round and ph ^ 1 for those before the wrap
            int st = s - 1 - (int)k;
            uint32_t full_par = ph ^ 1;
            if (st < 0) {
                st += cv.SA;
                full_par ^= 1;
            }
            const long long t0 = clock64();
            while (!mbar_try(a_full(st), full_par) && clock64() - t0 < kWaitCycles) {
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer: the whole warp runs the loop, one lane issues
        // The issue is a single serial chain, so this loop is kept to the bare
        // minimum: per k-chunk one barrier test, the MMAs and a commit.  The B
        // descriptor is built once per halo stage and moves by constant
        // offsets from tap to tap; the A descriptor moves by one stage.
        {
            int sa = 0, sb = 0;
            uint32_t pa = 0, pb = 0, uit = 0, ait = 0;
            bool ok = true;
            const int bin = c.bin, k = c.k, taps = p.taps, nT = sc.T, bb = c.b;
            // ROW: a tile's 64 pixels; POS: the unit's slots at one pixel; mode 2:
            // the 8 slots at each of an output row's b pixels (8 b rows of N)
            const int n_mma = p.mode == 0 ? 64 : p.mode == 2 ? 8 * bb : nT;
            const uint32_t idesc = idesc_bf16(n_mma);
            const uint32_t sk = p.mode == 0 ? (uint32_t)bin * 16 : (uint32_t)nT * 16;   // LBO
            const uint32_t sh = 8 * sk;      // ROW: halo row stride; POS: halo pixel stride
            // descriptor start-address steps (address >> 4)
            const uint64_t d_tile = (uint64_t)((bin * sh) >> 4);      // ROW: next tile
            const uint64_t d_ks = (uint64_t)((2 * sk) >> 4);          // next 16 channels
            const uint64_t d_col = p.mode == 0 ? 1u : (uint64_t)(sh >> 4);                 // tap column + 1
            const uint64_t d_row = p.mode == 0 ? (uint64_t)(sh >> 4) : (uint64_t)((bin * sh) >> 4);  // tap row + 1
            const uint64_t d_i = (uint64_t)((c.s * bin * sh) >> 4), d_j = (uint64_t)((c.s * sh) >> 4);  // POS
            const uint64_t a_desc0 = desc_sw128(sbase + cv.a_base);
            uint64_t a_cur = a_desc0;
#pragma unroll 1
            for (int u = blockIdx.x; u < sc.units && ok; u += gridDim.x) {
                const Unit un = decode_unit(p, sc, u);
                if (uit > 0 && !mbar_wait_w(acc_empty, (uit - 1) & 1, abort_flag, hdr, 2)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                int tap = un.kb % taps;
                uint32_t acc0 = 0;
#pragma unroll 1
                for (int kc = un.kb; kc < un.ke && ok;) {
                    // one halo stage: taps [tap, tap_end) of one 64-channel chunk
                    if (!mbar_wait_w(b_full(sb), pb, abort_flag, hdr, 3)) {
                        ok = false;
                        break;
                    }
                    const int tap_end = min(taps, tap + (un.ke - kc));
                    // N-groups of 8 rows: ROW, 8 halo pixels of a row (next group one
                    // halo row on); POS, 8 slots (next group 8 slots on); mode 2,
                    // the 8 slots at one pixel (next group the next output pixel,
                    // s halo pixels on)
                    const uint64_t b_stage = p.mode == 0
                        ? desc_plain(sbase + cv.b_base + sb * cv.stage_b, sk, sh)
                        : p.mode == 2 ? desc_plain(sbase + cv.b_base + sb * cv.stage_b, sk, (uint32_t)c.s * sh)
                                      : desc_plain(sbase + cv.b_base + sb * cv.stage_b, sk, 128);
                    int r = tap / k, cc = tap - r * k;
                    uint64_t b_tap = b_stage + (uint64_t)r * d_row + (uint64_t)cc * d_col;
                    if (p.mode == 0 && nT == 1) {
                        // one tile per unit: the whole k-chunk is one issue block
#pragma unroll 1
                        for (; tap < tap_end; ++tap, ++kc) {
                            if (!mbar_wait_w(a_full(sa), pa, abort_flag, hdr, 4)) {
                                ok = false;
                                break;
                            }
                            tc_mma4_commit_w(tmem, a_cur, b_tap, d_ks, idesc, acc0, a_empty(sa));
                            acc0 = 1;
                            ++ait;
                            if (++sa == cv.SA) {
                                sa = 0;
                                pa ^= 1;
                                a_cur = a_desc0;
                            } else {
                                a_cur += kAStageBytes >> 4;
                            }
                            if (++cc == k) {
                                cc = 0;
                                b_tap += d_row - (uint64_t)k * d_col;
                            }
                            b_tap += d_col;
                        }
                    } else {
#pragma unroll 1
                    for (; tap < tap_end; ++tap, ++kc) {
                        if (!mbar_wait_w(a_full(sa), pa, abort_flag, hdr, 4)) {
                            ok = false;
                            break;
                        }
                        // each accumulator block takes its four K steps in one
                        // issue block (per block the order is ks = 0..3)
                        if (p.mode == 0) {
                            uint64_t bt = b_tap;
#pragma unroll 1
                            for (int t = 0; t < nT; ++t, bt += d_tile)
                                tc_mma4_w(tmem + t * 64, a_cur, bt, d_ks, idesc, acc0);
                        } else if (p.mode == 2) {
                            uint64_t bi = b_tap;
                            uint32_t col = 0;
#pragma unroll 1
                            for (int i = 0; i < bb; ++i, bi += d_i, col += (uint32_t)(bb * 8))
                                tc_mma4_w(tmem + col, a_cur, bi, d_ks, idesc, acc0);
                        } else {
                            uint64_t bi = b_tap;
                            uint32_t col = 0;
#pragma unroll 1
                            for (int i = 0; i < bb; ++i, bi += d_i) {
                                uint64_t bj = bi;
#pragma unroll 1
                                for (int j = 0; j < bb; ++j, bj += d_j, col += nT)
                                    tc_mma4_w(tmem + col, a_cur, bj, d_ks, idesc, acc0);
                            }
                        }
                        acc0 = 1;
                        tc_commit_w(a_empty(sa));
                        ++ait;
                        if (++sa == cv.SA) {
                            sa = 0;
                            pa ^= 1;
                            a_cur = a_desc0;
                        } else {
                            a_cur += kAStageBytes >> 4;
                        }
                        if (++cc == k) {
                            cc = 0;
                            b_tap += d_row - (uint64_t)k * d_col;
                        }
                        b_tap += d_col;
                    }
                    }
                    if (!ok)
                        break;
                    tc_commit_w(b_empty(sb));
                    if (++sb == p.SB) {
                        sb = 0;
                        pb ^= 1;
                    }
                    tap = 0;
                }
                if (!ok)
                    break;
                tc_commit_w(acc_full);
                ++uit;
            }
            // every MMA issued by this thread must finish before tensor memory is freed
            if (ait > 0) {
                tc_commit_w(drain);
                const long long t0 = clock64();
                while (!mbar_try(drain, 0) && clock64() - t0 < kWaitCycles) {
                }
            }
            __syncwarp();
        }
    } else {
        // ---------------- halo producers + epilogue (warps 2..9)
        const int et = threadIdx.x - 64;
        const int sub = warp & 3;           // tensor-memory subpartition of this warp
        const int half = et >= 128 ? 1 : 0; // two warps per subpartition split the columns
        const int row = sub * 32 + lane;    // accumulator lane = output channel in the tile
        // One thread waits (bounded) and the group learns the outcome through a
        // named barrier, so that all 128 threads always take the same branch.
        auto group_wait = [&](uint32_t bar, uint32_t parity, int where) -> bool {
            if (et == 0)
                *group_ok = mbar_wait(bar, parity, abort_flag, hdr, where) ? 1 : 0;
            asm volatile("bar.sync 1, 256;" ::: "memory");
            const bool r = *group_ok != 0;
            asm volatile("bar.sync 1, 256;" ::: "memory");
            return r;
        };
        // the same on a barrier that a cluster peer completes (acquire at cluster scope)
        auto group_wait_c = [&](uint32_t bar, uint32_t parity, int where) -> bool {
            if (et == 0)
                *group_ok = mbar_wait_cluster(bar, parity, abort_flag, hdr, where) ? 1 : 0;
            asm volatile("bar.sync 1, 256;" ::: "memory");
            const bool r = *group_ok != 0;
            asm volatile("bar.sync 1, 256;" ::: "memory");
            return r;
        };
        uint32_t pit = 0;   // pair units done (phase of red_full / red_free)
        uint32_t rsit = 0;  // reduce-scatter units done (phase of rs_ready / rs_full)
        // output vectors: 8 bf16 channels (16 per 128-channel column) or 4 floats (32)
        const int vpc = (c.to_y && c.dtype == SIGE_BF16) ? 16 : 32;
        const int lvpc = vpc == 16 ? 4 : 5;   // log2 vpc
        const int cpv = 128 / vpc;          // channels per vector
        const int cg = et & (vpc - 1);      // this thread's vector within a column (fixed)
        float * const stage_d = reinterpret_cast<float *>(smem + cv.b_base);
        const int stage_cols = min(512, (int)((p.SB * cv.stage_b) / 512) & ~15);
        uint32_t bit = 0, uit = 0;
        bool ok = true;
        // one TMA per tile: the whole halo [hh][kc][ww][8 channels], zero outside
        // the image (issued by thread et 0 once the origins are in s_orig)
        auto issue_halo = [&](int sb, int q, int tb) {
            const uint32_t bl = b_load(sb);
            mbar_expect_tx(bl, (uint32_t)(sc.T * c.bin) * c.bin * 128u);
            const uint32_t st = smem_u32(smem + cv.b_base + sb * cv.stage_b);
#pragma unroll 1
            for (int slot = 0; slot < sc.T; ++slot) {
                const int g = tb * sc.T + slot;
                const int gg = g < G ? g : G - 1;   // past the list: any valid tile, unused
                const int2 o = s_orig[slot];
                const int x1 = c.from_image ? o.y * c.s - c.pad : 0;
                const int y0 = c.from_image ? o.x * c.s - c.pad : 0;
                const int n = c.from_image ? item_of(c, gg) : gg;
                tma_load_5d(st + b_offset(c, sc.T, slot, 0, 0, 0), &tmx, bl, 0, x1, q * 8, y0, n);
            }
        };
#pragma unroll 1
        for (int u = blockIdx.x; u < sc.units && ok; u += gridDim.x) {
            const Unit un = decode_unit(p, sc, u);
            // First unit of one tile: thread et 0 reads the origin and starts the
            // halo copy at once (its stage has never been used, so it is free).
            const bool early = uit == 0 && p.halo_tma && sc.T == 1;
            if (early && et == 0) {
                int h0 = 0, w0 = 0;
                if (un.tb < G && (c.from_image || c.to_y))
                    tile_origin_a(c, un.tb / c.N, h0, w0);
                s_orig[0] = make_int2(h0, w0);
                issue_halo(bit % p.SB, un.kb / p.taps, un.tb);
            }
            // the previous unit's epilogue may still be reading the origins
            asm volatile("bar.sync 1, 256;" ::: "memory");
#pragma unroll 1
            for (int slot = et; slot < sc.T && !early; slot += kProd) {
                const int g = un.tb * sc.T + slot;
                int h0 = 0, w0 = 0;
                if (g < G && (c.from_image || c.to_y))
                    tile_origin_a(c, c.N == 1 ? g : (int)udiv((uint32_t)g, c.dN), h0, w0);
                s_orig[slot] = make_int2(h0, w0);
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
#pragma unroll 1
            for (int kc = un.kb; kc < un.ke; ++kc) {
                const int q = kc / p.taps, tap = kc - q * p.taps;
                if (kc == un.kb || tap == 0) {
                    const int sb = bit % p.SB;
                    const bool issued = early && kc == un.kb;
                    if (!issued && !group_wait(b_empty(sb), ((bit / p.SB) & 1) ^ 1, 5)) {
                        ok = false;
                        break;
                    }
                    uint8_t *stage = smem + cv.b_base + sb * cv.stage_b;
                    if (p.halo_tma) {
                        if (et == 0 && !issued)
                            issue_halo(sb, q, un.tb);
                        float gsc[8], gsh[8];
                        load_gn8(c, q, et, gsc, gsh);
                        if (!group_wait(b_load(sb), (bit / p.SB) & 1, 7)) {
                            ok = false;
                            break;
                        }
                        transform_b(c, sc.T, un.tb, q, G, stage, et, s_orig, gsc, gsh);
                    } else {
                        if (p.mode == 0)
                            fill_b(c, sc.T, un.tb, q, G, stage, et, s_orig);
                        else
                            fill_b_slots(c, sc.T, sc.dT, un.tb, q, G, stage, et, s_orig);
                    }
                    fence_async_smem();
                    mbar_arrive(b_full(sb));
                    ++bit;
                }
            }
            if (!ok)
                break;
            // bias of this thread's output channels (fixed across the unit)
            const int co0 = un.mt * 128 + cg * cpv;
            float bias8[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (c.bias && co0 < c.Cout) {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    if (k < cpv)
                        bias8[k] = __ldg(c.bias + co0 + k);
            }
            const int ncols = unit_cols(p, sc.T);
            const bool write_ok = co0 < c.Cout;
            // 2-way K split summed through the cluster peer's shared memory:
            // rank 1 sends its partial, rank 0 adds it and writes the output
            const int skind = split_kind(p, sc, cv);
            const bool pair = skind == kSplitPair;
            const uint32_t rank = pair ? cluster_rank() : 0u;
            const bool rs = skind == kSplitCluster;
            // rank 0 (or an unsplit unit of one batch of items): the residual of
            // this thread's items is read while the MMAs run
            const bool pre = (pair ? rank == 0 : sc.S == 1 && ncols <= stage_cols) && ncols * vpc <= 4 * kProd &&
                             c.residual && c.to_y;
            int64_t e_pre[4];
            uint4 rr_pre[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int it = et + k * kProd;
                e_pre[k] = (it < ncols * vpc && write_ok) ? col_target(c, s_orig, sc, un.tb, G, (it >> lvpc), co0) : -1;
                rr_pre[k] = make_uint4(0, 0, 0, 0);
                if (pre && e_pre[k] >= 0)
                    rr_pre[k] = __ldg(reinterpret_cast<const uint4 *>(c.residual + e_pre[k] * (c.dtype == SIGE_BF16 ? 2 : 4)));
            }
            if ((pair || rs) && !cwaited) {
                cluster_wait();
                cwaited = true;
            }
            if (pair && rank == 1 && pit > 0 && !group_wait_c(red_free, (pit - 1) & 1, 8)) {
                ok = false;
                break;
            }
            if (!group_wait(acc_full, uit & 1, 6)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t tbase = tmem + ((uint32_t)(sub * 32) << 16);
            if (pair && rank == 1) {
                // partial -> rank 0's receive buffer, [column][128 channels] floats
                const uint32_t rbuf = map_peer(sbase + cv.red_base, 0);
#pragma unroll 1
                for (int c0 = 16 * half; c0 < ncols; c0 += 32) {
                    float v[16];
                    tmem_ld16(tbase + c0, v);
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        st_peer_f32(rbuf + (uint32_t)(((c0 + k) * 128 + row) * 4), v[k]);
                }
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (et == 0)
                    mbar_arrive_peer(map_peer(red_full, 0));
                ++pit;
            } else if (pair) {
                float *red = reinterpret_cast<float *>(smem + cv.red_base);
                if (!group_wait_c(red_full, pit & 1, 9)) {
                    ok = false;
                    break;
                }
                // own partial added in place (two terms: the order does not change the sum)
#pragma unroll 1
                for (int c0 = 16 * half; c0 < ncols; c0 += 32) {
                    float v[16];
                    tmem_ld16(tbase + c0, v);
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        red[(c0 + k) * 128 + row] += v[k];
                }
                asm volatile("bar.sync 1, 256;" ::: "memory");
#pragma unroll 1
                for (int it0 = et; it0 < ncols * vpc; it0 += 4 * kProd) {
                    int64_t e[4];
                    uint4 rr[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int it = it0 + k * kProd;
                        if (it0 == et) {
                            e[k] = e_pre[k];
                            rr[k] = rr_pre[k];
                        } else {
                            e[k] = (it < ncols * vpc && write_ok) ? col_target(c, s_orig, sc, un.tb, G, (it >> lvpc), co0)
                                                                  : -1;
                            rr[k] = make_uint4(0, 0, 0, 0);
                        }
                        if (e[k] >= 0 && c.residual && c.to_y && !(pre && it0 == et))
                            rr[k] = __ldg(reinterpret_cast<const uint4 *>(c.residual + e[k] * (c.dtype == SIGE_BF16 ? 2 : 4)));
                    }
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        if (e[k] < 0)
                            continue;
                        const int col = (it0 + k * kProd) >> lvpc;
                        float v[8];
                        const float4 *src = reinterpret_cast<const float4 *>(red + col * 128 + cg * cpv);
                        const float4 lo = src[0];
                        v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
                        if (cpv == 8) {
                            const float4 hi = src[1];
                            v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
                        }
                        store_vec(c, e[k], v, bias8, rr[k]);
                    }
                }
                // the buffer is free for the peer's next partial
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (et == 0)
                    mbar_arrive_peer(map_peer(red_free, 1));
                ++pit;
            } else if (rs) {
                // Every member sends column slice q of its partial to member q,
                // into q's halo stages laid out [member][128 channels][w (+4)]
                // floats (16-byte remote stores of 4 columns); each member sums
                // its slice in member order and writes it.
                const uint32_t S = (uint32_t)sc.S;
                const uint32_t crank = cluster_rank();
                const uint32_t me = crank % S, g0 = crank - me;
                const uint32_t share = (uint32_t)p.csize / S;
                const int w = ncols / (int)S;
                // row stride: 4 floats of padding when they fit keep the
                // 16-byte accesses of a warp free of bank conflicts
                const int rsw = (uint32_t)(ncols + 4 * (int)S) * 512u <= (uint32_t)p.SB * cv.stage_b ? w + 4 : w;
                const uint32_t rb = sbase + cv.b_base;
                float *slab = reinterpret_cast<float *>(smem + cv.b_base);
                // this CTA's MMAs are complete: its halo stages may be written
                if (et == 0) {
#pragma unroll 1
                    for (uint32_t q = 0; q < S; ++q)
                        mbar_arrive_peer_n(map_peer(rs_ready, g0 + q), share);
                }
                if (!group_wait_c(rs_ready, rsit & 1, 11)) {
                    ok = false;
                    break;
                }
                const uint32_t my_row = rb + (uint32_t)(((int)me * 128 + row) * rsw * 4);
#pragma unroll 1
                for (int c0 = 16 * half; c0 < ncols; c0 += 32) {
                    float v[16];
                    tmem_ld16(tbase + c0, v);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4) {
                        const int col = c0 + 4 * k4;
                        const int q = col / w, off = col - q * w;   // w % 4 == 0: 4 columns, one owner
                        st_peer_f32x4(map_peer(my_row + (uint32_t)off * 4u, g0 + (uint32_t)q), v[4 * k4],
                                      v[4 * k4 + 1], v[4 * k4 + 2], v[4 * k4 + 3]);
                    }
                }
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (et == 0) {
#pragma unroll 1
                    for (uint32_t q = 0; q < S; ++q)
                        mbar_arrive_peer_n(map_peer(rs_full, g0 + q), share);
                }
                if (!group_wait_c(rs_full, rsit & 1, 12)) {
                    ok = false;
                    break;
                }
                // fixed member order: the sum does not depend on arrival order
#pragma unroll 1
                for (int j = 4 * half; j < w; j += 8) {
                    float4 *d = reinterpret_cast<float4 *>(slab + row * rsw + j);
                    float4 acc = *d;
#pragma unroll 1
                    for (uint32_t s2 = 1; s2 < S; ++s2) {
                        const float4 t = *reinterpret_cast<const float4 *>(slab + ((int)s2 * 128 + row) * rsw + j);
                        acc.x += t.x;
                        acc.y += t.y;
                        acc.z += t.z;
                        acc.w += t.w;
                    }
                    *d = acc;
                }
                asm volatile("bar.sync 1, 256;" ::: "memory");
#pragma unroll 1
                for (int it0 = et; it0 < w * vpc; it0 += 4 * kProd) {
                    int64_t e[4];
                    uint4 rr[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int it = it0 + k * kProd;
                        e[k] = (it < w * vpc && write_ok)
                                   ? col_target(c, s_orig, sc, un.tb, G, (int)me * w + (it >> lvpc), co0) : -1;
                        rr[k] = make_uint4(0, 0, 0, 0);
                        if (e[k] >= 0 && c.residual && c.to_y)
                            rr[k] = __ldg(reinterpret_cast<const uint4 *>(c.residual + e[k] * (c.dtype == SIGE_BF16 ? 2 : 4)));
                    }
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        if (e[k] < 0)
                            continue;
                        const int col = (it0 + k * kProd) >> lvpc;
                        float v[8];
#pragma unroll
                        for (int m = 0; m < 8; ++m)
                            v[m] = m < cpv ? slab[(cg * cpv + m) * rsw + col] : 0.0f;
                        store_vec(c, e[k], v, bias8, rr[k]);
                    }
                }
                ++rsit;
            } else if (sc.S == 1) {
                // accumulator -> shared staging (column-major, 128 floats per
                // column) -> 16-byte vectors per pixel
#pragma unroll 1
                for (int c0 = 0; c0 < ncols; c0 += stage_cols) {
                    const int cc_n = min(stage_cols, ncols - c0);
#pragma unroll 1
                    for (int k0 = 16 * half; k0 < cc_n; k0 += 32) {
                        float v[16];
                        tmem_ld16(tbase + c0 + k0, v);
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            stage_d[(k0 + k) * 128 + row] = v[k];
                    }
                    asm volatile("bar.sync 1, 256;" ::: "memory");
#pragma unroll 1
                    for (int it0 = et; it0 < cc_n * vpc; it0 += 4 * kProd) {
                        // four items per thread: addresses and residual loads first
                        int64_t e[4];
                        uint4 rr[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int it = it0 + k * kProd;
                            if (pre) {   // one chunk, one batch: read before the accumulator wait
                                e[k] = e_pre[k];
                                rr[k] = rr_pre[k];
                                continue;
                            }
                            e[k] = (it < cc_n * vpc && write_ok)
                                       ? col_target(c, s_orig, sc, un.tb, G, c0 + (it >> lvpc), co0) : -1;
                            rr[k] = make_uint4(0, 0, 0, 0);
                            if (e[k] >= 0 && c.residual && c.to_y)
                                rr[k] = __ldg(reinterpret_cast<const uint4 *>(c.residual + e[k] * (c.dtype == SIGE_BF16 ? 2 : 4)));
                        }
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            if (e[k] < 0)
                                continue;
                            const int col = (it0 + k * kProd) >> lvpc;
                            float v[8];
                            const float4 *src = reinterpret_cast<const float4 *>(stage_d + col * 128 + cg * cpv);
                            const float4 lo = src[0];
                            v[0] = lo.x; v[1] = lo.y; v[2] = lo.z; v[3] = lo.w;
                            if (cpv == 8) {
                                const float4 hi = src[1];
                                v[4] = hi.x; v[5] = hi.y; v[6] = hi.z; v[7] = hi.w;
                            }
                            store_vec(c, e[k], v, bias8, rr[k]);
                        }
                    }
                    asm volatile("bar.sync 1, 256;" ::: "memory");
                }
            } else {
                const int group = un.tb * p.MT + un.mt;
                float *slab = p.partials + (size_t)(group * sc.S + un.split) * p.ncols * 128;
#pragma unroll 1
                for (int c0 = 16 * half; c0 < ncols; c0 += 32) {
                    float v[16];
                    tmem_ld16(tbase + c0, v);
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        slab[(size_t)(c0 + k) * 128 + row] = v[k];
                }
                __threadfence();
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (et == 0) {
                    const unsigned prev = atomicAdd(p.counters + group, 1u);
                    const int last = prev == (unsigned)(sc.S - 1);
                    if (last)
                        p.counters[group] = 0;
                    *bcast = last;
                }
                asm volatile("bar.sync 1, 256;" ::: "memory");
                if (*bcast) {
                    __threadfence();
                    const float *base = p.partials + (size_t)group * sc.S * p.ncols * 128;
#pragma unroll 1
                    for (int it0 = et; it0 < ncols * vpc; it0 += 4 * kProd) {
                        int64_t e[4];
                        uint4 rr[4];
                        float v[4][8];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int it = it0 + k * kProd;
                            e[k] = (it < ncols * vpc && write_ok)
                                       ? col_target(c, s_orig, sc, un.tb, G, (it >> lvpc), co0) : -1;
                            rr[k] = make_uint4(0, 0, 0, 0);
                            if (e[k] >= 0 && c.residual && c.to_y)
                                rr[k] = __ldg(reinterpret_cast<const uint4 *>(c.residual + e[k] * (c.dtype == SIGE_BF16 ? 2 : 4)));
#pragma unroll
                            for (int m = 0; m < 8; ++m)
                                v[k][m] = 0.0f;
                        }
#pragma unroll 1
                        for (int s2 = 0; s2 < sc.S; ++s2) {   // fixed order: deterministic sum
#pragma unroll
                            for (int k = 0; k < 4; ++k) {
                                if (e[k] < 0)
                                    continue;
                                const int col = (it0 + k * kProd) >> lvpc;
                                const float4 *src = reinterpret_cast<const float4 *>(
                                    base + ((size_t)s2 * p.ncols + col) * 128 + cg * cpv);
                                const float4 lo = __ldcg(src);
                                v[k][0] += lo.x; v[k][1] += lo.y; v[k][2] += lo.z; v[k][3] += lo.w;
                                if (cpv == 8) {
                                    const float4 hi = __ldcg(src + 1);
                                    v[k][4] += hi.x; v[k][5] += hi.y; v[k][6] += hi.z; v[k][7] += hi.w;
                                }
                            }
                        }
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            if (e[k] >= 0)
                                store_vec(c, e[k], v[k], bias8, rr[k]);
                    }
                }
                asm volatile("bar.sync 1, 256;" ::: "memory");
            }
            tc_fence_before();
            mbar_arrive(acc_empty);
            ++uit;
        }
        // rank 1 stays until rank 0 has signalled its last use of the pair
        // (that arrival writes this CTA's shared memory)
        if (p.pair && pit > 0 && cluster_rank() == 1)
            group_wait_c(red_free, (pit - 1) & 1, 10);
    }

    if (p.pair && !cwaited)
        cluster_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.ncols));
    }
}

// ------------------------------------------------------------------ host

PFN_cuTensorMapEncodeTiled_v12000 get_encode()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

struct TcPlan {
    int mode, T_max, SB, ncols;
    uint32_t per_slot;
};

static int pow2_at_least(int v)
{
    int r = 32;
    while (r < v)
        r <<= 1;
    return r;
}

// Shared memory / tensor memory plan for a layer; false if it does not fit.
// The launch always takes the full 227 KB; T_max is the most tiles (slots) a
// unit may hold with at least two weight stages beside SB halo stages.
static bool plan_layer(const sige_conv_desc *cd, TcPlan &pl)
{
    const int b = cd->block, s = cd->stride, k = cd->kernel;
    const int bin = (b - 1) * s + k;
    pl.per_slot = (uint32_t)bin * bin * 128;  // one tile, 64 channels
    // ROW for 8x8 tiles at stride 1; mode 2 where an output row of 8 slots is a
    // legal MMA width (8 b a multiple of 16); POS otherwise
    pl.mode = (b == 8 && s == 1) ? 0 : (b % 2 == 0 && 8 * b <= 256) ? 2 : 1;
    const int budget = kSmemLimit - 1024 /*alignment*/ - (int)kCtrlBytes - 2 * (int)kAStageBytes - 1024;
    for (int SB : {2, 1}) {
        int tmax;
        if (pl.mode == 0) {
            tmax = std::min(8, budget / (int)(SB * pl.per_slot));      // 64 TMEM columns per tile
        } else if (pl.mode == 2) {
            tmax = (8 * SB * (int)pl.per_slot <= budget && b * b * 8 <= 512) ? 8 : 0;
        } else {
            const int by_tmem = (512 / (b * b)) / 16 * 16;
            const int by_smem = (budget / (int)(SB * pl.per_slot)) / 16 * 16;
            tmax = std::min({256, by_tmem, by_smem});
            if (tmax < 16)
                tmax = 0;
        }
        // the epilogue stages at least 16 accumulator columns (8 KB) in the
        // halo stages of the smallest unit (1 tile, or 16 slots)
        const uint32_t min_stage = SB * pl.per_slot * (pl.mode == 0 ? 1u : pl.mode == 2 ? 8u : 16u);
        if (tmax >= 1 && min_stage >= 16u * 512u) {
            pl.T_max = tmax;
            pl.SB = SB;
            const int cols = pl.mode == 0 ? tmax * 64 : b * b * tmax;
            pl.ncols = pow2_at_least(cols);
            return pl.ncols <= 512;
        }
    }
    return false;
}

bool tc_supported(const sige_conv_desc *cd, int dtype)
{
    if (!cd || dtype != SIGE_BF16 || cd->c_in % 64 || cd->c_in < 64 || cd->c_out < 8 || cd->c_out % 8)
        return false;
    if ((long long)cd->kernel * cd->kernel * cd->c_in >= (1ll << 31))
        return false;
    TcPlan pl;
    return plan_layer(cd, pl);
}

// Schedule fields of the argument block that depend only on the layer and
// its plan (the launch adds the buffers and the grid).
static void plan_args(const sige_conv_desc *cd, const TcPlan &pl, TcArgs &p)
{
    p.k = cd->kernel;
    p.s = cd->stride;
    p.b = cd->block;
    p.bin = (cd->block - 1) * cd->stride + cd->kernel;
    p.mode = pl.mode;
    p.taps = cd->kernel * cd->kernel;
    p.kci = cd->c_in / 64;
    p.MT = (cd->c_out + 127) / 128;
    p.T_max = pl.T_max;
    p.SB = pl.SB;
    p.per_slot = pl.per_slot;
    p.smem_bytes = kSmemLimit - 1024;   // usable after aligning the base to 1024
    p.ncols = pl.ncols;
}

// Cluster size for a launch: 4 where the K split may reach 4 (so that it can
// reduce-scatter within the cluster), else 2.  The split is decided on the
// device from the tile count; G_hint = 1 gives its largest value (sparse
// launches), the full tile count its exact value (dense launches).
static int preferred_cluster(const TcArgs &p, int G_hint, int sms)
{
    const Sched s = make_sched_for(p.mode, p.T_max, p.MT, p.taps * p.kci, sms, 1, std::max(1, G_hint));
    return s.S >= 4 ? 4 : 2;
}

int tc_schedule(const sige_conv_desc *cd, int tiles, int grid, int csize, int32_t *out, int n_out)
{
    TcPlan pl;
    if (!cd || !out || n_out < 1 || tiles < 0 || grid < 1 || csize < 1 || grid % csize != 0 || !plan_layer(cd, pl))
        return SIGE_ERR_INVALID_ARG;
    TcArgs p{};
    plan_args(cd, pl, p);
    p.num_sms = grid;
    p.csize = csize;
    p.pair = csize >= 2;
    const Sched sc = make_sched_for(p.mode, p.T_max, p.MT, p.taps * p.kci, grid, csize, tiles);
    const Carve cv = carve(p, sc.T);
    const int ncols = unit_cols(p, sc.T);
    const int32_t v[] = {p.mode, sc.T, sc.TB, sc.S, sc.units, split_kind(p, sc, cv), ncols, cv.SA,
                         (int32_t)(p.SB * cv.stage_b), ncols * 512, p.MT, p.taps * p.kci,
                         preferred_cluster(p, 1, grid), (int32_t)cv.b_base, (int32_t)p.smem_bytes};
    const int n = (int)(sizeof(v) / sizeof(v[0]));
    for (int i = 0; i < n_out; ++i)
        out[i] = i < n ? v[i] : 0;
    return SIGE_OK;
}

size_t tc_workspace_bytes(const sige_conv_desc *cd, int batch, int ntiles)
{
    (void)batch;
    (void)ntiles;
    TcPlan pl;
    if (!cd || !plan_layer(cd, pl))
        return 0;
    const int sms = device_sm_count();
    // counters (one per tile group that may split) + one partial slab per CTA
    return (size_t)((sms * 4 + 255) / 256) * 256 + (size_t)sms * pl.ncols * 128 * sizeof(float);
}

int launch_conv_tc(const ConvParams &cp, cudaStream_t stream)
{
    sige_conv_desc cd{cp.k, cp.s, cp.pad, cp.Cin, cp.Cout, cp.b};
    TcPlan pl;
    if (!plan_layer(&cd, pl))
        return SIGE_ERR_UNSUPPORTED;
    auto encode = get_encode();
    if (!encode)
        return SIGE_ERR_CUDA;
    CUtensorMap map;
    const cuuint64_t K = (cuuint64_t)cp.k * cp.k * cp.Cin;
    cuuint64_t dims[2] = {K, (cuuint64_t)cp.Cout};
    cuuint64_t strides[1] = {K * 2};
    cuuint32_t box[2] = {64, 128};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint8_t *>(cp.w), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS)
        return SIGE_ERR_CUDA;

    // ROW mode: one TMA per tile from a 5-d view of the source
    // [n][y][x][c/8][8] (image) or [g][hh][ww][c/8][8] (stacked blocks),
    // box (8 channels, b_in pixels, 8 channel groups, b_in rows), zero outside.
    CUtensorMap xmap = map;
    int halo_tma = 0;
    // the TMA halo copies the image as it is: the transposed conv's virtual
    // input and the per-pixel modulation go through the per-thread copies
    if (pl.mode == 0 && cp.tstride == 0 && cp.sg == nullptr && !cp.leaky) {
        const cuuint64_t C = (cuuint64_t)cp.Cin;
        cuuint64_t xd[5], xs[4];
        if (cp.from_image) {
            xd[0] = 8; xd[1] = (cuuint64_t)cp.W; xd[2] = C / 8; xd[3] = (cuuint64_t)cp.H; xd[4] = (cuuint64_t)cp.N;
            xs[0] = C * 2; xs[1] = 16; xs[2] = (cuuint64_t)cp.W * C * 2; xs[3] = (cuuint64_t)cp.H * cp.W * C * 2;
        } else {
            const cuuint64_t bin = (cuuint64_t)cp.bin;
            xd[0] = 8; xd[1] = bin; xd[2] = C / 8; xd[3] = bin; xd[4] = (cuuint64_t)std::max(1, cp.cap) * cp.N;
            xs[0] = C * 2; xs[1] = 16; xs[2] = bin * C * 2; xs[3] = bin * bin * C * 2;
        }
        cuuint32_t xbox[5] = {8, (cuuint32_t)cp.bin, 8, (cuuint32_t)cp.bin, 1};
        cuuint32_t xes[5] = {1, 1, 1, 1, 1};
        if (encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<uint8_t *>(cp.src), xd, xs, xbox, xes,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            halo_tma = 1;
        else
            xmap = map;
    }

    TcArgs p{};
    p.halo_tma = halo_tma;
    p.src = cp.src; p.idx = cp.idx; p.count = cp.count; p.gsc = cp.gsc; p.gsh = cp.gsh; p.bias = cp.bias;
    p.residual = cp.residual; p.y = cp.y; p.out_blocks = cp.out_blocks; p.ws = cp.ws;
    p.N = cp.N; p.H = cp.H; p.W = cp.W; p.Cin = cp.Cin; p.Cout = cp.Cout; p.dtype = cp.dtype;
    p.k = cp.k; p.s = cp.s; p.pad = cp.pad; p.b = cp.b; p.bin = cp.bin; p.Ho = cp.Ho; p.Wo = cp.Wo;
    p.dN = udiv_make((uint32_t)std::max(1, cp.N));
    p.dbin = udiv_make((uint32_t)std::max(1, cp.bin));
    p.db = udiv_make((uint32_t)std::max(1, cp.b));
    p.cap = cp.cap; p.dense = cp.dense; p.tiles_w = cp.tiles_w; p.tiles_total = cp.tiles_total;
    p.silu = cp.silu; p.from_image = cp.from_image; p.to_y = cp.to_y;
    p.sg = cp.sg; p.sb = cp.sb; p.leaky = cp.leaky; p.tstride = cp.tstride;
    plan_args(&cd, pl, p);
    p.num_sms = device_sm_count();
    uint8_t *ws = cp.ws + kWsHeader;
    p.counters = reinterpret_cast<uint32_t *>(ws);
    p.partials = reinterpret_cast<float *>(ws + ((p.num_sms * 4 + 255) / 256) * 256);

    const int want_c = preferred_cluster(p, cp.dense ? cp.tiles_total * cp.N : 1, p.num_sms);

    // per device: attribute set, co-resident clusters of 2 and of 4 CTAs (0 =
    // not yet known, -1 = none); concurrent first calls compute the same values
    static std::atomic<int> smem_set[64];
    static std::atomic<int> pair_clusters[64];
    static std::atomic<int> quad_clusters[64];
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64)
        dev = 0;
    if (!smem_set[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(k_conv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) != cudaSuccess)
            return SIGE_ERR_CUDA;
        smem_set[dev].store(1, std::memory_order_release);
    }
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = kSmemLimit;
    cfg.stream = stream;
    cfg.attrs = attr;
    auto clusters_of = [&](int csz, std::atomic<int> &slot) {
        if (!slot.load(std::memory_order_acquire)) {
            int n = 0;
            attr[1].val.clusterDim.x = csz;
            cfg.gridDim = dim3(csz * ((p.num_sms + csz - 1) / csz));
            cfg.numAttrs = 2;
            if (cudaOccupancyMaxActiveClusters(&n, k_conv_tc, &cfg) != cudaSuccess || n < 1) {
                cudaGetLastError();
                n = -1;
            }
            slot.store(n, std::memory_order_release);
        }
        return slot.load(std::memory_order_acquire);
    };
    // clusters of csize CTAs, as many as are co-resident; otherwise one CTA per SM
    cudaError_t e = cudaErrorUnknown;
    const int sms = p.num_sms;
    for (int csz : {want_c, 2}) {
        if (csz == 4 && want_c != 4)
            continue;
        const int clusters = clusters_of(csz, csz == 4 ? quad_clusters[dev] : pair_clusters[dev]);
        if (clusters <= 0)
            continue;
        p.pair = 1;
        p.csize = csz;
        p.num_sms = csz * std::min(clusters, sms / csz);
        attr[1].val.clusterDim.x = csz;
        cfg.gridDim = dim3(p.num_sms);
        cfg.numAttrs = 2;
        e = cudaLaunchKernelEx(&cfg, k_conv_tc, p, map, xmap);
        if (e == cudaSuccess)
            break;
        cudaGetLastError();
        (csz == 4 ? quad_clusters[dev] : pair_clusters[dev]).store(-1, std::memory_order_release);
        p.num_sms = sms;
    }
    if (e != cudaSuccess) {
        p.pair = 0;
        p.csize = 1;
        p.num_sms = device_sm_count();
        e = launch_pdl(k_conv_tc, dim3(p.num_sms), dim3(kTcThreads), kSmemLimit, stream, p, map, xmap);
    }
    count_launch();
    if (e != cudaSuccess)
        return SIGE_ERR_CUDA;
    return launch_check();
}

} // namespace sige
