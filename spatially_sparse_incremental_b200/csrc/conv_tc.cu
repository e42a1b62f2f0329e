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
// Two B layouts:
//   ROW (b = 8, stride 1): an N-group of 8 rows is one output row of a tile,
//     i.e. 8 consecutive halo pixels; one MMA per (tile, tap, 16 channels),
//     N = 64 (the tile's 8 x 8 pixels).
//   POS (any other b, stride, kernel): an N-group of 8 rows is 8 tiles at the
//     same halo position; one MMA per (output position (i, j), tap, 16
//     channels), N = the number of tiles of the unit (16..256).
// The producers apply the GroupNorm affine + SiLU (and the zero padding
// outside the image) while moving the halo into shared memory; the epilogue
// adds bias and residual and rounds once into the cached output, or writes
// float32 output blocks.  When the active tiles are too few to fill the GPU,
// the K loop is split over several CTAs; the last CTA to finish a tile group
// sums the partial accumulators in a fixed order (deterministic) and runs the
// epilogue.
//
// Warp roles (192 threads): warp 0 issues the weight TMA, warp 1 allocates
// tensor memory and one thread issues the MMAs, warps 2-5 stage the halo and
// run the epilogue.  Every mbarrier wait is bounded; on expiry the kernel
// records SIGE_ERR_TIMEOUT in the workspace header and unwinds.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "conv_tc.cuh"
#include "transform.cuh"

namespace sige {

constexpr int kTcThreads = 192;
constexpr uint32_t kAStageBytes = 128 * 64 * 2;
constexpr int kMaxSplit = 32;
constexpr long long kWaitCycles = 1ll << 31;   // ~1.1 s at 1.9 GHz
constexpr int kSmemLimit = 232448;             // 227 KB opt-in per CTA
constexpr int kSmemFloor = 120 * 1024;         // keeps one CTA (and one TMEM owner) per SM

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
    // schedule / shared-memory plan
    int32_t mode;             // 0 = ROW, 1 = POS
    int32_t taps, kci;        // k*k, C_in / 64
    int32_t MT;               // output-channel tiles of 128
    int32_t T_max;            // ROW: tiles per unit; POS: slots (multiple of 16)
    int32_t SA, SB;           // pipeline stages
    uint32_t b_off, bar_off, stage_b;
    int32_t ncols;            // tensor-memory columns allocated (power of 2)
    int32_t num_sms;
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

// ------------------------------------------------------------------ PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: false when the limit expired or another role gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag, WsHeader *hdr,
                                          int where)
{
    if (mbar_try(bar, parity))
        return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try(bar, parity))
            return true;
        if (*abort_flag)
            return false;
        if (clock64() - t0 > kWaitCycles) {
            *abort_flag = 1;
            record_error(hdr, SIGE_ERR_TIMEOUT, where);
            return false;
        }
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < 16; ++k)
        v[k] = __uint_as_float(r[k]);
}

// Shared-memory matrix descriptors (tcgen05 format, version 1).
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr)
{
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ uint64_t desc_plain(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | ((uint64_t)1 << 46);
}

// kind::f16, A = B = bf16, D = f32, both K-major, M = 128.
__device__ __forceinline__ uint32_t idesc_bf16(int n)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

// ------------------------------------------------------------------ schedule

struct Sched {
    int T;      // tiles per unit (POS: slots, multiple of 16)
    int TB;     // tile groups
    int S;      // K splits
    int units;
};

__device__ __forceinline__ Sched make_sched(const TcArgs &p, int G)
{
    Sched s;
    const int want = max(1, (G * p.MT + p.num_sms - 1) / p.num_sms);
    if (p.mode == 0)
        s.T = min(p.T_max, want);
    else
        s.T = min(p.T_max, ((want + 15) / 16) * 16);
    s.TB = (G + s.T - 1) / s.T;
    const int KC = p.taps * p.kci;
    s.S = max(1, min(p.num_sms / max(1, s.TB * p.MT), min(KC, kMaxSplit)));
    s.units = s.TB * p.MT * s.S;
    return s;
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
    const int KC = p.taps * p.kci;
    r.kb = (int)((long long)r.split * KC / s.S);
    r.ke = (int)((long long)(r.split + 1) * KC / s.S);
    return r;
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

// Fill one B stage: 64 input channels (chunk q) of the halo of every tile of
// the unit, transformed and zero-padded, in the core-matrix layout.
__device__ __forceinline__ void fill_b(const TcArgs &p, const Sched &s, int tb, int q, int G, uint8_t *stage, int et,
                                       const int2 *s_orig)
{
    const TcArgs &c = p;
    const int bin2 = c.bin * c.bin;
    const int slots = s.T;
    const int n_ent = slots * bin2 * 8;
    const bool affine = c.gsc != nullptr;
    const bool xform = affine || c.silu;
    // entries e = et + 128 k all share the 16-byte channel group kc = et & 7,
    // so a thread needs the affine parameters of 8 channels only
    const int kc = et & 7;
    const int ch = q * 64 + kc * 8;
    float gsc[8], gsh[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        gsc[k] = 1.0f;
        gsh[k] = 0.0f;
    }
    if (affine && c.N == 1) {
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            gsc[k] = __ldg(c.gsc + ch + k);
            gsh[k] = __ldg(c.gsh + ch + k);
        }
    }
    constexpr int U = 8;
    for (int e0 = et; e0 < n_ent; e0 += 128 * U) {
        uint4 v[U];
        uint32_t dst[U];
        int gsel[U];
        bool inb[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int e = e0 + u * 128;
            inb[u] = false;
            v[u] = make_uint4(0, 0, 0, 0);
            dst[u] = 0xFFFFFFFFu;
            gsel[u] = 0;
            if (e >= n_ent)
                continue;
            const int pix = (e >> 3) % bin2;
            const int slot = (e >> 3) / bin2;
            const int hh = pix / c.bin, ww = pix % c.bin;
            dst[u] = b_offset(p, slots, slot, hh, ww, kc);
            const int g = tb * s.T + slot;
            gsel[u] = g;
            if (g >= G)
                continue;
            const uint8_t *src;
            if (c.from_image) {
                const int2 o = s_orig[slot];
                const int y = o.x * c.s - c.pad + hh, x = o.y * c.s - c.pad + ww;
                if (y < 0 || y >= c.H || x < 0 || x >= c.W)
                    continue;
                const int n = g % c.N;
                src = c.src + ((((int64_t)n * c.H + y) * c.W + x) * c.Cin + ch) * 2;
            } else {
                src = c.src + (((int64_t)g * bin2 + pix) * c.Cin + ch) * 2;
            }
            v[u] = ld_nc16(src);
            inb[u] = true;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (dst[u] == 0xFFFFFFFFu)
                continue;
            uint4 w = v[u];
            if (inb[u] && xform) {
                if (affine && c.N > 1) {
                    const int n = gsel[u] % c.N;
                    w = transform16(w, SIGE_BF16, c.gsc + (int64_t)n * c.Cin + ch, c.gsh + (int64_t)n * c.Cin + ch,
                                    c.silu);
                } else {
                    w = transform16_bf16_reg(w, gsc, gsh, affine, c.silu);
                }
            }
            *reinterpret_cast<uint4 *>(stage + dst[u]) = w;
        }
    }
}

// ------------------------------------------------------------------ epilogue

// Write 16 consecutive accumulator columns (pixels) of one output channel.
// Addresses are computed first and every load (residual) is issued before the
// first store, so the 16 loads are in flight together.
__device__ __forceinline__ void emit16(const TcArgs &p, const Sched &s, const int2 *s_orig, int tb, int c0,
                                       int co, float bias_c, const float (&v)[16], int G)
{
    const TcArgs &c = p;
    int64_t e[16];
    bool ok[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const int col = c0 + k;
        int slot, i, j;
        if (p.mode == 0) {
            slot = col >> 6;
            i = (col >> 3) & 7;
            j = col & 7;
        } else {
            const int pos = col / s.T;
            slot = col - pos * s.T;
            i = pos / c.b;
            j = pos - i * c.b;
        }
        const int g = tb * s.T + slot;
        ok[k] = g < G && co < c.Cout;
        e[k] = 0;
        if (ok[k]) {
            if (c.to_y) {
                const int2 o = s_orig[slot];
                const int yo = o.x + i, xo = o.y + j;
                ok[k] = yo < c.Ho && xo < c.Wo;
                e[k] = (((int64_t)(g % c.N) * c.Ho + yo) * c.Wo + xo) * c.Cout + co;
            } else {
                e[k] = (((int64_t)g * c.b + i) * c.b + j) * c.Cout + co;
            }
        }
    }
    if (c.to_y) {
        float r[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            r[k] = 0.0f;
            if (ok[k] && c.residual) {
                if (c.dtype == SIGE_BF16)
                    r[k] = __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short *>(c.residual) + e[k]) << 16);
                else
                    r[k] = __ldg(reinterpret_cast<const float *>(c.residual) + e[k]);
            }
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            if (!ok[k])
                continue;
            const float y = (v[k] + bias_c) + r[k];
            if (c.dtype == SIGE_BF16)
                reinterpret_cast<__nv_bfloat16 *>(c.y)[e[k]] = __float2bfloat16_rn(y);
            else
                reinterpret_cast<float *>(c.y)[e[k]] = y;
        }
    } else {
#pragma unroll
        for (int k = 0; k < 16; ++k)
            if (ok[k])
                c.out_blocks[e[k]] = v[k];
    }
}

__device__ __forceinline__ int unit_cols(const TcArgs &p, const Sched &s)
{
    return p.mode == 0 ? s.T * 64 : p.b * p.b * s.T;
}

// ------------------------------------------------------------------ kernel

__global__ void __launch_bounds__(kTcThreads, 1)
    k_conv_tc(const __grid_constant__ TcArgs args, const __grid_constant__ CUtensorMap tmw)
{
    const TcArgs p = args;   // registers, see TcArgs
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw_addr + 1023) & ~1023u) - raw_addr);
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + p.bar_off);
    const uint32_t bar0 = smem_u32(bars);
    auto a_full = [&](int i) { return bar0 + 8u * i; };
    auto a_empty = [&](int i) { return bar0 + 8u * (p.SA + i); };
    auto b_full = [&](int i) { return bar0 + 8u * (2 * p.SA + i); };
    auto b_empty = [&](int i) { return bar0 + 8u * (2 * p.SA + p.SB + i); };
    const uint32_t acc_full = bar0 + 8u * (2 * p.SA + 2 * p.SB);
    const uint32_t acc_empty = acc_full + 8u;
    const uint32_t drain = acc_full + 16u;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * p.SA + 2 * p.SB + 3);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *bcast = abort_flag + 1;
    volatile int *group_ok = abort_flag + 2;
    int2 *s_orig = reinterpret_cast<int2 *>(smem + p.bar_off + 1024);   // tile origins of the current unit
    WsHeader *hdr = reinterpret_cast<WsHeader *>(p.ws);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < p.SA; ++i) {
            mbar_init(a_full(i), 1);
            mbar_init(a_empty(i), 1);
        }
        for (int i = 0; i < p.SB; ++i) {
            mbar_init(b_full(i), 128);
            mbar_init(b_empty(i), 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 128);
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0 && lane == 0)
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmw)) : "memory");
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(p.ncols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const TcArgs &c = p;
    const int ntile = c.dense ? c.tiles_total : min(__ldg(c.count), c.cap);
    const int G = ntile * c.N;
    const Sched sc = make_sched(p, G);

    if (warp == 0) {
        // ---------------- weight producer (TMA)
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < sc.units && ok; u += gridDim.x) {
                const Unit un = decode_unit(p, sc, u);
                for (int kc = un.kb; kc < un.ke; ++kc) {
                    const int s = it % p.SA;
                    if (!mbar_wait(a_empty(s), ((it / p.SA) & 1) ^ 1, abort_flag, hdr, 1)) {
                        ok = false;
                        break;
                    }
                    const int q = kc / p.taps, tap = kc - q * p.taps;
                    mbar_expect_tx(a_full(s), kAStageBytes);
                    tma_load_2d(sbase + s * kAStageBytes, &tmw, a_full(s), tap * c.Cin + q * 64, un.mt * 128);
                    ++it;
                }
            }
            // drain: every issued load must land before the CTA may exit
            for (uint32_t k = (it > (uint32_t)p.SA ? it - p.SA : 0); k < it; ++k) {
                const int s = k % p.SA;
                const long long t0 = clock64();
                while (!mbar_try(a_full(s), (k / p.SA) & 1) && clock64() - t0 < kWaitCycles) {
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer
        if (lane == 0) {
            uint32_t ait = 0, bit = 0, uit = 0;
            bool ok = true;
            const int bin = c.bin;
            for (int u = blockIdx.x; u < sc.units && ok; u += gridDim.x) {
                const Unit un = decode_unit(p, sc, u);
                if (uit > 0 && !mbar_wait(acc_empty, (uit - 1) & 1, abort_flag, hdr, 2)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int n_mma = p.mode == 0 ? 64 : sc.T;
                const uint32_t idesc = idesc_bf16(n_mma);
                const uint32_t sk = p.mode == 0 ? (uint32_t)bin * 16 : (uint32_t)sc.T * 16;   // LBO
                int sb = 0;
                for (int kc = un.kb; kc < un.ke; ++kc) {
                    const int q = kc / p.taps, tap = kc - q * p.taps;
                    if (kc == un.kb || tap == 0) {
                        sb = bit % p.SB;
                        if (!mbar_wait(b_full(sb), (bit / p.SB) & 1, abort_flag, hdr, 3)) {
                            ok = false;
                            break;
                        }
                    }
                    const int sa = ait % p.SA;
                    if (!mbar_wait(a_full(sa), (ait / p.SA) & 1, abort_flag, hdr, 4)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int r = tap / c.k, cc = tap - r * c.k;
                    const uint32_t a_base = sbase + sa * kAStageBytes;
                    const uint32_t b_base = sbase + p.b_off + sb * p.stage_b;
                    const bool first = (kc == un.kb);
#pragma unroll
                    for (int ks = 0; ks < 4; ++ks) {
                        const uint64_t ad = desc_sw128(a_base + ks * 32);
                        const uint32_t acc = (first && ks == 0) ? 0u : 1u;
                        if (p.mode == 0) {
                            const uint32_t sh = 8 * sk;  // halo row stride
                            for (int t = 0; t < sc.T; ++t) {
                                const uint32_t bs = b_base + t * bin * sh + r * sh + cc * 16 + 2 * ks * sk;
                                tc_mma(tmem + t * 64, ad, desc_plain(bs, sk, sh), idesc, acc);
                            }
                        } else {
                            const uint32_t sp = 8 * sk;  // halo pixel stride
                            for (int pos = 0; pos < c.b * c.b; ++pos) {
                                const int i = pos / c.b, j = pos - i * c.b;
                                const uint32_t bs =
                                    b_base + ((i * c.s + r) * bin + (j * c.s + cc)) * sp + 2 * ks * sk;
                                tc_mma(tmem + pos * sc.T, ad, desc_plain(bs, sk, 128), idesc, acc);
                            }
                        }
                    }
                    tc_commit(a_empty(sa));
                    ++ait;
                    if (kc == un.ke - 1 || tap == p.taps - 1) {
                        tc_commit(b_empty(sb));
                        ++bit;
                    }
                }
                if (!ok)
                    break;
                tc_commit(acc_full);
                ++uit;
            }
            // every MMA issued by this thread must finish before tensor memory is freed
            if (ait > 0) {
                tc_commit(drain);
                const long long t0 = clock64();
                while (!mbar_try(drain, 0) && clock64() - t0 < kWaitCycles) {
                }
            }
        }
    } else {
        // ---------------- halo producers + epilogue (warps 2..5)
        const int et = threadIdx.x - 64;
        const int sub = warp & 3;           // tensor-memory subpartition of this warp
        const int row = sub * 32 + lane;    // accumulator lane = output channel in the tile
        // One thread waits (bounded) and the group learns the outcome through a
        // named barrier, so that all 128 threads always take the same branch.
        auto group_wait = [&](uint32_t bar, uint32_t parity, int where) -> bool {
            if (et == 0)
                *group_ok = mbar_wait(bar, parity, abort_flag, hdr, where) ? 1 : 0;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            const bool r = *group_ok != 0;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            return r;
        };
        uint32_t bit = 0, uit = 0;
        bool ok = true;
        for (int u = blockIdx.x; u < sc.units && ok; u += gridDim.x) {
            const Unit un = decode_unit(p, sc, u);
            // the previous unit's epilogue may still be reading the origins
            asm volatile("bar.sync 1, 128;" ::: "memory");
            for (int slot = et; slot < sc.T; slot += 128) {
                const int g = un.tb * sc.T + slot;
                int h0 = 0, w0 = 0;
                if (g < G && (c.from_image || c.to_y))
                    tile_origin_a(c, g / c.N, h0, w0);
                s_orig[slot] = make_int2(h0, w0);
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            for (int kc = un.kb; kc < un.ke; ++kc) {
                const int q = kc / p.taps, tap = kc - q * p.taps;
                if (kc == un.kb || tap == 0) {
                    const int sb = bit % p.SB;
                    if (!group_wait(b_empty(sb), ((bit / p.SB) & 1) ^ 1, 5)) {
                        ok = false;
                        break;
                    }
                    fill_b(p, sc, un.tb, q, G, smem + p.b_off + sb * p.stage_b, et, s_orig);
                    fence_async_smem();
                    mbar_arrive(b_full(sb));
                    ++bit;
                }
            }
            if (!ok)
                break;
            if (!group_wait(acc_full, uit & 1, 6)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int co = un.mt * 128 + row;
            const float bias_c = (c.bias && co < c.Cout) ? __ldg(c.bias + co) : 0.0f;
            const int ncols = unit_cols(p, sc);
            const uint32_t tbase = tmem + ((uint32_t)(sub * 32) << 16);
            if (sc.S == 1) {
                for (int c0 = 0; c0 < ncols; c0 += 16) {
                    float v[16];
                    tmem_ld16(tbase + c0, v);
                    emit16(p, sc, s_orig, un.tb, c0, co, bias_c, v, G);
                }
            } else {
                const int group = un.tb * p.MT + un.mt;
                float *slab = p.partials + (size_t)(group * sc.S + un.split) * p.ncols * 128;
                for (int c0 = 0; c0 < ncols; c0 += 16) {
                    float v[16];
                    tmem_ld16(tbase + c0, v);
#pragma unroll
                    for (int k = 0; k < 16; ++k)
                        slab[(size_t)(c0 + k) * 128 + row] = v[k];
                }
                __threadfence();
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (et == 0) {
                    const unsigned prev = atomicAdd(p.counters + group, 1u);
                    const int last = prev == (unsigned)(sc.S - 1);
                    if (last)
                        p.counters[group] = 0;
                    *bcast = last;
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (*bcast) {
                    __threadfence();
                    const float *base = p.partials + (size_t)group * sc.S * p.ncols * 128;
                    for (int c0 = 0; c0 < ncols; c0 += 16) {
                        float acc[16];
#pragma unroll
                        for (int k = 0; k < 16; ++k)
                            acc[k] = 0.0f;
                        for (int s2 = 0; s2 < sc.S; ++s2) {   // fixed order: deterministic sum
                            float t[16];
#pragma unroll
                            for (int k = 0; k < 16; ++k)
                                t[k] = __ldcg(base + ((size_t)s2 * p.ncols + c0 + k) * 128 + row);
#pragma unroll
                            for (int k = 0; k < 16; ++k)
                                acc[k] += t[k];
                        }
                        emit16(p, sc, s_orig, un.tb, c0, co, bias_c, acc, G);
                    }
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
            }
            tc_fence_before();
            mbar_arrive(acc_empty);
            ++uit;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.ncols));
    }
}

// ------------------------------------------------------------------ host

static PFN_cuTensorMapEncodeTiled_v12000 get_encode()
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
    int mode, T_max, SA, SB, ncols;
    uint32_t stage_b, b_off, bar_off, smem;
};

static int pow2_at_least(int v)
{
    int r = 32;
    while (r < v)
        r <<= 1;
    return r;
}

// Shared memory / tensor memory plan for a layer; false if it does not fit.
static bool plan_layer(const sige_conv_desc *cd, TcPlan &pl)
{
    const int b = cd->block, s = cd->stride, k = cd->kernel;
    const int bin = (b - 1) * s + k;
    const uint32_t per_slot = (uint32_t)bin * bin * 128;  // one tile, 64 channels
    pl.mode = (b == 8 && s == 1) ? 0 : 1;
    const uint32_t bar_bytes = 1024 + 256 * 8;   // barriers and flags, then tile origins
    for (int SA : {4, 2}) {
        const uint32_t a_bytes = SA * kAStageBytes;
        const int budget = kSmemLimit - 1024 /*alignment slack*/ - (int)a_bytes - (int)bar_bytes;
        for (int SB : {2, 1}) {
            int tmax;
            if (pl.mode == 0) {
                tmax = std::min(8, budget / (int)(SB * per_slot));      // 64 TMEM columns per tile
            } else {
                const int by_tmem = (512 / (b * b)) / 16 * 16;
                const int by_smem = (budget / (int)(SB * per_slot)) / 16 * 16;
                tmax = std::min({256, by_tmem, by_smem});
                if (tmax < 16)
                    tmax = 0;
            }
            if (tmax >= 1) {
                pl.T_max = tmax;
                pl.SA = SA;
                pl.SB = SB;
                pl.stage_b = (uint32_t)tmax * per_slot;
                pl.b_off = a_bytes;
                pl.bar_off = (pl.b_off + SB * pl.stage_b + 15) & ~15u;
                pl.smem = std::max<uint32_t>(pl.bar_off + bar_bytes + 1024, kSmemFloor);
                const int cols = pl.mode == 0 ? tmax * 64 : b * b * tmax;
                pl.ncols = pow2_at_least(cols);
                return pl.ncols <= 512 && pl.smem <= (uint32_t)kSmemLimit;
            }
        }
    }
    return false;
}

bool tc_supported(const sige_conv_desc *cd, int dtype)
{
    if (!cd || dtype != SIGE_BF16 || cd->c_in % 64 || cd->c_in < 64 || cd->c_out < 1)
        return false;
    if ((long long)cd->kernel * cd->kernel * cd->c_in >= (1ll << 31))
        return false;
    TcPlan pl;
    return plan_layer(cd, pl);
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

    TcArgs p{};
    p.src = cp.src; p.idx = cp.idx; p.count = cp.count; p.gsc = cp.gsc; p.gsh = cp.gsh; p.bias = cp.bias;
    p.residual = cp.residual; p.y = cp.y; p.out_blocks = cp.out_blocks; p.ws = cp.ws;
    p.N = cp.N; p.H = cp.H; p.W = cp.W; p.Cin = cp.Cin; p.Cout = cp.Cout; p.dtype = cp.dtype;
    p.k = cp.k; p.s = cp.s; p.pad = cp.pad; p.b = cp.b; p.bin = cp.bin; p.Ho = cp.Ho; p.Wo = cp.Wo;
    p.cap = cp.cap; p.dense = cp.dense; p.tiles_w = cp.tiles_w; p.tiles_total = cp.tiles_total;
    p.silu = cp.silu; p.from_image = cp.from_image; p.to_y = cp.to_y;
    p.mode = pl.mode;
    p.taps = cp.k * cp.k;
    p.kci = cp.Cin / 64;
    p.MT = (cp.Cout + 127) / 128;
    p.T_max = pl.T_max;
    p.SA = pl.SA;
    p.SB = pl.SB;
    p.b_off = pl.b_off;
    p.bar_off = pl.bar_off;
    p.stage_b = pl.stage_b;
    p.ncols = pl.ncols;
    p.num_sms = device_sm_count();
    uint8_t *ws = cp.ws + kWsHeader;
    p.counters = reinterpret_cast<uint32_t *>(ws);
    p.partials = reinterpret_cast<float *>(ws + ((p.num_sms * 4 + 255) / 256) * 256);

    static int smem_set[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !smem_set[dev]) {
        if (cudaFuncSetAttribute(k_conv_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) != cudaSuccess)
            return SIGE_ERR_CUDA;
        smem_set[dev] = 1;
    }
    k_conv_tc<<<p.num_sms, kTcThreads, pl.smem, stream>>>(p, map);
    count_launch();
    return launch_check();
}

} // namespace sige
