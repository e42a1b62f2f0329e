// One 3x3 stride-1 conv layer F_l on 8x8 output tiles, on the tensor cores:
// gather (+GroupNorm affine +SiLU), the block conv and scatter (+bias
// +residual) in one launch (SIGE project page, "Overview": gather the active
// blocks with their halo, run F_l on them, scatter into the cached output).
// Used for every bf16 layer with a 3x3 kernel, stride 1, pad 1, 8x8 tiles,
// C_in a multiple of 64 and C_out a multiple of 32 up to 256 -- sparse (a
// tile list) and dense (every tile: the cache of the original and the dense
// baseline).
//
// The tensor core runs M=128 x N x K=16 at its full rate only for N >= 128;
// this kernel keeps N = C_out and makes the PIXELS the M dimension:
//   * a unit is two accumulators of 128 pixel rows sharing every weight
//     stage: in a dense launch a vertical strip of four tiles (32 x 8 output
//     pixels; accumulator a holds output rows 16a .. 16a + 15, every row
//     used), in a sparse launch two listed tiles (accumulator a holds tile a:
//     8 of its 16 row groups are output rows, the other 8 are discarded);
//   * A (pixels) in shared memory as [channel group][36 halo rows][10 cols]
//     [8 channels]: an M-group of 8 rows is one output row of a tile, the
//     next M-group the next halo row (160 bytes on), the tap (r, c) an offset
//     of 10 r + c pixels of the descriptor start; B (weights) by TMA, one
//     stage per (64-channel chunk, tap) of C_out rows x 64 K, 128-byte
//     swizzle; D in tensor memory, lane = pixel row, column = output channel;
//   * per 64-channel chunk the halo comes by one TMA of 128-byte pixel rows
//     (64 channels x 10 x 34 rows of a strip, or 64 x 10 x 10 per tile, zero
//     outside the image) into a staging buffer; warps 2-9 apply the GroupNorm
//     affine + SiLU (one tanh per element) and write the A layout,
//     into the other of two A buffers while the MMAs of the previous chunk run;
//   * warps 10-13 run the epilogue from the other tensor-memory buffer while
//     the next unit's MMAs run: + bias (+ residual), one rounding to bf16,
//     16-byte stores of each pixel's channels into the cached output;
//   * every CTA on the device wants the same weight stages at about the same
//     time; each CTA takes the nine taps of a chunk starting at tap
//     (CTA index mod 9), so that the requests spread over nine stages' lines
//     of the L2 instead of one.
// Warp roles (448 threads): 0 weight TMA, 1 tensor memory + MMA issue (one
// elected lane), 2-9 halo TMA + transform, 10-13 epilogue.  CTAs are
// persistent (one per SM) and take units with a stride of the grid.  Every
// wait is bounded; on expiry the kernel records SIGE_ERR_TIMEOUT (detail =
// wait site), the roles leave their loops, copies and MMAs in flight are
// drained (bounded) and tensor memory is freed.
#include <algorithm>
#include <atomic>

#include "conv_tc.cuh"
#include "tc_ptx.cuh"
#include "transform.cuh"

namespace sige {
namespace c8 {

constexpr int kThreads = 448;
constexpr int kHaloT = 256;                  // warps 2-9
constexpr int kEpiT = 128;                   // warps 10-13
constexpr int kRows = 36;                    // A-buffer halo rows (a strip's 34, or 2 x 18 per tile pair)
constexpr int kCols = 10;
constexpr int kPix = kRows * kCols;          // 360
constexpr uint32_t kKc = (kPix + 1) * 16;    // channel-group stride of an A buffer (16 mod 128: conflict-free writes)
constexpr uint32_t kABuf = 8 * kKc;          // one 64-channel chunk
constexpr uint32_t kStageS = kPix * 128;     // staging: pixel-major, 64 channels
constexpr int kMaxN = 256;
constexpr uint32_t kOffA = 1024;
constexpr uint32_t kOffS = kOffA + 2 * kABuf;
constexpr uint32_t kOffW = ((kOffS + kStageS + 1023) / 1024) * 1024;
constexpr uint32_t kSmemLimit = 232448;
constexpr uint32_t kEpiBias = kMaxN * 4;    // per epilogue warp: a copy of the bias
constexpr int kMaxStages = 8;
// control words
constexpr uint32_t kBarWFull = 0, kBarWEmpty = 64, kBarSFull = 128, kBarSEmpty = 136, kBarAFull = 144,
                   kBarAEmpty = 160, kBarAccFull = 176, kBarAccEmpty = 192, kBarDrain = 208;
constexpr uint32_t kTmemSlot = 256, kAbort = 260;

enum : int { kSiteWEmpty = 201, kSiteWFull, kSiteAFull, kSiteAEmpty, kSiteAccEmpty, kSiteAccFull, kSiteSFull,
             kSiteSEmpty };

}  // namespace c8

struct C8Args {
    const uint8_t *x;           // input, NHWC bf16 [N][H][W][Cin]
    const int32_t *idx;         // sparse: tile origins (h0, w0)
    const int32_t *count;
    const float *gsc, *gsh;     // GroupNorm affine [N][Cin] or null
    const float *bias;          // [Cout] or null
    const uint8_t *residual;    // [N][H][W][Cout] or null
    uint8_t *y;                 // output [N][H][W][Cout]
    WsHeader *hdr;
    int32_t N, H, W, Cin, Cout;
    int32_t cap, dense, th, tw;
    int32_t silu;
    int32_t stages;             // weight stages in the ring
    uint32_t stage_bytes;       // Cout x 128
    uint32_t tmem_cols;         // allocated columns
    int32_t dbuf;               // 1: two accumulator pairs (double-buffered units)
};

// SiLU of two values from their halves u = v / 2: v sigmoid(v) =
// u + u tanh(u), one tanh.approx.f32 (absolute error about 2^-11) and one
// FMA per element (the f16x2 tanh has the same element rate on the
// special-function pipe and adds conversions at half rate).
__device__ __forceinline__ uint32_t c8_silu2(float ua, float ub)
{
    float ta, tb;
    asm("tanh.approx.f32 %0, %1;" : "=f"(ta) : "f"(ua));
    asm("tanh.approx.f32 %0, %1;" : "=f"(tb) : "f"(ub));
    return pack_bf16x2(__fmaf_rn(ua, ta, ua), __fmaf_rn(ub, tb, ub));
}

// GroupNorm affine (sc, sh; identity when absent) and SiLU of 8 bf16
// channels.  With SiLU the affine arrives pre-halved (u = v / 2).
__device__ __forceinline__ uint4 c8_transform(uint4 in, const float (&sc)[8], const float (&sh)[8], int silu)
{
    uint4 out;
    uint32_t *o = reinterpret_cast<uint32_t *>(&out);
    const uint32_t *w = reinterpret_cast<const uint32_t *>(&in);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float a = __fmaf_rn(bf16_lo(w[q]), sc[2 * q], sh[2 * q]);
        const float b = __fmaf_rn(bf16_hi(w[q]), sc[2 * q + 1], sh[2 * q + 1]);
        o[q] = silu ? c8_silu2(a, b) : pack_bf16x2(a, b);
    }
    return out;
}

__device__ __forceinline__ void c8_tma_load_4d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1,
                                               int c2, int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// Eight K=16 MMAs of one weight stage: four for each accumulator (A of
// accumulator 1 starts a1_off descriptor units after accumulator 0's); the
// commit frees the stage.  acc1 == 0 skips accumulator 1.
__device__ __forceinline__ void c8_mma8(uint32_t d0, uint32_t d1, uint64_t a0, uint64_t a1_off, uint64_t a_step,
                                        uint64_t b, uint32_t idesc, uint32_t accumulate, uint32_t acc1, uint32_t bar)
{
    asm volatile(
        "{\n .reg .pred p, e, t, q;\n .reg .b32 l;\n .reg .b64 x1, x2, x3, y0, y1, y2, y3, b1, b2, b3;\n"
        " elect.sync l|e, 0xffffffff;\n setp.ne.b32 p, %5, 0;\n setp.eq.b32 t, 0, 0;\n setp.ne.b32 q, %6, 0;\n"
        " add.s64 x1, %2, %4;\n add.s64 x2, x1, %4;\n add.s64 x3, x2, %4;\n"
        " add.s64 y0, %2, %3;\n add.s64 y1, x1, %3;\n add.s64 y2, x2, %3;\n add.s64 y3, x3, %3;\n"
        " add.s64 b1, %7, 2;\n add.s64 b2, %7, 4;\n add.s64 b3, %7, 6;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %2, %7, %8, p;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], x1, b1, %8, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], x2, b2, %8, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], x3, b3, %8, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%1], y0, %7, %8, p;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%1], y1, b1, %8, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%1], y2, b2, %8, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%1], y3, b3, %8, t;\n"
        " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%9];\n}\n"
        ::"r"(d0), "r"(d1), "l"(a0), "l"(a1_off), "l"(a_step), "r"(accumulate), "r"(acc1), "l"(b), "r"(idesc),
        "r"(bar)
        : "memory");
    (void)acc1;
}

__device__ __forceinline__ void c8_mma4(uint32_t d0, uint64_t a0, uint64_t a_step, uint64_t b, uint32_t idesc,
                                        uint32_t accumulate, uint32_t bar)
{
    asm volatile(
        "{\n .reg .pred p, e, t;\n .reg .b32 l;\n .reg .b64 x1, x2, x3, b1, b2, b3;\n"
        " elect.sync l|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.eq.b32 t, 0, 0;\n"
        " add.s64 x1, %1, %3;\n add.s64 x2, x1, %3;\n add.s64 x3, x2, %3;\n"
        " add.s64 b1, %2, 2;\n add.s64 b2, %2, 4;\n add.s64 b3, %2, 6;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %5, p;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], x1, b1, %5, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], x2, b2, %5, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], x3, b3, %5, t;\n"
        " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n}\n"
        ::"r"(d0), "l"(a0), "l"(b), "l"(a_step), "r"(accumulate), "r"(idesc), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void c8_tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < 32; ++k)
        v[k] = __uint_as_float(r[k]);
}

// A unit's geometry: in a dense launch a strip of up to four tiles, in a
// sparse one up to two listed tiles (items; item g = tile g / N, batch g % N).
struct C8Unit {
    int n0, n1;          // batch item of accumulator 0 / 1
    int y0, x0;          // image origin of accumulator 0's output rows
    int y1, x1;          // image origin of accumulator 1's output rows
    int rows0, rows1;    // output rows of each accumulator (0: none)
};

__device__ __forceinline__ C8Unit c8_unit(const C8Args &p, int u)
{
    C8Unit r;
    if (p.dense) {
        const int n = u % p.N, strip = u / p.N;
        const int ts = strip / p.tw, tx = strip - ts * p.tw;
        r.n0 = r.n1 = n;
        r.y0 = ts * 32;
        r.x0 = r.x1 = tx * 8;
        r.y1 = r.y0 + 16;
        const int rows = min(32, p.H - r.y0);   // output rows in the image
        r.rows0 = min(16, rows);
        r.rows1 = max(0, rows - 16);
    } else {
        const int G = min(__ldg(p.count), p.cap) * p.N;
        const int g0 = 2 * u, g1 = 2 * u + 1;
        const int2 o0 = __ldg(reinterpret_cast<const int2 *>(p.idx) + g0 / p.N);
        r.n0 = g0 % p.N;
        r.y0 = o0.x;
        r.x0 = o0.y;
        r.rows0 = min(8, p.H - o0.x);
        if (g1 < G) {
            const int2 o1 = __ldg(reinterpret_cast<const int2 *>(p.idx) + g1 / p.N);
            r.n1 = g1 % p.N;
            r.y1 = o1.x;
            r.x1 = o1.y;
            r.rows1 = min(8, p.H - o1.x);
        } else {
            r.n1 = 0;
            r.y1 = r.x1 = 0;
            r.rows1 = 0;
        }
    }
    return r;
}

__global__ void __launch_bounds__(c8::kThreads, 1)
    k_conv8(const __grid_constant__ C8Args args, const __grid_constant__ CUtensorMap tmw,
            const __grid_constant__ CUtensorMap tm34, const __grid_constant__ CUtensorMap tm10)
{
    using namespace c8;
    const C8Args p = args;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
    const uint32_t sb = smem_u32(smem);
    auto w_full = [&](int i) { return sb + kBarWFull + 8u * i; };
    auto w_empty = [&](int i) { return sb + kBarWEmpty + 8u * i; };
    auto a_full = [&](int i) { return sb + kBarAFull + 8u * i; };
    auto a_empty = [&](int i) { return sb + kBarAEmpty + 8u * i; };
    auto acc_full = [&](int i) { return sb + kBarAccFull + 8u * i; };
    auto acc_empty = [&](int i) { return sb + kBarAccEmpty + 8u * i; };
    const uint32_t s_full = sb + kBarSFull, s_empty = sb + kBarSEmpty, drain = sb + kBarDrain;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kAbort);
    WsHeader *hdr = p.hdr;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = p.stages;
    const int NC = p.Cout;
    const int kch = p.Cin / 64;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(w_full(i), 1);
            mbar_init(w_empty(i), 1);
        }
        mbar_init(s_full, 1);
        mbar_init(s_empty, kHaloT);
        for (int i = 0; i < 2; ++i) {
            mbar_init(a_full(i), kHaloT);
            mbar_init(a_empty(i), 1);
            mbar_init(acc_full(i), 1);
            mbar_init(acc_empty(i), kEpiT);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmw)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(p.dense ? &tm34 : &tm10))
                     : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sb + kTmemSlot),
                     "r"(p.tmem_cols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + kTmemSlot);
    pdl_trigger();

    if (warp == 0) {
        // ------------------------------------------------ weight stages
        int s = 0, issued = 0;
        uint32_t ph = 1;
        bool ok = true;
        auto issue = [&](int q, int tap) -> bool {
            if (!mbar_wait_w(w_empty(s), ph, abort_flag, hdr, kSiteWEmpty))
                return false;
            tma_load_2d_w(sb + kOffW + (uint32_t)s * p.stage_bytes, &tmw, w_full(s), p.stage_bytes,
                          tap * p.Cin + q * 64, 0);
            ++issued;
            if (++s == S) {
                s = 0;
                ph ^= 1;
            }
            return true;
        };
        // the weights do not come from the previous kernel: the first stages
        // go out before the wait for it
        const int per_unit = kch * 9;
        const int pre = min(S, per_unit);
        const int rot = (int)(blockIdx.x % 9);          // first tap of every chunk
        for (int j = 0; j < pre && ok; ++j)
            ok = issue(j / 9, (j % 9 + rot) % 9);
        pdl_wait();
        const int units = p.dense ? ((p.th + 3) / 4) * p.tw * p.N : (min(__ldg(p.count), p.cap) * p.N + 1) / 2;
        bool first = true;
#pragma unroll 1
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
#pragma unroll 1
            for (int j = first ? pre : 0; j < per_unit && ok; ++j)
                ok = issue(j / 9, (j % 9 + rot) % 9);
            first = false;
        }
#pragma unroll 1
        for (int k = 1; k <= S && k <= issued; ++k) {
            const int g = issued - k;
            const int st = g % S;
            const uint32_t par = (uint32_t)(g / S) & 1u;
            const long long t0 = clock64();
            while (!mbar_try(w_full(st), par) && clock64() - t0 < kWaitCycles) {
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        pdl_wait();
        const int units = p.dense ? ((p.th + 3) / 4) * p.tw * p.N : (min(__ldg(p.count), p.cap) * p.N + 1) / 2;
        const uint32_t idesc = idesc_bf16(NC);
        const uint64_t b_desc0 = desc_sw128(sb + kOffW);
        const uint64_t w_step = p.stage_bytes >> 4;
        const uint64_t a_step = (2 * kKc) >> 4;
        // accumulator 1's A rows: 16 halo rows on in a strip, 18 for a tile pair
        const uint64_t a1_off = (uint64_t)(((p.dense ? 16 : 18) * kCols * 16) >> 4);
        const int rot = (int)(blockIdx.x % 9);          // the weight producer's tap order
        int s = 0;
        uint32_t ph = 0, ait = 0, qit = 0;
        bool ok = true;
        uint64_t b_cur = b_desc0;
        uint32_t k = 0;
#pragma unroll 1
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++k) {
            const int buf = p.dbuf ? (int)(k & 1) : 0;
            const uint32_t use = p.dbuf ? (k >> 1) : k;   // earlier uses of this accumulator pair
            if (use > 0 && !mbar_wait_w(acc_empty(buf), (use - 1) & 1, abort_flag, hdr, kSiteAccEmpty)) {
                ok = false;
                break;
            }
            tc_fence_after();
            // accumulator 1 is used unless a tile pair has a single tile
            uint32_t acc1 = 1;
            if (!p.dense) {
                const int G = min(__ldg(p.count), p.cap) * p.N;
                acc1 = (2 * u + 1 < G) ? 1u : 0u;
            } else {
                acc1 = (min(32, p.H - (u / p.N / p.tw) * 32) > 16) ? 1u : 0u;
            }
            const uint32_t d0 = tmem + (uint32_t)(buf * 2 * NC), d1 = d0 + (uint32_t)NC;
#pragma unroll 1
            for (int q = 0; q < kch && ok; ++q, ++qit) {
                const int ab = (int)(qit & 1);
                if (!mbar_wait_w(a_full(ab), (qit >> 1) & 1, abort_flag, hdr, kSiteAFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t abase = sb + kOffA + (uint32_t)ab * kABuf;
#pragma unroll 1
                for (int tap = 0; tap < 9; ++tap) {
                    const int tr = tap + rot < 9 ? tap + rot : tap + rot - 9;
                    const int r = tr / 3, c = tr - r * 3;
                    if (!mbar_wait_w(w_full(s), ph, abort_flag, hdr, kSiteWFull)) {
                        ok = false;
                        break;
                    }
                    const uint64_t a_desc = desc_plain(abase + (uint32_t)(r * kCols + c) * 16u, kKc, kCols * 16);
                    const uint32_t accum = (q | tap) ? 1u : 0u;
                    if (acc1)
                        c8_mma8(d0, d1, a_desc, a1_off, a_step, b_cur, idesc, accum, 1u, w_empty(s));
                    else
                        c8_mma4(d0, a_desc, a_step, b_cur, idesc, accum, w_empty(s));
                    ++ait;
                    if (++s == S) {
                        s = 0;
                        ph ^= 1;
                        b_cur = b_desc0;
                    } else {
                        b_cur += w_step;
                    }
                }
                if (!ok)
                    break;
                tc_commit_w(a_empty(ab));   // this A buffer may take a later chunk
            }
            if (!ok)
                break;
            tc_commit_w(acc_full(buf));
        }
        if (ait > 0) {
            tc_commit_w(drain);
            const long long t0 = clock64();
            while (!mbar_try(drain, 0) && clock64() - t0 < kWaitCycles) {
            }
        }
        __syncwarp();
    } else if (warp < 10) {
        // ------------------------------------------------ halo: TMA + transform
        const int ht = threadIdx.x - 64;                 // 0..255
        const int kcl = ht & 7, pq = ht >> 3;            // channel group; pixel phase 0..31
        constexpr int kPhases = kHaloT / 8;
        pdl_wait();
        const int units = p.dense ? ((p.th + 3) / 4) * p.tw * p.N : (min(__ldg(p.count), p.cap) * p.N + 1) / 2;
        const bool affine = p.gsc != nullptr;
        bool ok = true, pending = false;
        uint32_t qit = 0;
#pragma unroll 1
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            const C8Unit g = c8_unit(p, u);
#pragma unroll 1
            for (int q = 0; q < kch && ok; ++q, ++qit) {
                // the staging buffer is free (the previous chunk's transform
                // read it); one TMA per strip or per tile
                if (qit > 0 && !mbar_wait_w(s_empty, (qit - 1) & 1, abort_flag, hdr, kSiteSEmpty)) {
                    ok = false;
                    break;
                }
                if (ht == 0) {
                    if (p.dense) {
                        mbar_expect_tx(s_full, 34u * kCols * 128u);
                        c8_tma_load_4d(sb + kOffS, &tm34, s_full, q * 64, g.x0 - 1, g.y0 - 1, g.n0);
                    } else {
                        mbar_expect_tx(s_full, (g.rows1 > 0 ? 2u : 1u) * 10u * kCols * 128u);
                        c8_tma_load_4d(sb + kOffS, &tm10, s_full, q * 64, g.x0 - 1, g.y0 - 1, g.n0);
                        if (g.rows1 > 0)
                            c8_tma_load_4d(sb + kOffS + 18u * kCols * 128u, &tm10, s_full, q * 64, g.x1 - 1, g.y1 - 1,
                                           g.n1);
                    }
                    pending = true;
                }
                // GroupNorm parameters of this thread's 8 channels, per item
                // (halved for the SiLU's u = v / 2)
                float sc0[8], sh0[8], sc1[8], sh1[8];
                const int ch = q * 64 + kcl * 8;
                const float hs = p.silu ? 0.5f : 1.0f;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    sc0[e] = hs * (affine ? __ldg(p.gsc + (int64_t)g.n0 * p.Cin + ch + e) : 1.0f);
                    sh0[e] = hs * (affine ? __ldg(p.gsh + (int64_t)g.n0 * p.Cin + ch + e) : 0.0f);
                    sc1[e] = hs * (affine ? __ldg(p.gsc + (int64_t)g.n1 * p.Cin + ch + e) : 1.0f);
                    sh1[e] = hs * (affine ? __ldg(p.gsh + (int64_t)g.n1 * p.Cin + ch + e) : 0.0f);
                }
                // the A buffer is free (the MMAs of the chunk before last read it)
                const int ab = (int)(qit & 1);
                if (qit >= 2 && !mbar_wait_w(a_empty(ab), ((qit >> 1) - 1) & 1, abort_flag, hdr, kSiteAEmpty)) {
                    ok = false;
                    break;
                }
                if (!mbar_wait_w(s_full, qit & 1, abort_flag, hdr, kSiteSFull)) {
                    ok = false;
                    break;
                }
                if (ht == 0)
                    pending = false;
                const uint8_t *stg = smem + kOffS + kcl * 16;
                uint8_t *dst = smem + kOffA + ab * kABuf + kcl * kKc;
                // pixels of the unit's halo rows: a strip's rows 0..33, or each
                // tile's rows 0..9 at row offsets 0 and 18
                const int nrow = p.dense ? 34 : 10;
                const int npx = nrow * kCols;
#pragma unroll 1
                for (int part = 0; part < (p.dense ? 1 : 2); ++part) {
                    const bool second = part == 1;
                    if (second && g.rows1 == 0)
                        break;
                    const int row_off = second ? 18 : 0;
                    const int oy = (second ? g.y1 : g.y0) - 1, ox = (second ? g.x1 : g.x0) - 1;
#pragma unroll 1
                    for (int i = pq; i < npx; i += kPhases) {
                        const int hr = i / kCols, hc = i - hr * kCols;
                        const int Y = oy + hr, X = ox + hc;
                        const int px = (row_off + hr) * kCols + hc;
                        uint4 v = make_uint4(0, 0, 0, 0);   // outside the image: the conv's zero padding
                        if (Y >= 0 && Y < p.H && X >= 0 && X < p.W) {
                            v = *reinterpret_cast<const uint4 *>(stg + px * 128);
                            if (affine || p.silu)
                                v = second ? c8_transform(v, sc1, sh1, p.silu) : c8_transform(v, sc0, sh0, p.silu);
                        }
                        *reinterpret_cast<uint4 *>(dst + px * 16) = v;
                    }
                }
                mbar_arrive(s_empty);                      // staging read
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(a_full(ab));                   // A buffer written
            }
        }
        if (pending) {
            const long long t0 = clock64();
            while (!mbar_try(s_full, qit & 1) && clock64() - t0 < kWaitCycles) {
            }
        }
    } else {
        // ------------------------------------------------ epilogue
        const int sp = warp & 3;                         // tensor-memory subpartition
        const int row = sp * 32 + lane;                  // accumulator row
        const int oi = row >> 3, oj = row & 7;           // output row / column within the accumulator
        const uint32_t t_lane = tmem + ((uint32_t)(sp * 32) << 16);
        // this warp's copy of the bias: a global load per 32 columns would sit
        // behind the tensor-memory wait (a memory clobber) and cost a round
        // trip each time
        const float4 *bsm = reinterpret_cast<const float4 *>(smem + kOffW + (uint32_t)p.stages * p.stage_bytes +
                                                             (uint32_t)(warp - 10) * kEpiBias);
        pdl_wait();
        for (int c = lane * 4; c < NC; c += 128)
            const_cast<float4 *>(bsm)[c / 4] =
                p.bias ? __ldg(reinterpret_cast<const float4 *>(p.bias + c)) : make_float4(0.f, 0.f, 0.f, 0.f);
        __syncwarp();
        const int units = p.dense ? ((p.th + 3) / 4) * p.tw * p.N : (min(__ldg(p.count), p.cap) * p.N + 1) / 2;
        bool ok = true;
        uint32_t k = 0;
#pragma unroll 1
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++k) {
            const C8Unit g = c8_unit(p, u);
            const int buf = p.dbuf ? (int)(k & 1) : 0;
            const uint32_t use = p.dbuf ? (k >> 1) : k;
            if (!mbar_wait_w(acc_full(buf), use & 1, abort_flag, hdr, kSiteAccFull)) {
                ok = false;
                break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int a = 0; a < 2; ++a) {
                const int rows = a ? g.rows1 : g.rows0;
                const int n = a ? g.n1 : g.n0;
                const int Y = (a ? g.y1 : g.y0) + oi, X = (a ? g.x1 : g.x0) + oj;
                const bool valid = rows > 0 && oi < (p.dense ? 16 : 8) && oi < rows && Y >= 0 && X >= 0 && X < p.W;
                const int64_t e = ((((int64_t)n * p.H + Y) * p.W + X) * p.Cout);
                const uint32_t tcol = (uint32_t)((buf * 2 + a) * NC);
                // both accumulators of a strip exist; a tile pair may have one
                if (rows == 0)
                    continue;
#pragma unroll 1
                for (int c0 = 0; c0 < NC; c0 += 32) {
                    // the slice's residual is requested before the tensor-memory
                    // load, so that its round trip overlaps the load and wait
                    const uint4 *res = p.residual && valid
                                           ? reinterpret_cast<const uint4 *>(p.residual + (e + c0) * 2)
                                           : nullptr;
                    uint4 rq[4];
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8)
                        rq[g8] = res ? __ldg(res + g8) : make_uint4(0, 0, 0, 0);
                    float v[32];
                    c8_tmem_ld32(t_lane + tcol + (uint32_t)c0, v);
                    if (!valid)
                        continue;
                    uint4 *dst = reinterpret_cast<uint4 *>(p.y + (e + c0) * 2);
#pragma unroll
                    for (int g8 = 0; g8 < 4; ++g8) {
                        const float4 b0 = bsm[(c0 + 8 * g8) / 4], b1 = bsm[(c0 + 8 * g8) / 4 + 1];
                        const float bb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
                        const uint4 rr = rq[g8];
                        const uint32_t *rw = reinterpret_cast<const uint32_t *>(&rr);
                        uint32_t o[4];
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            const float r0 = res ? bf16_lo(rw[t]) : 0.0f, r1 = res ? bf16_hi(rw[t]) : 0.0f;
                            o[t] = pack_bf16x2((v[8 * g8 + 2 * t] + bb[2 * t]) + r0,
                                               (v[8 * g8 + 2 * t + 1] + bb[2 * t + 1]) + r1);
                        }
                        dst[g8] = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(acc_empty(buf));
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols));
    }
}

// ------------------------------------------------------------------ host

bool conv8_supported(const sige_conv_desc *cd, int dtype)
{
    return cd && dtype == SIGE_BF16 && cd->kernel == 3 && cd->stride == 1 && cd->pad == 1 && cd->block == 8 &&
           cd->c_in >= 64 && cd->c_in % 64 == 0 && cd->c_out >= 32 && cd->c_out <= c8::kMaxN && cd->c_out % 32 == 0;
}

static bool c8_encode_halo(CUtensorMap *map, const void *x, int N, int H, int W, int C, int rows,
                           PFN_cuTensorMapEncodeTiled_v12000 encode)
{
    cuuint64_t dims[4] = {(cuuint64_t)C, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)N};
    cuuint64_t strides[3] = {(cuuint64_t)C * 2, (cuuint64_t)W * C * 2, (cuuint64_t)H * W * C * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)c8::kCols, (cuuint32_t)rows, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(x), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int launch_conv8(const ConvParams &cp, cudaStream_t stream)
{
    using namespace c8;
    auto encode = get_encode();
    if (!encode)
        return SIGE_ERR_CUDA;
    CUtensorMap tmw, tm34, tm10;
    {
        const cuuint64_t K = (cuuint64_t)9 * cp.Cin;
        cuuint64_t dims[2] = {K, (cuuint64_t)cp.Cout};
        cuuint64_t strides[1] = {K * 2};
        cuuint32_t box[2] = {64, (cuuint32_t)cp.Cout};
        cuuint32_t es[2] = {1, 1};
        if (encode(&tmw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint8_t *>(cp.w), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return SIGE_ERR_UNSUPPORTED;
    }
    if (!c8_encode_halo(&tm34, cp.src, cp.N, cp.H, cp.W, cp.Cin, 34, encode) ||
        !c8_encode_halo(&tm10, cp.src, cp.N, cp.H, cp.W, cp.Cin, 10, encode))
        return SIGE_ERR_UNSUPPORTED;
    C8Args a{};
    a.x = cp.src;
    a.idx = cp.idx;
    a.count = cp.count;
    a.gsc = cp.gsc;
    a.gsh = cp.gsh;
    a.bias = cp.bias;
    a.residual = cp.residual;
    a.y = cp.y;
    a.hdr = reinterpret_cast<WsHeader *>(cp.ws);
    a.N = cp.N;
    a.H = cp.H;
    a.W = cp.W;
    a.Cin = cp.Cin;
    a.Cout = cp.Cout;
    a.cap = cp.cap;
    a.dense = cp.dense;
    a.th = (cp.Ho + 7) / 8;
    a.tw = (cp.Wo + 7) / 8;
    a.silu = cp.silu;
    a.stage_bytes = (uint32_t)cp.Cout * 128u;
    const uint32_t room = kSmemLimit - 1024 - kOffW - 4 * kEpiBias;
    a.stages = (int)std::min<uint32_t>(kMaxStages, room / a.stage_bytes);
    if (a.stages < 2)
        return SIGE_ERR_UNSUPPORTED;
    const uint32_t cols = 2u * (uint32_t)cp.Cout;
    a.dbuf = 2 * cols <= 512 ? 1 : 0;
    uint32_t tc = 32;
    while (tc < (a.dbuf ? 2 * cols : cols))
        tc <<= 1;
    a.tmem_cols = tc;
    const size_t smem = kOffW + (size_t)a.stages * a.stage_bytes + 4 * kEpiBias + 1024;
    static std::atomic<int> attr_set[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return SIGE_ERR_CUDA;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(k_conv8, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit) != cudaSuccess)
            return SIGE_ERR_CUDA;
        attr_set[dev].store(1, std::memory_order_release);
    }
    const int64_t units = cp.dense ? (int64_t)((a.th + 3) / 4) * a.tw * cp.N : ((int64_t)cp.cap * cp.N + 1) / 2;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(device_sm_count(), units));
    const cudaError_t e = launch_pdl(k_conv8, dim3(grid), dim3(kThreads), smem, stream, a, tmw, tm34, tm10);
    count_launch();
    if (e != cudaSuccess)
        return SIGE_ERR_CUDA;
    return launch_check();
}

} // namespace sige
