// The sparse residual block in one launch: GroupNorm1+SiLU -> 3x3 conv1 (+b1)
// -> GroupNorm2+SiLU -> 3x3 conv2 (+b2 + x) on the active 8x8 tiles, with the
// intermediate y1 kept on chip.  SIGE project page, "Overview": the layers F_l
// run on the gathered active blocks one after the other, each scattering into
// its cached output; mer.dev notes on SIGE, section 3 "Method": the cached
// activations of the original image are reused everywhere else.
//
// Halo recompute.  conv2 on an 8x8 tile reads y1 on the tile plus a one-pixel
// ring, and y1 there needs x on the tile plus a two-pixel ring.  Each tile's
// y1 is therefore computed on 10 x 10 pixels (1.56x the MACs of conv1 on the
// tile alone) from a 12 x 12 halo of x, and never goes through memory on its
// way to conv2.  Where the ring falls in another active tile this is the value
// that tile writes; where it falls in an inactive tile, no input of its 3x3
// window was edited (the list is dilated by at least one pixel beyond every
// edit), so it is the cached value.  The tile interior of y1 is still written
// to the cached y1, which stays valid for the next edit.
//
// Data path of one tile (one "unit"), on a cluster of two CTAs; CTA r owns
// output channels [64 r, 64 r + 64) of both convs:
//   * x halo: one TMA per 64 channels, box (64 channels, 12 x, 12 y) of the
//     NHWC tensor, landing pixel-major (128-byte rows, zero outside the
//     image); GroupNorm1 + SiLU then writes it as the conv's input,
//     [channel group][12 x 12 pixels][8 ch], zero outside the image (the
//     conv's padding);
//   * conv1 as an implicit GEMM D[pixel][c_out] = X[pixel][K] W1[c_out][K]^T,
//     K = (64-channel chunk, tap): A = the halo, read as 128 consecutive
//     "flat" pixels o = 12 yy + xx (pitch 12), the tap (r, c) being an offset
//     of 12 r + c pixels of the descriptor's start address (rows whose xx >= 10
//     are discarded); B = W1, 64 output channels x 64 K per TMA stage
//     (128-byte swizzle); D in tensor memory, one lane per flat pixel;
//   * epilogue 1: y1 = round_bf16(D + b1), stored to the cached y1 at the tile
//     interior; t = round_bf16(SiLU(GN2(y1))) (zero outside the image) into the
//     conv2 input buffer [channel group][10 x 10 pixels][8 ch] of BOTH CTAs
//     (distributed shared memory), so each holds all 128 channels;
//   * conv2 the same way on that buffer (pitch 10, rows with j >= 8 discarded);
//   * epilogue 2: out = round_bf16(D + b2 + x) at the tile's 64 pixels.
//
// Warp roles (320 threads): warp 0 streams the weight stages (TMA), warp 1
// owns tensor memory and issues the MMAs (one elected lane), warps 2-9 load
// and transform the x halo and run both epilogues (warp w reads tensor-memory
// lanes 32 (w mod 4) .. +31, and half (w - 2) / 4 of the 64 columns).  The
// CTA pair walks the units with a stride of the number of pairs; while the
// epilogue of tile k's conv2 runs, the halo of tile k+1 is already loaded and
// conv1 of tile k+1 is on the tensor cores.  Every wait is bounded: on
// expiry the kernel records SIGE_ERR_TIMEOUT (detail = wait site), the roles
// leave their loops, outstanding copies and MMAs are drained (bounded) and
// tensor memory is freed.
#include <algorithm>
#include <atomic>

#include "tc_ptx.cuh"
#include "transform.cuh"

namespace sige {
namespace rb {

constexpr int kThreads = 320;
constexpr int kEpi = 256;                  // halo / epilogue threads (warps 2-9)
constexpr int kC = 128;                    // channels of x, y1 and out
constexpr int kB = 8;                      // output tile edge
constexpr int kXE = 12;                    // x halo edge (tile + 2-pixel ring)
constexpr int kXPix = kXE * kXE;           // 144
// bytes of one 8-channel group of the conv1 input: 144 pixels and one of
// padding, so that the groups start 16 bytes apart modulo 128 and the
// transform's scattered 16-byte writes of 8 groups fall in 8 bank groups
constexpr uint32_t kXKc = (kXPix + 1) * 16;
constexpr uint32_t kXHalf = 8 * kXKc;      // 64 channels of the conv1 input
constexpr uint32_t kSHalf = kXPix * 128;   // 64 channels of the raw halo (the TMA box holds both, pixel-major)
constexpr int kYE = 10;                    // conv2 input edge (tile + 1-pixel ring)
constexpr uint32_t kYKc = kYE * kYE * 16;  // bytes of one 8-channel group of the conv2 input
constexpr uint32_t kWTap = 64 * 64 * 2;    // one tap: 64 output channels x 64 K, bf16
constexpr int kTapsPerStage = 3;           // one kernel row: a weight stage is ONE TMA of 24 KB
constexpr uint32_t kWStage = kTapsPerStage * kWTap;
constexpr int kStages = 5;                 // weight ring
constexpr int kChunks = 6;                 // weight stages per conv: 2 channel halves x 3 kernel rows
constexpr uint32_t kOffX = 1024;
constexpr uint32_t kOffS = kOffX + 16 * kXKc;                       // raw halo, two halves
constexpr uint32_t kOffY = kOffS + 2 * kSHalf;
constexpr uint32_t kOffW = ((kOffY + 16 * kYKc + 1023) / 1024 + 1) * 1024;   // (+1 KB: garbage-row reads of conv2)
// Per-unit parameter tables, two buffers (unit k uses buffer k & 1), filled
// by warp 0 from global memory ahead of the unit; floats: [0, 128) GroupNorm1
// scale / 2 and [128, 256) shift / 2 (all input channels of the unit's batch
// item), [256, 320) GroupNorm2 scale / 2 and [320, 384) shift / 2, [384, 448)
// b1, [448, 512) b2 (this CTA's 64 output channels).  The halving folds the
// SiLU's u = v / 2 into the affine.
constexpr uint32_t kOffP = kOffW + kStages * kWStage;
constexpr uint32_t kParBytes = 512 * 4;
constexpr uint32_t kSmem = kOffP + 2 * kParBytes + 1024;   // + alignment of the base
constexpr uint32_t kTmemCols = 128;        // conv1 accumulator [0, 64), conv2 [64, 128)
static_assert(kSmem <= 232448, "shared memory");
static_assert(kOffS % 128 == 0 && kSHalf % 128 == 0 && kOffY % 16 == 0, "TMA destinations");

// mbarriers and control words in [0, 1024)
constexpr uint32_t kBarWFull = 0, kBarWEmpty = 160, kBarXFull = 320, kBarXReady = 336;
constexpr uint32_t kBarParFull = 40, kBarParEmpty = 56;   // [2] each (after the 5 weight-stage barriers)
constexpr uint32_t kBarEpiSync = 72;                       // the 256 halo / epilogue threads meet (bounded)
constexpr uint32_t kBarAcc1Full = 352, kBarAcc1Empty = 360, kBarAcc2Full = 368, kBarAcc2Empty = 376;
constexpr uint32_t kBarY1tFull = 384, kBarY1tEmpty = 392, kBarDrain = 400, kBarY1tLocal = 408;
constexpr uint32_t kTmemSlot = 416, kAbort = 420, kUnits = 448;   // kUnits: the step's unit table (int2)
constexpr int kMaxUnits = 64;              // units one CTA pair takes in the step (tile origins at kUnits)
constexpr int kMaxTiles = 16384;           // tile grid of the step's mask (flags staged in the halo buffer)
// the step's difference stream: a ring of kRing slots, each a chunk of x_orig
// and the same chunk of x_edit (kRingVec 16-byte vectors each), filled by
// bulk copies in the halo / conv2-input region before the first halo
constexpr int kRing = 3;
constexpr int kRingVec = 1024;
constexpr uint32_t kRingBytes = kRingVec * 16;
constexpr uint32_t kOffRing = kOffX;
constexpr uint32_t kBarRingFull = 960, kBarRingEmpty = 992;
constexpr uint32_t kRingTag = 80;          // [kRing] int: the chunk each ring slot holds (-1: the stream is done)
static_assert(kOffRing + 2 * kRing * kRingBytes <= kOffW && kRingVec % 256 == 0, "ring");
static_assert(kUnits + 8 * kMaxUnits <= kBarRingFull, "control words");

// wait sites recorded in the error detail on a timeout
enum : int { kSiteWEmpty = 101, kSiteWFull, kSiteXReady, kSiteAcc1Empty, kSiteAcc2Empty, kSiteY1tFull,
             kSiteXFull, kSiteAcc1Full, kSiteY1tEmpty, kSiteAcc2Full, kSiteGrid, kSiteY1tLocal, kSiteRing,
             kSiteParFull, kSiteParEmpty, kSiteEpiSync };

}  // namespace rb

struct RbArgs {
    const uint8_t *x;           // x_edit, NHWC bf16 [N][H][W][128]
    const int32_t *idx;         // tile origins (h0, w0)
    const int32_t *count;
    const float *b1, *b2;       // [128] or null
    const float *g1s, *g1h;     // GroupNorm1 affine [N][128]
    const float *g2s, *g2h;     // GroupNorm2 affine [N][128]
    uint8_t *y1;                // cached y1, updated at the tile interiors
    uint8_t *out;               // cached out, updated at the tiles
    WsHeader *hdr;
    const uint8_t *w1, *w2;     // the weights (L2 prefetch; the stages come by TMA)
    int32_t N, H, W, cap;
    // the one-launch step: the tile list is made here from x_orig vs x (the
    // list and its count are then outputs: idx / count)
    const uint8_t *xo;          // x_orig, NHWC bf16 like x
    float thr;                  // difference threshold (strict >)
    int32_t dilate;             // tile dilation
    int32_t th, tw;             // tile grid
    uint32_t *flags;            // [th * tw] tile flags in the workspace: the epoch of the call that set them
    unsigned long long *ctr;    // grid-barrier arrivals in the workspace header (only grows)
    unsigned long long *chunk_ctr;   // difference-stream chunks handed out (workspace header, only grows)
    long long grid_wait;        // bound of the grid barrier's wait, in clocks (sige_set_wait_cycles, else ~1 s)
    UDiv div_hw, div_w;         // by H * W and by W, when every pixel index fits 32 bits (fast_px)
    int32_t fast_px;
};

// Four K=16 MMAs of one 64-channel weight stage: A (pixels, no swizzle)
// advances by a_step (descriptor units of 16 bytes) per step, B (weights,
// 128-byte swizzle) by 32 bytes; then the commit that frees the stage.  One
// elected lane issues.
__device__ __forceinline__ void rb_mma4(uint32_t d_tmem, uint64_t a_desc, uint64_t a_step, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate, uint32_t bar)
{
    asm volatile(
        "{\n .reg .pred p, e, t;\n .reg .b32 l;\n .reg .b64 a1, a2, a3, b1, b2, b3;\n"
        " elect.sync l|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.eq.b32 t, 0, 0;\n"
        " add.s64 a1, %1, %5;\n add.s64 a2, a1, %5;\n add.s64 a3, a2, %5;\n"
        " add.s64 b1, %2, 2;\n add.s64 b2, %2, 4;\n add.s64 b3, %2, 6;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %3, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %3, t;\n"
        " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "l"(a_step), "r"(bar)
        : "memory");
}

// Four K=16 MMAs (A advances by a_step, B by 32 bytes), no commit.
__device__ __forceinline__ void rb_mma4_nc(uint32_t d_tmem, uint64_t a_desc, uint64_t a_step, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p, e, t;\n .reg .b32 l;\n .reg .b64 a1, a2, a3, b1, b2, b3;\n"
        " elect.sync l|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.eq.b32 t, 0, 0;\n"
        " add.s64 a1, %1, %5;\n add.s64 a2, a1, %5;\n add.s64 a3, a2, %5;\n"
        " add.s64 b1, %2, 2;\n add.s64 b2, %2, 4;\n add.s64 b3, %2, 6;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %3, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %3, t;\n}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "l"(a_step)
        : "memory");
}

// expect_tx on `bar` and one 4-d tile load completing on it, from one lane.
__device__ __forceinline__ void rb_tma4_w(uint32_t dst, const CUtensorMap *map, uint32_t bar, uint32_t bytes, int c0,
                                          int c1, int c2, int c3)
{
    asm volatile(
        "{\n .reg .pred e;\n .reg .b32 l;\n elect.sync l|e, 0xffffffff;\n"
        " @e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%2], %3;\n"
        " @e cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%4, %5, %6, %7}], [%2];\n}\n"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(bytes), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

// Commit that arrives on the mbarrier at offset `bar` of both CTAs of the pair.
__device__ __forceinline__ void rb_commit_pair(uint32_t bar)
{
    asm volatile(
        "{\n .reg .pred e;\n .reg .b32 l;\n .reg .b16 m;\n elect.sync l|e, 0xffffffff;\n mov.b16 m, 3;\n"
        " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n}\n"
        ::"r"(bar)
        : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
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

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8])
{
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < 8; ++k)
        v[k] = __uint_as_float(r[k]);
}

// SiLU of two values from their halves u = v / 2 (the GroupNorm affine is
// pre-scaled by 1/2): v sigmoid(v) = v (1 + tanh(v / 2)) / 2 = u + u tanh(u),
// one special-function instruction (tanh.approx.f32, absolute error about
// 2^-11) and one FMA per element, one rounding to bf16 at the end.  The
// special-function pipe (16 results per clock and SM, the same for the f16x2
// form, which adds conversions at half rate) bounds the halo transform and
// epilogue 1.
__device__ __forceinline__ uint32_t rb_silu2(float ua, float ub)
{
    float ta, tb;
    asm("tanh.approx.f32 %0, %1;" : "=f"(ta) : "f"(ua));
    asm("tanh.approx.f32 %0, %1;" : "=f"(tb) : "f"(ub));
    return pack_bf16x2(__fmaf_rn(ua, ta, ua), __fmaf_rn(ub, tb, ub));
}

// GroupNorm affine (pre-halved, in registers) + SiLU of 8 bf16 channels.
__device__ __forceinline__ uint4 rb_gn_silu16(uint4 in, const float (&sc)[8], const float (&sh)[8])
{
    uint4 out;
    uint32_t *o = reinterpret_cast<uint32_t *>(&out);
    const uint32_t *w = reinterpret_cast<const uint32_t *>(&in);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        o[q] = rb_silu2(__fmaf_rn(bf16_lo(w[q]), sc[2 * q], sh[2 * q]),
                        __fmaf_rn(bf16_hi(w[q]), sc[2 * q + 1], sh[2 * q + 1]));
    return out;
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1, int c2,
                                            int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// A staged 8x8 tile (64 pixels x this CTA's 64 channels, 16-byte chunk c of
// pixel r at chunk c ^ (r & 7)) to the NHWC tensor `dst` at (n, h0.., w0..,
// 64 rank..): thread et of 256 moves chunks et and et + 256, eight threads per
// pixel, so a warp stores four pixels' 128 contiguous bytes at a time.
__device__ __forceinline__ void rb_copy_out(uint32_t stage, uint8_t *dst, int n, int h0, int w0, int H, int W,
                                            int rank, int et)
{
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
        const int idx = et + 256 * pass, r = idx >> 3, c = idx & 7;
        const int Y = h0 + (r >> 3), X = w0 + (r & 7);
        uint4 v;
        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                     : "r"(stage + (uint32_t)(r * 128) + ((uint32_t)(c ^ (r & 7)) << 4)));
        if (Y < H && X < W)
            *reinterpret_cast<uint4 *>(dst + ((((int64_t)n * H + Y) * W + X) * 128 + rank * 64 + c * 8) * 2) = v;
    }
}

__device__ __forceinline__ void st_peer_v4(uint32_t addr, uint4 v)
{
    asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
                 "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void cluster_arrive_rel() { asm volatile("barrier.cluster.arrive.release;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait_acq() { asm volatile("barrier.cluster.wait.acquire;" ::: "memory"); }


// ------------------------------------------------------------------ step mode

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t *ptr)
{
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

// Bits 0..7 of x to bits 0, 4, .., 28.
__device__ __forceinline__ uint32_t rb_spread4(uint32_t x)
{
    x &= 0xFFu;
    x = (x | (x << 12)) & 0x000F000Fu;
    x = (x | (x << 6)) & 0x03030303u;
    return (x | (x << 3)) & 0x11111111u;
}

// Bulk copy of `bytes` (a multiple of 16) from global memory into this CTA's
// shared memory, completing on the mbarrier `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// Some bf16 of 16 bytes differ by more than thr (the difference taken in float32).
__device__ __forceinline__ bool rb_exceeds(uint4 a, uint4 b, float thr)
{
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w};
    bool r = false;
#pragma unroll
    for (int q = 0; q < 4; ++q)
        r |= fabsf(bf16_lo(bw[q]) - bf16_lo(aw[q])) > thr || fabsf(bf16_hi(bw[q]) - bf16_hi(aw[q])) > thr;
    return r;
}

// Phases of the one-launch step before the res block (mer.dev notes on SIGE,
// sections 3 and 3.2: difference mask, dilation, tile selection; SIGE project
// page, "Overview": active block indices):
//   A. every CTA streams its contiguous share of x_orig and x_edit through a
//      ring of kRing shared-memory slots: one lane of warp 1 fills a slot with
//      two bulk copies (the same kRingVec 16-byte vectors of both inputs),
//      warps 2-9 compare it and release it, while warp 0 issues the first
//      weight stages; a pixel some channel of which differs by more than thr
//      marks its 8x8 tile: the tile's 32-bit flag is set to this call's epoch;
//   B. grid barrier (bounded): every CTA adds one arrival to a 64-bit counter
//      in the workspace header that only grows, and waits until it reaches
//      (generation + 1) * CTAs;
//   C. every CTA reads the flags once (16-byte loads) into a bitmap (one
//      ballot per flag position), takes as active the tiles whose flag equals
//      the epoch, dilates by `dilate` tiles (clipped) on 64-bit row words, and
//      compacts them in row-major order -- every CTA computes the same list;
//      CTA 0 writes it and its count out, each pair finds the origins of its
//      own units (u = pair + j * npairs, tile u / N) by a binary search of the
//      row prefix and a bit select.
// The generation is the counter's value at entry divided by the number of
// CTAs (every CTA of every call arrives exactly once, so the counter moves by
// exactly that much per call) and the epoch is the generation modulo
// 2^32 - 1, plus 1: flags of the last 2^32 - 2 calls never equal it and 0 (a
// flag never set) never does, so nothing is cleared between calls.
// Returns the number of units, min(count, cap) * N.
__device__ __forceinline__ int rb_step_list(const RbArgs &p, uint8_t *smem, volatile int *abort_flag, int pair,
                                            int npairs)
{
    using namespace rb;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int H = p.H, W = p.W, tw = p.tw, nt = p.th * p.tw;
    volatile int *s_ok = reinterpret_cast<volatile int *>(smem + kAbort + 12);
    // Every warp reads the counter itself, before this CTA's arrival: fewer
    // than gridDim.x arrivals of this call can precede the read, so all warps
    // of all CTAs find the same generation (and no warp waits for another to
    // start streaming).
    unsigned long long c0 = 0;
    if (lane == 0)
        asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(c0) : "l"(p.ctr) : "memory");
    c0 = __shfl_sync(0xFFFFFFFFu, c0, 0);
    const unsigned long long gen = c0 / gridDim.x;
    const unsigned long long target = (gen + 1) * gridDim.x;   // the counter value that ends the grid barrier
    const uint32_t epoch = (uint32_t)(gen % 0xFFFFFFFFull) + 1u; // never 0, the value of an unset flag
    // ---- A: difference mask -> tile flags
    bool wrote = false;
    {
        const int64_t nvec = (int64_t)p.N * H * W * (kC / 8);
        const int nchunks = (int)((nvec + kRingVec - 1) / kRingVec);
        // chunks are handed out by a counter in the workspace that only grows:
        // each call takes exactly nchunks + gridDim.x values from it (every
        // CTA stops at its first index past the end), so this call's first
        // value is gen * (nchunks + gridDim.x)
        const unsigned long long cbase = gen * (unsigned long long)(nchunks + (int)gridDim.x);
        const uint32_t sb = smem_u32(smem);
        auto ring_full = [&](int i) { return sb + kBarRingFull + 8u * i; };
        auto ring_empty = [&](int i) { return sb + kBarRingEmpty + 8u * i; };
        volatile int *s_tag = reinterpret_cast<volatile int *>(smem + kRingTag);   // chunk of each slot, -1: none
        if (wid == 1) {
            // one lane fills the ring: per slot, one chunk of both inputs
            if (lane == 0) {
                auto grab = [&]() -> int {
                    const long long j = (long long)(atomicAdd(p.chunk_ctr, 1ull) - cbase);
                    return j >= 0 && j < nchunks ? (int)j : -1;
                };
                int issued = 0, next = grab();
                bool stopped = false;
                for (int c = 0;; ++c) {
                    const int sl = c % kRing;
                    if (c >= kRing && !mbar_wait(ring_empty(sl), (uint32_t)((c / kRing) - 1) & 1u, abort_flag, p.hdr,
                                                 kSiteRing)) {
                        while (next >= 0)   // keep the count exact: claim the rest
                            next = grab();
                        break;
                    }
                    const int j = next;
                    s_tag[sl] = j;
                    if (j < 0) {
                        mbar_arrive(ring_full(sl));   // the comparing warps stop at this slot
                        stopped = true;
                        break;
                    }
                    const int64_t a = (int64_t)j * kRingVec;
                    const uint32_t bytes = (uint32_t)min((int64_t)kRingVec, nvec - a) * 16u;
                    const uint32_t dst = sb + kOffRing + (uint32_t)sl * 2u * kRingBytes;
                    mbar_expect_tx(ring_full(sl), 2u * bytes);
                    bulk_load(dst, p.xo + a * 16, bytes, ring_full(sl));
                    bulk_load(dst + kRingBytes, p.x + a * 16, bytes, ring_full(sl));
                    ++issued;
                    next = grab();   // the next index while these copies are in flight
                }
                // every copy lands before the region is reused (bounded); the
                // copy that shared its slot with the stop mark is complete (its
                // slot was released before the mark) and its phase parity has
                // been passed twice, so it is not waited for
                for (int c = max(0, issued - kRing + (stopped ? 1 : 0)); c < issued; ++c) {
                    const long long t0 = clock64();
                    while (!mbar_try(ring_full(c % kRing), (uint32_t)(c / kRing) & 1u) && clock64() - t0 < kWaitCycles) {
                    }
                }
            }
            __syncwarp();
        } else if (wid >= 2) {
            // warps 2-9 compare; a warp releases a slot once its lanes read it
            const int ct = tid - 64;
            int last = -1;
            for (int c = 0;; ++c) {
                const int sl = c % kRing;
                if (!mbar_wait_w(ring_full(sl), (uint32_t)(c / kRing) & 1u, abort_flag, p.hdr, kSiteRing))
                    break;
                const int j = s_tag[sl];
                if (j < 0)
                    break;
                const int64_t a = (int64_t)j * kRingVec;
                const int n = (int)min((int64_t)kRingVec, nvec - a);
                const uint4 *so = reinterpret_cast<const uint4 *>(smem + kOffRing + (uint32_t)sl * 2u * kRingBytes);
                const uint4 *se = so + kRingVec;
#pragma unroll
                for (int k = 0; k < kRingVec / kEpi; ++k) {
                    const int i = k * kEpi + ct;
                    if (i < n) {
                        const uint4 va = so[i], vb = se[i];
                        if (((va.x ^ vb.x) | (va.y ^ vb.y) | (va.z ^ vb.z) | (va.w ^ vb.w)) && rb_exceeds(va, vb, p.thr)) {
                            int y, x;
                            if (p.fast_px) {
                                const uint32_t pix = (uint32_t)((a + i) >> 4);   // 16 vectors per pixel
                                const uint32_t hw = pix - udiv(pix, p.div_hw) * ((uint32_t)H * (uint32_t)W);
                                const uint32_t yq = udiv(hw, p.div_w);
                                y = (int)yq;
                                x = (int)(hw - yq * (uint32_t)W);
                            } else {
                                const int64_t pix = (a + i) >> 4;
                                const int64_t hw = pix % ((int64_t)H * W);
                                y = (int)(hw / W);
                                x = (int)(hw - (int64_t)y * W);
                            }
                            const int t = (y >> 3) * tw + (x >> 3);
                            if (t != last) {
                                p.flags[t] = epoch;
                                last = t;
                                wrote = true;
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(ring_empty(sl));
            }
        }
    }
    // ---- B: grid barrier; the fence (cumulative, after the CTA barrier)
    // publishes every thread's flags before this CTA's arrival
    const bool any = __syncthreads_or(wrote);
    if (tid == 0) {
        if (any)
            __threadfence();
        atomicAdd(p.ctr, 1ull);
        const long long t0 = clock64();
        int ok = 1;
        while (true) {
            unsigned long long v;
            asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p.ctr) : "memory");
            if (v >= target)
                break;
            if (clock64() - t0 > p.grid_wait) {
                record_error(p.hdr, SIGE_ERR_TIMEOUT, kSiteGrid);
                ok = 0;
                break;
            }
            // a short pause between polls of the counter's line
            __nanosleep(32);
        }
        *s_ok = ok;
    }
    __syncthreads();
    const bool ok = *s_ok != 0;
    // ---- C: flags -> bits, dilate, compact
    uint8_t *s_flag = smem + kOffX;                 // ring / halo region, unused until the first halo
    uint8_t *s_act = s_flag + kMaxTiles;
    int *s_wsum = reinterpret_cast<int *>(smem + kOffY);
    int2 *s_units = reinterpret_cast<int2 *>(smem + kUnits);
    const int D = p.dilate;
    int total = 0, n_list = 0;
    if (p.th <= 64 && tw <= 64) {
        // rows of tiles as 64-bit words (grids of up to 64 x 64 tiles)
        uint64_t *s_row = reinterpret_cast<uint64_t *>(smem + kOffY);      // [64] dilated rows
        int *s_pre = reinterpret_cast<int *>(smem + kOffY + 512);          // [65] row prefix, [th] = total
        uint32_t *s_bits = reinterpret_cast<uint32_t *>(smem + kOffY + 1024);   // [128] flags, 32 tiles a word
        // One round of 16-byte loads: a warp reads 128 consecutive flags (4 a
        // lane) and four ballots (one per position in the vector) give the
        // four bitmap words of that range.
        const int nwords = (nt + 31) >> 5;
        for (int base = wid * 128; base < nt; base += kThreads * 4) {
            const int i = base + 4 * lane;
            const uint4 f = (ok && i < nt) ? __ldcg(reinterpret_cast<const uint4 *>(p.flags + i))
                                           : make_uint4(0, 0, 0, 0);
            const uint32_t b0 = __ballot_sync(0xFFFFFFFFu, f.x == epoch), b1 = __ballot_sync(0xFFFFFFFFu, f.y == epoch);
            const uint32_t b2 = __ballot_sync(0xFFFFFFFFu, f.z == epoch), b3 = __ballot_sync(0xFFFFFFFFu, f.w == epoch);
            if (lane < 4) {
                // flag base + 32 lane + 4 m + k is bit 8 lane + m of ballot k
                const int sh = 8 * lane;
                s_bits[(base >> 5) + lane] = rb_spread4(b0 >> sh) | (rb_spread4(b1 >> sh) << 1) |
                                             (rb_spread4(b2 >> sh) << 2) | (rb_spread4(b3 >> sh) << 3);
            }
        }
        __syncthreads();
        // Thread y < th: row y of the bitmap, dilated across the row; then the
        // OR of rows y - D .. y + D and its count; then the exclusive prefix of
        // the counts (independent loads).  Short dependency chains on many
        // threads: a chain of shuffles in one warp was measured at several us.
        uint64_t *s_h = reinterpret_cast<uint64_t *>(smem + kOffY + 1536);   // [64] rows dilated across
        int *s_cnt = reinterpret_cast<int *>(smem + kOffY + 2048);          // [64] active tiles per row
        const uint64_t full = tw == 64 ? ~0ull : ((1ull << tw) - 1);
        if (tid < p.th) {
            // bits [y tw, y tw + tw) of the bitmap
            const int st = tid * tw, w0 = st >> 5, sh = st & 31;
            const uint64_t lo = (uint64_t)s_bits[w0] | ((uint64_t)(w0 + 1 < nwords ? s_bits[w0 + 1] : 0u) << 32);
            const uint64_t hi = w0 + 2 < nwords ? s_bits[w0 + 2] : 0u;
            const uint64_t m = ((lo >> sh) | (sh ? hi << (64 - sh) : 0ull)) & full;
            uint64_t hd = m;
            for (int k = 1; k <= D && k < 64; ++k)
                hd |= (m << k) | (m >> k);
            s_h[tid] = hd & full;
        }
        __syncthreads();
        if (tid < p.th) {
            uint64_t d = 0;
            for (int yy = max(0, tid - D); yy <= min(p.th - 1, tid + D); ++yy)
                d |= s_h[yy];
            s_row[tid] = d;
            s_cnt[tid] = __popcll(d);
        }
        __syncthreads();
        if (tid <= p.th) {
            int pre = 0;
            for (int i = 0; i < tid; ++i)
                pre += s_cnt[i];
            s_pre[tid] = pre;                                             // s_pre[th]: the total
        }
        __syncthreads();
        total = s_pre[p.th];
        n_list = min(total, p.cap);
        // CTA 0 writes the list: thread y takes row y
        if (blockIdx.x == 0 && tid < p.th) {
            uint64_t m = s_row[tid];
            int pos = s_pre[tid];
            while (m && pos < n_list) {
                const int x = __ffsll((long long)m) - 1;
                m &= m - 1;
                reinterpret_cast<int2 *>(const_cast<int32_t *>(p.idx))[pos++] = make_int2(tid * kB, x * kB);
            }
        }
        // this pair's units u = pair + j * npairs: the (u / N)-th active tile
        if (tid < kMaxUnits) {
            const int u = pair + tid * npairs;
            if (u < n_list * p.N) {
                const int pos = u / p.N;
                // the last row whose prefix is <= pos, then the (pos - prefix)-th
                // set bit of that row
                int lo = 0, hi = p.th - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (s_pre[mid] <= pos)
                        lo = mid;
                    else
                        hi = mid - 1;
                }
                uint64_t m = s_row[lo];
                int r = pos - s_pre[lo], x = 0;
#pragma unroll
                for (int w = 32; w > 0; w >>= 1) {
                    const int c = __popcll(m & ((1ull << w) - 1));
                    if (r >= c) {
                        r -= c;
                        m >>= w;
                        x += w;
                    }
                }
                s_units[tid] = make_int2(lo * kB, x * kB);
            }
        }
    } else {
        // larger grids: flags to bytes, then one pass per thread over a
        // contiguous run of tiles
        for (int i = tid * 4; i < nt; i += kThreads * 4) {
            const uint4 f = ok ? __ldcg(reinterpret_cast<const uint4 *>(p.flags + i)) : make_uint4(0, 0, 0, 0);
            s_flag[i] = f.x == epoch;
            s_flag[i + 1] = f.y == epoch;
            s_flag[i + 2] = f.z == epoch;
            s_flag[i + 3] = f.w == epoch;
        }
        __syncthreads();
        const int seg = (nt + kThreads - 1) / kThreads;
        const int t0 = min(nt, tid * seg), t1 = min(nt, t0 + seg);
        int cnt = 0;
        for (int t = t0; t < t1; ++t) {
            const int ty = t / tw, tx = t - ty * tw;
            int act = 0;
            for (int dy = max(0, ty - D); dy <= min(p.th - 1, ty + D) && !act; ++dy)
                for (int dx = max(0, tx - D); dx <= min(tw - 1, tx + D) && !act; ++dx)
                    act = s_flag[dy * tw + dx];
            s_act[t] = (uint8_t)act;
            cnt += act;
        }
        // exclusive scan of the per-thread counts in thread order (= tile order)
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o)
                incl += v;
        }
        if (lane == 31)
            s_wsum[wid] = incl;
        __syncthreads();
        int before = 0;
        for (int w = 0; w < kThreads / 32; ++w) {
            const int v = s_wsum[w];
            before += w < wid ? v : 0;
            total += v;
        }
        int pos = before + incl - cnt;
        n_list = min(total, p.cap);
        for (int t = t0; t < t1; ++t) {
            if (!s_act[t])
                continue;
            const int2 org = make_int2((t / tw) * kB, (t - (t / tw) * tw) * kB);
            if (pos < n_list) {
                if (blockIdx.x == 0)
                    reinterpret_cast<int2 *>(const_cast<int32_t *>(p.idx))[pos] = org;
                for (int n = 0; n < p.N; ++n) {
                    const int u = pos * p.N + n;
                    if (u % npairs == pair && u / npairs < kMaxUnits)
                        s_units[u / npairs] = org;
                }
            }
            ++pos;
        }
    }
    if (blockIdx.x == 0 && tid == 0) {
        *const_cast<int32_t *>(p.count) = total;
        if (total > p.cap)
            record_error(p.hdr, SIGE_ERR_CAPACITY, 0);
    }
    __syncthreads();
    if (!ok)
        *abort_flag = 1;
    return ok ? n_list * p.N : 0;
}

template <bool kStep>
__global__ void __launch_bounds__(rb::kThreads, 1)
    k_resblock(const __grid_constant__ RbArgs args, const __grid_constant__ CUtensorMap tmx,
               const __grid_constant__ CUtensorMap tw1, const __grid_constant__ CUtensorMap tw2)
{
    using namespace rb;
    const RbArgs p = args;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023) & ~1023u) - raw);
    const uint32_t sb = smem_u32(smem);
    auto w_full = [&](int i) { return sb + kBarWFull + 8u * i; };
    auto w_empty = [&](int i) { return sb + kBarWEmpty + 8u * i; };
    auto x_full = [&](int h) { return sb + kBarXFull + 8u * h; };
    auto x_ready = [&](int h) { return sb + kBarXReady + 8u * h; };
    const uint32_t acc1_full = sb + kBarAcc1Full, acc1_empty = sb + kBarAcc1Empty;
    const uint32_t acc2_full = sb + kBarAcc2Full, acc2_empty = sb + kBarAcc2Empty;
    const uint32_t y1t_full = sb + kBarY1tFull, y1t_empty = sb + kBarY1tEmpty, drain = sb + kBarDrain;
    const uint32_t y1t_local = sb + kBarY1tLocal;
    auto par_full = [&](int b) { return sb + kBarParFull + 8u * b; };
    auto par_empty = [&](int b) { return sb + kBarParEmpty + 8u * b; };
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kAbort);
    WsHeader *hdr = p.hdr;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();          // output-channel half of this CTA
    const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(w_full(i), 1);
            mbar_init(w_empty(i), 1);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(x_full(h), 1);
            mbar_init(x_ready(h), kEpi);
        }
        mbar_init(acc1_full, 1);
        mbar_init(acc1_empty, kEpi);
        mbar_init(acc2_full, 1);
        mbar_init(acc2_empty, kEpi);
        mbar_init(y1t_full, 1);          // this CTA's half written + the peer's half copied in (tx bytes)
        mbar_init(y1t_empty, 2);         // the conv2 commits of both CTAs
        mbar_init(y1t_local, kEpi);      // every epilogue thread has written its part of this CTA's half
        mbar_init(drain, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(par_full(b), 1);
            mbar_init(par_empty(b), kEpi);
        }
        mbar_init(sb + kBarEpiSync, kEpi);
        if constexpr (kStep) {
            for (int i = 0; i < kRing; ++i) {
                mbar_init(sb + kBarRingFull + 8u * i, 1);
                mbar_init(sb + kBarRingEmpty + 8u * i, kEpi / 32);   // one arrival per comparing warp
            }
        }
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tw1)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tw2)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmx)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(sb + kTmemSlot),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + kTmemSlot);
    // Both CTAs' barriers are initialised before either side signals the
    // other: every thread waits on this cluster barrier before its first
    // access to the peer (and before the final one).
    cluster_arrive_rel();
    bool cwaited = false;
    pdl_trigger();

    // ---------------------------------------------------- weight stages (TMA)
    // The weights do not come from the previous kernel: the first stages of W1
    // go out before the wait for it (and, in the step, while the difference
    // mask streams).
    int s = 0, issued = 0;
    uint32_t ph = 1;
    bool ok = true;
    const int pre = kStages < kChunks ? kStages : kChunks;
    // stage j of a conv: channel half j / 3, kernel row j % 3 (its three
    // taps), this CTA's 64 output channels: one 24 KB box
    auto issue = [&](int conv, int j) -> bool {
            if (!mbar_wait_w(w_empty(s), ph, abort_flag, hdr, kSiteWEmpty))
                return false;
            const int half = j / 3, row = j - half * 3;
            rb_tma4_w(sb + kOffW + (uint32_t)s * kWStage, conv ? &tw2 : &tw1, w_full(s), kWStage, 0, (int)rank * 64,
                      row * 3, half);
            ++issued;
            if (++s == kStages) {
                s = 0;
                ph ^= 1;
            }
            return true;
    };
    if (warp == 0) {
        for (int j = 0; j < pre && ok; ++j)
            ok = issue(0, j);
    } else if (warp == 1 && lane == 0) {
        // Both weight tensors into the L2 (4 KB slices over the grid): every
        // CTA with a tile reads all of them, the first reads of a line after
        // a cold start would otherwise each wait for the DRAM.
        constexpr int kSlice = 4096, kSlices = (int)(9 * kC * kC * 2 / kSlice);   // per tensor
        for (int q = (int)blockIdx.x; q < 2 * kSlices; q += (int)gridDim.x) {
            const uint8_t *src = (q < kSlices ? p.w1 : p.w2) + (size_t)(q % kSlices) * kSlice;
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)),
                         "r"(kSlice) : "memory");
        }
    }
    pdl_wait();
    // Parameter table of this pair's unit k (batch item (pair + k npairs) mod
    // N) into buffer k & 1, by warp 0; the first one (two for a batch) while
    // the difference streams / the list is read.
    auto load_params = [&](int k) {
        const int n = (pair + k * npairs) % p.N;
        float *tab = reinterpret_cast<float *>(smem + kOffP + (uint32_t)(k & 1) * kParBytes);
        const int c_half = (int)rank * 64;
#pragma unroll
        for (int i = lane; i < 128; i += 32) {   // four independent loads per lane
            const int f = 4 * i;
            float4 v;
            if (f < 256) {
                const float *src = (f < 128 ? p.g1s : p.g1h) + n * kC + (f & 127);
                v = __ldg(reinterpret_cast<const float4 *>(src));
                v = make_float4(0.5f * v.x, 0.5f * v.y, 0.5f * v.z, 0.5f * v.w);
            } else if (f < 384) {
                const float *src = (f < 320 ? p.g2s : p.g2h) + n * kC + c_half + (f & 63);
                v = __ldg(reinterpret_cast<const float4 *>(src));
                v = make_float4(0.5f * v.x, 0.5f * v.y, 0.5f * v.z, 0.5f * v.w);
            } else {
                const float *b = f < 448 ? p.b1 : p.b2;
                v = b ? __ldg(reinterpret_cast<const float4 *>(b + c_half + (f & 63))) : make_float4(0.f, 0.f, 0.f, 0.f);
            }
            reinterpret_cast<float4 *>(tab)[i] = v;
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(par_full(k & 1));
    };
    if (warp == 0) {
        load_params(0);
        if (p.N > 1)
            load_params(1);
    }
    int units;
    int2 org0 = make_int2(0, 0);   // list mode: the pair's first tile origin, read beside the count
    if constexpr (kStep) {
        units = rb_step_list(p, smem, abort_flag, pair, npairs);
    } else {
        if (warp >= 2 && pair < p.cap * p.N)
            org0 = __ldg(reinterpret_cast<const int2 *>(p.idx) + pair / p.N);
        units = min(__ldg(p.count), p.cap) * p.N;
    }

    if (warp == 0) {
        bool first = true;
#pragma unroll 1
        for (int u = pair, k = 0; u < units && ok; u += npairs, ++k) {
            // the parameter buffer of unit k, once unit k - 2's epilogues are done with it
            if (p.N > 1 && k >= 2) {
                if (!mbar_wait_w(par_empty(k & 1), (uint32_t)((k >> 1) - 1) & 1u, abort_flag, hdr, kSiteParEmpty)) {
                    ok = false;
                    break;
                }
                load_params(k);
            }
#pragma unroll 1
            for (int conv = 0; conv < 2 && ok; ++conv)
#pragma unroll 1
                for (int j = (first && conv == 0) ? pre : 0; j < kChunks && ok; ++j)
                    ok = issue(conv, j);
            first = false;
        }
        // every load must land before the CTA may exit: wait for the last
        // use of each ring slot (a prefetch nothing consumed included)
#pragma unroll 1
        for (int k = 1; k <= kStages && k <= issued; ++k) {
            const int g = issued - k;
            const int st = g % kStages;
            const uint32_t par = (uint32_t)(g / kStages) & 1u;
            const long long t0 = clock64();
            while (!mbar_try(w_full(st), par) && clock64() - t0 < kWaitCycles) {
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        const uint32_t idesc = idesc_bf16(64);          // M = 128 pixels, N = 64 output channels
        const uint64_t b_desc0 = desc_sw128(sb + kOffW);
        const uint64_t w_step = kWStage >> 4;
        s = 0;
        ph = 0;
        uint32_t ait = 0;
        cluster_wait_acq();
        cwaited = true;
        uint64_t b_cur = b_desc0;
        // one conv: 2 chunks of 64 input channels x 9 taps, A = the pixel
        // buffer at `a_base` (pitch `pitch`, 8-channel groups `kc_bytes` apart)
        auto conv = [&](uint32_t a_base, int pitch, uint32_t kc_bytes, uint32_t d_col, bool wait_x, uint32_t xpar)
            -> bool {
            const uint64_t a_step = (2 * kc_bytes) >> 4;
#pragma unroll 1
            for (int kc2 = 0; kc2 < 2; ++kc2) {
                if (wait_x) {
                    if (!mbar_wait_w(x_ready(kc2), xpar, abort_flag, hdr, kSiteXReady))
                        return false;
                    tc_fence_after();
                }
                const uint32_t chunk = a_base + (uint32_t)kc2 * 8u * kc_bytes;
#pragma unroll 1
                for (int r = 0; r < 3; ++r) {
                    if (!mbar_wait_w(w_full(s), ph, abort_flag, hdr, kSiteWFull))
                        return false;
                    // the kernel row's three taps (r, c): A shifted by pitch r + c
                    // pixels, B the stage's c-th 8 KB tile
#pragma unroll
                    for (int c = 0; c < 3; ++c) {
                        const uint64_t a_desc = desc_plain(chunk + (uint32_t)(pitch * r + c) * 16u, kc_bytes, 128);
                        rb_mma4_nc(tmem + d_col, a_desc, a_step, b_cur + (uint64_t)(c * (kWTap >> 4)), idesc,
                                   (kc2 | r | c) ? 1u : 0u);
                    }
                    tc_commit_w(w_empty(s));
                    ++ait;
                    if (++s == kStages) {
                        s = 0;
                        ph ^= 1;
                        b_cur = b_desc0;
                    } else {
                        b_cur += w_step;
                    }
                }
            }
            return true;
        };
        uint32_t k = 0;
#pragma unroll 1
        for (int u = pair; u < units && ok; u += npairs, ++k) {
            // conv1, then conv2 through ONE copy of the issue code (code run
            // for the first time in a launch is fetched slowly)
#pragma unroll 1
            for (int cv = 0; cv < 2; ++cv) {
                if (cv == 0) {
                    // accumulator [0, 64) free once epilogue 1 of the previous tile has read it
                    if (k > 0 && !mbar_wait_w(acc1_empty, (k - 1) & 1, abort_flag, hdr, kSiteAcc1Empty)) {
                        ok = false;
                        break;
                    }
                } else {
                    // conv2: its input written by both CTAs' epilogue 1
                    if (k > 0 && !mbar_wait_w(acc2_empty, (k - 1) & 1, abort_flag, hdr, kSiteAcc2Empty)) {
                        ok = false;
                        break;
                    }
                    if (!__all_sync(0xFFFFFFFFu, mbar_wait_cluster(y1t_full, k & 1, abort_flag, hdr, kSiteY1tFull))) {
                        ok = false;
                        break;
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                tc_fence_after();
                if (!conv(cv ? sb + kOffY : sb + kOffX, cv ? kYE : kXE, cv ? kYKc : kXKc, cv ? 64u : 0u, cv == 0,
                          k & 1)) {
                    ok = false;
                    break;
                }
                tc_commit_w(cv ? acc2_full : acc1_full);
            }
            if (!ok)
                break;
            // the conv2 input buffers of both CTAs may be rewritten (none is
            // after the pair's last tile)
            if (u + npairs < units)
                rb_commit_pair(y1t_empty);
        }
        // every MMA issued here completes before tensor memory is freed
        if (ait > 0) {
            tc_commit_w(drain);
            const long long t0 = clock64();
            while (!mbar_try(drain, 0) && clock64() - t0 < kWaitCycles) {
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ x halo + epilogues
        const int et = threadIdx.x - 64;
        const int sp = warp & 3;                       // tensor-memory subpartition
        const int colh = (warp - 2) >> 2;              // columns [32 colh, 32 colh + 32)
        const int row = sp * 32 + lane;                // accumulator lane = flat pixel
        const uint32_t t_lane = tmem + ((uint32_t)(sp * 32) << 16);
        const int cb = (int)rank * 64 + colh * 32;     // first output channel of this thread
        const int H = p.H, W = p.W;
        bool x_pending = false;
        uint32_t xk = 0;                               // halos loaded so far (phase of x_full / x_ready)
        // The 256 threads meet on an mbarrier (bounded wait, unlike a named
        // barrier, so a thread that left on an error cannot hang the rest).
        uint32_t esync = 0;
        auto epi_sync = [&]() -> bool {
            mbar_arrive(sb + kBarEpiSync);
            const bool r = mbar_wait_w(sb + kBarEpiSync, esync & 1u, abort_flag, hdr, kSiteEpiSync);
            ++esync;
            return r;
        };

        auto origin = [&](int u, int &h0, int &w0, int &n) {
            int2 o;
            if constexpr (kStep)
                o = reinterpret_cast<const int2 *>(smem + kUnits)[(u - pair) / npairs];
            else
                o = u == pair ? org0 : __ldg(reinterpret_cast<const int2 *>(p.idx) + u / p.N);
            h0 = o.x;
            w0 = o.y;
            n = u % p.N;
        };
        // Load the x halo of unit u (thread 0 issues both TMAs) and apply
        // GroupNorm1 + SiLU in place at its in-image pixels.  The halo buffer
        // is free: conv1 of the previous tile has completed.
        auto load_x = [&](int u) -> bool {
            int h0, w0, n;
            origin(u, h0, w0, n);
            if (et == 0) {
                mbar_expect_tx(x_full(0), 2 * kSHalf);
                tma_load_4d(sb + kOffS, &tmx, x_full(0), 0, w0 - 2, h0 - 2, n);
                x_pending = true;
            }
            // thread: channel group kcl of each half, pixels 4 m + (lane >> 3)
            // of warp (et >> 5)'s share; a warp reads 4 raw pixels (512
            // contiguous bytes) and writes 8 groups x 4 pixels
            const int kcl = et & 7, pq = (et >> 3) & 3, ew = et >> 5;
            // both halves' GroupNorm1 parameters (halved) from this unit's table
            const int pb = p.N > 1 ? (int)(xk & 1) : 0;
            if (!mbar_wait_w(par_full(pb), p.N > 1 ? (xk >> 1) & 1u : 0u, abort_flag, hdr, kSiteParFull))
                return false;
            const float *tab = reinterpret_cast<const float *>(smem + kOffP + (uint32_t)pb * kParBytes);
            float gsa[2][8], gha[2][8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int ch = (h * 8 + kcl) * 8;
                const float4 s0 = *reinterpret_cast<const float4 *>(tab + ch);
                const float4 s1 = *reinterpret_cast<const float4 *>(tab + ch + 4);
                const float4 h0v = *reinterpret_cast<const float4 *>(tab + 128 + ch);
                const float4 h1v = *reinterpret_cast<const float4 *>(tab + 128 + ch + 4);
                gsa[h][0] = s0.x; gsa[h][1] = s0.y; gsa[h][2] = s0.z; gsa[h][3] = s0.w;
                gsa[h][4] = s1.x; gsa[h][5] = s1.y; gsa[h][6] = s1.z; gsa[h][7] = s1.w;
                gha[h][0] = h0v.x; gha[h][1] = h0v.y; gha[h][2] = h0v.z; gha[h][3] = h0v.w;
                gha[h][4] = h1v.x; gha[h][5] = h1v.y; gha[h][6] = h1v.z; gha[h][7] = h1v.w;
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float (&gs)[8] = gsa[h];
                const float (&gh)[8] = gha[h];
                if (h == 0 && !mbar_wait_w(x_full(0), xk & 1, abort_flag, hdr, kSiteXFull))
                    return false;
                if (et == 0)
                    x_pending = false;
                const uint8_t *raw = smem + kOffS + h * 128 + kcl * 16;
                uint8_t *dst = smem + kOffX + (h * 8 + kcl) * kXKc;
#pragma unroll 2
                for (int px = 4 * ew + pq; px < kXPix; px += 32) {
                    const int yy = px / kXE, xx = px - yy * kXE;
                    const int Y = h0 - 2 + yy, X = w0 - 2 + xx;
                    uint4 v = make_uint4(0, 0, 0, 0);   // outside the image: the conv's zero padding
                    if (Y >= 0 && Y < H && X >= 0 && X < W)
                        v = rb_gn_silu16(*reinterpret_cast<const uint4 *>(raw + px * 256), gs, gh);
                    *reinterpret_cast<uint4 *>(dst + px * 16) = v;
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(x_ready(h));
            }
            ++xk;
            return true;
        };

        if (pair < units)
            ok = load_x(pair);
        uint32_t k = 0;
#pragma unroll 1
        for (int u = pair; u < units && ok; u += npairs, ++k) {
            int h0, w0, n;
            origin(u, h0, w0, n);
            // this unit's parameter table (waited for by load_x)
            const int pb = p.N > 1 ? (int)(k & 1) : 0;
            const float *tab = reinterpret_cast<const float *>(smem + kOffP + (uint32_t)pb * kParBytes);
            // ------------ epilogue 1: y1 on the 10 x 10 pixels (flat o = 12 yy + xx)
            {
                const int yy = row / kXE, xx = row - yy * kXE;
                const bool valid = yy < kYE && xx < kYE;
                const int Y = h0 - 1 + yy, X = w0 - 1 + xx;
                const bool inimg = valid && Y >= 0 && Y < H && X >= 0 && X < W;
                const bool interior = inimg && yy >= 1 && yy <= kB && xx >= 1 && xx <= kB;
                // this thread's 32 channels of b1 and GroupNorm2 (halved) from the
                // unit's table, before the wait
                const int cl0 = colh * 32;
                float bias[32], gs[32], gh[32];
#pragma unroll
                for (int q = 0; q < 32; q += 4) {
                    const float4 s4 = *reinterpret_cast<const float4 *>(tab + 256 + cl0 + q);
                    const float4 h4 = *reinterpret_cast<const float4 *>(tab + 320 + cl0 + q);
                    const float4 b4 = *reinterpret_cast<const float4 *>(tab + 384 + cl0 + q);
                    gs[q] = s4.x; gs[q + 1] = s4.y; gs[q + 2] = s4.z; gs[q + 3] = s4.w;
                    gh[q] = h4.x; gh[q + 1] = h4.y; gh[q + 2] = h4.z; gh[q + 3] = h4.w;
                    bias[q] = b4.x; bias[q + 1] = b4.y; bias[q + 2] = b4.z; bias[q + 3] = b4.w;
                }
                if (!mbar_wait_w(acc1_full, k & 1, abort_flag, hdr, kSiteAcc1Full)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // both CTAs' conv2 of the previous tile have read the buffers
                if (!cwaited) {
                    cluster_wait_acq();
                    cwaited = true;
                }
                if (k > 0 && !__all_sync(0xFFFFFFFFu, mbar_wait_cluster(y1t_empty, (k - 1) & 1, abort_flag, hdr,
                                                                        kSiteY1tEmpty))) {
                    ok = false;
                    break;
                }
                const uint32_t pix = (uint32_t)(yy * kYE + xx) * 16u;
                // the tile interior of y1 goes through a staging tile in the
                // conv1 input buffer (free once conv1 is complete): 64 pixels x
                // 128 bytes, 16-byte chunk c of pixel r at chunk c ^ (r & 7)
                const uint32_t y1s = sb + kOffX + (uint32_t)(((yy - 1) * kB + (xx - 1)) * 128);
                const uint32_t y1s_sw = (uint32_t)((yy - 1) * kB + (xx - 1)) & 7u;
                float v[32];
                tmem_ld32(t_lane + (uint32_t)cl0, v);
                // all 32 columns in straight-line code: four independent groups
                // keep the special-function pipe busy
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    uint32_t y1p[4], tp[4];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const int c = 8 * g + 2 * q;
                        y1p[q] = pack_bf16x2(v[c] + bias[c], v[c + 1] + bias[c + 1]);
                        // GroupNorm2 (halved: u = v / 2 for the SiLU)
                        const float ua = __fmaf_rn(bf16_lo(y1p[q]), gs[c], gh[c]);
                        const float ub = __fmaf_rn(bf16_hi(y1p[q]), gs[c + 1], gh[c + 1]);
                        tp[q] = inimg ? rb_silu2(ua, ub) : 0u;
                    }
                    if (valid)
                        st_shared_v4(sb + kOffY + (uint32_t)(cb / 8 + g) * kYKc + pix,
                                     make_uint4(tp[0], tp[1], tp[2], tp[3]));
                    if (interior)
                        st_shared_v4(y1s + ((((uint32_t)(colh * 4 + g)) ^ y1s_sw) << 4),
                                     make_uint4(y1p[0], y1p[1], y1p[2], y1p[3]));
                }
                // the accumulator may take the next tile's conv1
                tc_fence_before();
                mbar_arrive(acc1_empty);
                // written through the generic proxy, read next by the tensor
                // cores and the bulk copy (async proxy)
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(y1t_local);
                if (et == 0) {
                    // once the whole half is written: one bulk copy of it (this
                    // CTA's 8 channel groups, 12800 bytes) into the peer's
                    // buffer, completing on the peer's y1t_full; here, the
                    // local half is ready and the peer's copy is expected
                    if (!mbar_wait(y1t_local, k & 1, abort_flag, hdr, kSiteY1tLocal)) {
                        ok = false;
                    } else {
                        const uint32_t src = sb + kOffY + rank * 8u * kYKc;
                        asm volatile(
                            "cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                            ::"r"(map_peer(src, rank ^ 1u)), "r"(src), "r"(8u * kYKc),
                            "r"(map_peer(y1t_full, rank ^ 1u))
                            : "memory");
                        mbar_expect_tx(y1t_full, 8u * kYKc);
                    }
                }
                // the staged y1 interior to the cached y1, coalesced: a warp
                // writes four pixels' 128 contiguous bytes per instruction
                ok = __all_sync(0xFFFFFFFFu, ok);   // thread 0's wait, warp-uniform
                if (!ok || !epi_sync()) {
                    ok = false;
                    break;
                }
                rb_copy_out(sb + kOffX, p.y1, n, h0, w0, H, W, (int)rank, et);
            }
            // ------------ the next tile's halo, while conv2 of this one runs
            // every thread has copied the staged y1 out of the conv1 input buffer
            if (u + npairs < units && !epi_sync()) {
                ok = false;
                break;
            }
            if (u + npairs < units && !load_x(u + npairs)) {
                ok = false;
                break;
            }
            // ------------ epilogue 2: out on the tile's 8 x 8 pixels (flat o = 10 i + j)
            {
                const int i = row / kYE, j = row - i * kYE;
                const int Y = h0 + i, X = w0 + j;
                const bool inimg = i < kB && j < kB && Y < H && X < W;
                const int64_t e = (((int64_t)n * H + Y) * W + X) * kC + cb;
                uint4 res[4];
                float bias[32];
#pragma unroll
                for (int g = 0; g < 4; ++g)
                    res[g] = inimg ? __ldg(reinterpret_cast<const uint4 *>(p.x + e * 2) + g) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int q = 0; q < 32; q += 4) {
                    const float4 b = *reinterpret_cast<const float4 *>(tab + 448 + (cb - (int)rank * 64) + q);
                    bias[q] = b.x; bias[q + 1] = b.y; bias[q + 2] = b.z; bias[q + 3] = b.w;
                }
                if (!mbar_wait_w(acc2_full, k & 1, abort_flag, hdr, kSiteAcc2Full)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                float v[32];
                tmem_ld32(t_lane + 64u + (uint32_t)(colh * 32), v);
                tc_fence_before();
                mbar_arrive(acc2_empty);
                // out through a staging tile in this CTA's half of the conv2
                // input buffer (conv2 is complete; the peer writes only the
                // other half), then coalesced stores
                const uint32_t os = sb + kOffY + rank * 8u * kYKc;
                if (inimg) {
                    const uint32_t r = (uint32_t)(i * kB + j);
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const uint32_t *rr = reinterpret_cast<const uint32_t *>(&res[g]);
                        uint32_t o4[4];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const int c0 = 8 * g + 2 * q;
                            o4[q] = pack_bf16x2((v[c0] + bias[c0]) + bf16_lo(rr[q]),
                                                (v[c0 + 1] + bias[c0 + 1]) + bf16_hi(rr[q]));
                        }
                        st_shared_v4(os + r * 128u + ((((uint32_t)(colh * 4 + g)) ^ (r & 7u)) << 4),
                                     make_uint4(o4[0], o4[1], o4[2], o4[3]));
                    }
                }
                if (!epi_sync()) {
                    ok = false;
                    break;
                }
                rb_copy_out(os, p.out, n, h0, w0, H, W, (int)rank, et);
                // the staging half may take the next tile's conv2 input
                if (u + npairs < units && !epi_sync()) {
                    ok = false;
                    break;
                }
                // this unit's parameter table may take unit k + 2's
                if (p.N > 1)
                    mbar_arrive(par_empty(pb));
            }
        }
        // a halo copy still in flight (a wait gave up) lands before the exit
        if (x_pending) {
            const long long t0 = clock64();
            while (!mbar_try(x_full(0), xk & 1) && clock64() - t0 < kWaitCycles) {
            }
        }
    }

    if (!cwaited)
        cluster_wait_acq();
    tc_fence_before();
    __syncthreads();
    // no CTA leaves while its peer may still write to it
    cluster_arrive_rel();
    cluster_wait_acq();
    tc_fence_after();
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
}

// ------------------------------------------------------------------ host

// Weights [c_out][3][3][c_in] as a 4-d map (64 input channels, c_out, tap,
// channel half) with strides 2304 / 256 / 128 bytes: a box of 64 output
// channels x 3 taps of one half lands as three 8 KB K-major tiles with the
// 128-byte swizzle, one TMA per weight stage.
static bool encode_weights(CUtensorMap *map, const void *w, PFN_cuTensorMapEncodeTiled_v12000 encode)
{
    cuuint64_t dims[4] = {64, (cuuint64_t)rb::kC, 9, 2};
    cuuint64_t strides[3] = {(cuuint64_t)9 * rb::kC * 2, (cuuint64_t)rb::kC * 2, 128};
    cuuint32_t box[4] = {64, 64, (cuuint32_t)rb::kTapsPerStage, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(w), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The NHWC tensor as a 4-d map [n][y][x][c]; a box of all 128 channels x 12 x
// 12 pixels lands pixel-major (256-byte rows) in shared memory, zero outside
// the image.
static bool encode_halo(CUtensorMap *map, const void *x, int N, int H, int W,
                        PFN_cuTensorMapEncodeTiled_v12000 encode)
{
    const cuuint64_t C = rb::kC;
    cuuint64_t dims[4] = {C, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)N};
    cuuint64_t strides[3] = {C * 2, (cuuint64_t)W * C * 2, (cuuint64_t)H * W * C * 2};
    cuuint32_t box[4] = {(cuuint32_t)C, (cuuint32_t)rb::kXE, (cuuint32_t)rb::kXE, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(x), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool aligned(const void *ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0; }

static bool overlaps(const void *a, const void *b, size_t n)
{
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + n && y < x + n;
}

// Shared-memory opt-in and co-resident pairs of a kernel instance, per device.
template <bool kStep>
static int rb_pairs(int dev, cudaLaunchConfig_t &cfg)
{
    static std::atomic<int> pairs_of[64];
    int pairs = pairs_of[dev].load(std::memory_order_acquire);
    if (pairs == 0) {
        if (cudaFuncSetAttribute(k_resblock<kStep>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rb::kSmem) !=
            cudaSuccess)
            return -1;
        cfg.gridDim = dim3(2 * (device_sm_count() / 2));
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, k_resblock<kStep>, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();
            return -1;
        }
        pairs = n;
        pairs_of[dev].store(n, std::memory_order_release);
    }
    return pairs;
}

// Checks shared by both entry points; fills the tensor maps and the
// argument block.
static int rb_prepare(const void *x_edit, const sige_tensor_desc *xd, const void *w1, const float *b1,
                      const float *gn1_scale, const float *gn1_shift, const void *w2, const float *b2,
                      const float *gn2_scale, const float *gn2_shift, int32_t block, const int32_t *idx,
                      const int32_t *count, int32_t capacity, void *y1, void *out, void *workspace,
                      size_t workspace_bytes, size_t ws_need, bool maps, RbArgs &a, CUtensorMap &tmx,
                      CUtensorMap &tw1, CUtensorMap &tw2)
{
    if (!x_edit || !xd || !w1 || !w2 || !gn1_scale || !gn1_shift || !gn2_scale || !gn2_shift || !idx || !count ||
        !y1 || !out || capacity < 0)
        return SIGE_ERR_INVALID_ARG;
    if (xd->n < 1 || xd->h < 1 || xd->w < 1 || xd->c < 1 || block < 1)
        return SIGE_ERR_INVALID_ARG;
    if (xd->dtype != SIGE_BF16 || xd->layout != SIGE_NHWC || xd->c != rb::kC || block != rb::kB)
        return SIGE_ERR_UNSUPPORTED;
    if (!aligned(idx, 8))
        return SIGE_ERR_INVALID_ARG;
    if (!aligned(x_edit, 16) || !aligned(w1, 16) || !aligned(w2, 16) || !aligned(y1, 16) || !aligned(out, 16) ||
        !aligned(gn1_scale, 16) || !aligned(gn1_shift, 16) || !aligned(gn2_scale, 16) || !aligned(gn2_shift, 16) ||
        !aligned(b1, 16) || !aligned(b2, 16))
        return SIGE_ERR_UNSUPPORTED;
    const size_t bytes = (size_t)xd->n * xd->h * xd->w * xd->c * 2;
    if (overlaps(x_edit, y1, bytes) || overlaps(x_edit, out, bytes) || overlaps(y1, out, bytes))
        return SIGE_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < ws_need || !aligned(workspace, 16))
        return SIGE_ERR_WORKSPACE;
    if (maps) {
        auto encode = get_encode();
        if (!encode)
            return SIGE_ERR_CUDA;
        if (!encode_halo(&tmx, x_edit, xd->n, xd->h, xd->w, encode) || !encode_weights(&tw1, w1, encode) ||
            !encode_weights(&tw2, w2, encode))
            return SIGE_ERR_UNSUPPORTED;
    }
    a = RbArgs{};
    a.x = static_cast<const uint8_t *>(x_edit);
    a.idx = idx;
    a.count = count;
    a.b1 = b1;
    a.b2 = b2;
    a.g1s = gn1_scale;
    a.g1h = gn1_shift;
    a.g2s = gn2_scale;
    a.g2h = gn2_shift;
    a.y1 = static_cast<uint8_t *>(y1);
    a.out = static_cast<uint8_t *>(out);
    a.hdr = static_cast<WsHeader *>(workspace);
    a.w1 = static_cast<const uint8_t *>(w1);
    a.w2 = static_cast<const uint8_t *>(w2);
    a.N = xd->n;
    a.H = xd->h;
    a.W = xd->w;
    a.cap = capacity;
    return SIGE_OK;
}

template <bool kStep>
static int rb_launch(const RbArgs &a, const CUtensorMap &tmx, const CUtensorMap &tw1, const CUtensorMap &tw2,
                     int64_t units_max, sige_stream_t stream)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return SIGE_ERR_CUDA;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(rb::kThreads);
    cfg.dynamicSmemBytes = rb::kSmem;
    cfg.stream = (cudaStream_t)stream;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    const int pairs = rb_pairs<kStep>(dev, cfg);
    if (pairs < 1)
        return SIGE_ERR_CUDA;
    // the step's grid barrier needs every CTA resident at once: as many pairs
    // as fit (and every unit a pair takes must fit its table); the list call
    // launches no more pairs than there can be units
    int64_t g = pairs;
    if (kStep) {
        if (units_max > (int64_t)rb::kMaxUnits * pairs)
            return SIGE_ERR_UNSUPPORTED;
    } else {
        g = std::min<int64_t>(pairs, units_max);
    }
    cfg.gridDim = dim3(2 * (unsigned)g);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, k_resblock<kStep>, a, tmx, tw1, tw2);
    count_launch();
    if (e != cudaSuccess)
        return SIGE_ERR_CUDA;
    return launch_check();
}

size_t rb_step_workspace_bytes(int32_t tiles)
{
    return kWsHeader + (((size_t)std::max(tiles, 0) * 4 + 15) & ~(size_t)15);
}

} // namespace sige

using namespace sige;

extern "C" int sige_resblock_fused(const void *x_edit, const sige_tensor_desc *xd, const void *w1, const float *b1,
                                   const float *gn1_scale, const float *gn1_shift, const void *w2, const float *b2,
                                   const float *gn2_scale, const float *gn2_shift, int32_t block,
                                   const int32_t *idx, const int32_t *count, int32_t capacity, void *y1, void *out,
                                   void *workspace, size_t workspace_bytes, sige_stream_t stream)
{
    RbArgs a;
    CUtensorMap tmx, tw1, tw2;
    const int st = rb_prepare(x_edit, xd, w1, b1, gn1_scale, gn1_shift, w2, b2, gn2_scale, gn2_shift, block, idx,
                              count, capacity, y1, out, workspace, workspace_bytes, kWsHeader, capacity > 0, a, tmx,
                              tw1, tw2);
    if (st != SIGE_OK || capacity == 0)
        return st;
    return rb_launch<false>(a, tmx, tw1, tw2, (int64_t)capacity * xd->n, stream);
}

extern "C" size_t sige_resblock_step_workspace_bytes(const sige_tensor_desc *xd, int32_t block)
{
    if (!xd || xd->h < 1 || xd->w < 1 || block < 1)
        return 0;
    const int64_t tiles = (int64_t)((xd->h + block - 1) / block) * ((xd->w + block - 1) / block);
    return tiles > INT32_MAX ? 0 : rb_step_workspace_bytes((int32_t)tiles);
}

extern "C" int sige_resblock_step(const void *x_orig, const void *x_edit, const sige_tensor_desc *xd, float threshold,
                                  int32_t dilate, const void *w1, const float *b1, const float *gn1_scale,
                                  const float *gn1_shift, const void *w2, const float *b2, const float *gn2_scale,
                                  const float *gn2_shift, int32_t block, int32_t *idx, int32_t *count,
                                  int32_t capacity, void *y1, void *out, void *workspace, size_t workspace_bytes,
                                  sige_stream_t stream)
{
    if (!x_orig || !(threshold >= 0.0f) || dilate < 0)
        return SIGE_ERR_INVALID_ARG;
    if (!xd || xd->h < 1 || xd->w < 1 || block != rb::kB)
        return !xd || xd->h < 1 || xd->w < 1 || block < 1 ? SIGE_ERR_INVALID_ARG : SIGE_ERR_UNSUPPORTED;
    const int th = (xd->h + block - 1) / block, tw = (xd->w + block - 1) / block;
    if ((int64_t)th * tw > rb::kMaxTiles)
        return SIGE_ERR_UNSUPPORTED;
    RbArgs a;
    CUtensorMap tmx, tw1, tw2;
    const int st = rb_prepare(x_edit, xd, w1, b1, gn1_scale, gn1_shift, w2, b2, gn2_scale, gn2_shift, block, idx,
                              count, capacity, y1, out, workspace, workspace_bytes,
                              rb_step_workspace_bytes(th * tw), false, a, tmx, tw1, tw2);
    if (st != SIGE_OK)
        return st;
    const size_t bytes = (size_t)xd->n * xd->h * xd->w * xd->c * 2;
    if (!aligned(x_orig, 16))
        return SIGE_ERR_UNSUPPORTED;
    if (overlaps(x_orig, y1, bytes) || overlaps(x_orig, out, bytes))
        return SIGE_ERR_INVALID_ARG;
    auto encode = get_encode();
    if (!encode)
        return SIGE_ERR_CUDA;
    if (!encode_halo(&tmx, x_edit, xd->n, xd->h, xd->w, encode) || !encode_weights(&tw1, w1, encode) ||
        !encode_weights(&tw2, w2, encode))
        return SIGE_ERR_UNSUPPORTED;
    a.xo = static_cast<const uint8_t *>(x_orig);
    a.thr = threshold;
    a.dilate = dilate;
    a.th = th;
    a.tw = tw;
    // the arrival counter: 8 bytes at offset 16 of the header
    a.ctr = reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(workspace) + 16);
    a.chunk_ctr = reinterpret_cast<unsigned long long *>(static_cast<uint8_t *>(workspace) + 24);
    a.grid_wait = wait_cycles_or(kWaitCycles);
    a.flags = reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(workspace) + kWsHeader);
    const uint64_t pixels = (uint64_t)xd->n * xd->h * xd->w;
    a.fast_px = pixels <= 0xFFFFFFFFull && (uint64_t)xd->h * xd->w <= (1ull << 31) ? 1 : 0;
    if (a.fast_px) {
        a.div_hw = udiv_make((uint32_t)(xd->h * xd->w));
        a.div_w = udiv_make((uint32_t)xd->w);
    }
    return rb_launch<true>(a, tmx, tw1, tw2, (int64_t)capacity * xd->n, stream);
}
