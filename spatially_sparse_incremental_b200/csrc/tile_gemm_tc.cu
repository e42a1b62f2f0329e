// Stride-1 "same" convolutions (1x1, or 3x3 with padding 1) on a tile list (or
// every tile) as a GEMM over the tiles' pixels:
//   y[pixel][co] = sum_{tap, ci} W[co][tap][ci] * t(x[pixel + tap - pad][ci]) + bias[co] (+ residual),
// one rounding to bf16, for the pixels under the listed tiles; every other
// pixel of y keeps its cached value.  (SIGE project page, "Overview": gather
// the active blocks with their halo, run the layer, scatter the results.  Here
// the gather is the GEMM's operand fill: tap (dr, dc) of the window reads the
// tile shifted by (dr - pad, dc - pad), zero outside the map, which is the
// conv's zero padding.)
//
// A unit is 128 pixel slots (slot s = pixel s mod b^2 of the (tile, batch
// item) pair s / b^2, 128 / b^2 pairs per unit; rows of clipped pixels are
// never written) times up to 128 output channels.  K runs over (tap, 64-channel
// chunk), tap-major, matching the weights' [C_out][k][k][C_in] order:
//   * A, for b = 4 or 8: warp 2 loads, per K chunk, one TMA box of 64 channels
//     x b x b pixels per (tile, item), at the tile's origin shifted by the
//     chunk's tap; it lands as that pair's b^2 rows of the 128-byte-swizzled
//     K-major A layout (row = slot, 128 bytes = 64 channels).  Other tile
//     sizes: warps 4..7, one slot per thread, copy their shifted pixel's
//     chunk with cp.async straight into the same layout (zero-filled outside
//     the map), all stages but one in flight;
//   * warps 4..7 apply GroupNorm + SiLU to their row in place when asked (rows
//     outside the map stay zero) and hand the stage to the MMAs; with no
//     transform and a TMA fill the MMAs take a stage as soon as it lands;
//   * warp 0 loads the weights by TMA (64 channels of one tap x the unit's
//     output channels per stage, 128-byte swizzle), four stages;
//   * warp 1 issues D += A W^T (M 128 slots, N the unit's output channels, K
//     16 per instruction) into tensor memory;
//   * K split: the CTAs of a cluster of 4 take 4 / s units at a time, s CTAs
//     per unit, each running a contiguous share of the K chunks (s: the
//     largest power of two up to 4 such that the units times s fit the grid,
//     every split keeps at least 8 K chunks and nt / s is a power of two of
//     at least 16 columns).  With s > 1 each CTA has a single unit: once every CTA of the
//     unit has finished its MMAs, each pushes column slice i of its float32
//     partial into the A stages of the unit's CTA i, which sums the s slices
//     in split order (the same order every time) and runs the epilogue (bias,
//     residual, bf16) for its slice; with s = 1 the epilogue reads tensor
//     memory directly.
// Persistent clusters over the units; the tile count is read on the device.
// Every mbarrier wait is bounded: on expiry the kernel records
// SIGE_ERR_TIMEOUT in the workspace header and unwinds, and every thread still
// meets the cluster barrier at the end, so no CTA leaves while a peer may
// address its shared memory.
#include <algorithm>
#include <atomic>

#include "conv_tc.cuh"
#include "tc_ptx.cuh"
#include "transform.cuh"

namespace sige {
namespace tg {

constexpr int kThreads = 256;        // warp 0 weights, warp 1 MMA, warp 2 A boxes, warps 4..7 rows + epilogue
constexpr int kRows = 128;
constexpr int kCluster = 4;          // K splits of one unit, at most
constexpr int kAStages = 6, kWStages = 6;
constexpr int kMaxNT = 128;          // output channels per unit
constexpr uint32_t kABytes = kRows * 128;                 // 16 KB
constexpr uint32_t kWBytes = kMaxNT * 128;                // 16 KB at most
constexpr uint32_t kOffA = 0;
// K split: s slices of 128 rows x nt / s floats, received in the A stages (a
// CTA of a split has one unit, whose MMAs are done before peers push)
constexpr uint32_t kOffRecv = kOffA;
constexpr uint32_t kRecvBytes = kRows * kMaxNT * 4;
static_assert(kRecvBytes <= kAStages * kABytes, "receive buffer");
constexpr uint32_t kOffW = kOffA + kAStages * kABytes;
constexpr uint32_t kStage = kOffW;                        // K split: the partial to send, in the weight stages
static_assert(kRecvBytes <= kWStages * kWBytes, "staging buffer");
constexpr uint32_t kOffBias = kOffW + kWStages * kWBytes;  // per rows warp: the unit's bias (kMaxNT floats)
constexpr uint32_t kOffBar = kOffBias + 4 * kMaxNT * 4;
constexpr uint32_t kBarAFull = 0, kBarAEmpty = kBarAFull + 8 * kAStages, kBarALand = kBarAEmpty + 8 * kAStages,
                   kBarWFull = kBarALand + 8 * kAStages, kBarWEmpty = kBarWFull + 8 * kWStages,
                   kBarAccFull = kBarWEmpty + 8 * kWStages, kBarAccEmpty = kBarAccFull + 8,
                   kBarRecv = kBarAccEmpty + 8, kBarReady = kBarRecv + 8, kTmemSlot = kBarReady + 8,
                   kAbort = kTmemSlot + 4;
static_assert(kAbort + 4 <= 512, "barrier block");
constexpr uint32_t kSmem = kOffBar + 512 + 1024;          // + alignment slack
static_assert(kSmem <= 232448, "shared memory per CTA");

enum : int {
    kSiteWEmpty = 301, kSiteWFull, kSiteAFull, kSiteAEmpty, kSiteAccFull, kSiteAccEmpty, kSiteRecv, kSiteReady
};

struct Args {
    const uint8_t *x;          // NHWC bf16 [N][H][W][Cin]
    const int32_t *idx;        // sparse: tile origins (h0, w0)
    const int32_t *count;
    int32_t cap, dense, tiles_w, tiles_total;
    int32_t N, H, W, Cin, Cout, b;   // H, W: the input map
    int32_t k, pad, s;         // kernel size, padding, stride
    int32_t tstride;           // > 0: a transposed conv run as a stride-1 conv over the input with
                               // tstride - 1 zeros between pixels, taps reversed (rows copied per thread)
    int32_t Ho, Wo;            // the output map
    int32_t nt, ntn;           // output channels per unit, units along C_out
    const float *gsc, *gsh;    // GroupNorm affine [N][Cin] (or null)
    int32_t silu;
    const float *bias;
    const uint8_t *residual;   // NHWC bf16 [N][H][W][Cout] (or null)
    uint8_t *y;                // NHWC bf16 [N][H][W][Cout]
    WsHeader *hdr;
    uint32_t tmem_cols;
    int32_t tma_a;             // A by one TMA box per (tile, chunk) (b^2 rows fill whole 1 KB swizzle atoms)
};

__device__ __forceinline__ void tma4(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1, int c2, int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int n>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(n) : "memory"); }

__device__ __forceinline__ float4 lds4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// K chunk q = (tap, 64-channel chunk): the chunk and the tap's offsets from
// the output pixel, stepped along q without divisions.
struct TapPos {
    int cc, dr, dc;
};
__device__ __forceinline__ TapPos tap_at(int q, int kcin, int k, int pad)
{
    const int tap = q / kcin, dr = tap / k;
    return TapPos{q - tap * kcin, dr - pad, tap - dr * k - pad};
}
__device__ __forceinline__ void tap_next(TapPos &t, int kcin, int k, int pad)
{
    if (++t.cc == kcin) {
        t.cc = 0;
        if (++t.dc == k - pad) {
            t.dc = -pad;
            ++t.dr;
        }
    }
}

// 32 columns of this warp's tensor-memory lanes, one wait.
__device__ __forceinline__ void ld32_split(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr + 16u));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < 32; ++k)
        v[k] = __uint_as_float(r[k]);
}

__device__ __forceinline__ void sts4(uint32_t addr, float a, float b, float c, float d)
{
    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}

// Bulk copy of this CTA's shared memory into a peer's, counted on the peer's
// mbarrier (16-byte aligned addresses, a multiple of 16 bytes).
__device__ __forceinline__ void bulk_to_peer(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "r"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// Arrive on a peer's mbarrier with no ordering of this thread's earlier
// memory operations (a "ready" signal that carries no data).
__device__ __forceinline__ void mbar_arrive_peer_relaxed(uint32_t addr)
{
    asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

// D (tensor memory) (+)= A (shared memory) B (shared memory), one elected lane.
__device__ __forceinline__ void mma_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n .reg .pred p, e;\n .reg .b32 l;\n elect.sync l|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
                 " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
                 "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// 16 float32 outputs of one pixel: + bias (shared memory), + residual, one
// rounding to bf16, two 16-byte stores.
__device__ __forceinline__ void store_out16(float (&v)[16], const float4 *bsm, const uint8_t *res, uint8_t *dst)
{
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float4 bq = bsm[q];
        v[4 * q] += bq.x;
        v[4 * q + 1] += bq.y;
        v[4 * q + 2] += bq.z;
        v[4 * q + 3] += bq.w;
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t o[4];
        if (res) {
            const uint4 rq = __ldg(reinterpret_cast<const uint4 *>(res) + h);
            const uint32_t rw[4] = {rq.x, rq.y, rq.z, rq.w};
#pragma unroll
            for (int t = 0; t < 4; ++t)
                o[t] = pack_bf16x2(v[8 * h + 2 * t] + bf16_lo(rw[t]), v[8 * h + 2 * t + 1] + bf16_hi(rw[t]));
        } else {
#pragma unroll
            for (int t = 0; t < 4; ++t)
                o[t] = pack_bf16x2(v[8 * h + 2 * t], v[8 * h + 2 * t + 1]);
        }
        reinterpret_cast<uint4 *>(dst)[h] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

} // namespace tg

using namespace tg;

__global__ void __launch_bounds__(tg::kThreads, 1)
    k_tile_gemm(const __grid_constant__ tg::Args p, const __grid_constant__ CUtensorMap tw,
                const __grid_constant__ CUtensorMap tx)
{
    extern __shared__ __align__(1024) uint8_t tg_raw[];
    const uint32_t raw = smem_u32(tg_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t *smem = tg_raw + (sb - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar = sb + kOffBar;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffBar + kAbort);
    WsHeader *hdr = p.hdr;
    auto a_full = [&](int i) { return bar + kBarAFull + 8u * i; };
    auto a_empty = [&](int i) { return bar + kBarAEmpty + 8u * i; };
    auto a_land = [&](int i) { return bar + kBarALand + 8u * i; };
    auto w_full = [&](int i) { return bar + kBarWFull + 8u * i; };
    auto w_empty = [&](int i) { return bar + kBarWEmpty + 8u * i; };

    pdl_wait();
    const int ntile = p.dense ? p.tiles_total : max(0, min(__ldg(p.count), p.cap));
    const int bb = p.b * p.b, tpb = kRows / bb;             // (tile, item) pairs per unit
    const int64_t items = (int64_t)ntile * p.N;
    const int units = (int)((items + tpb - 1) / tpb) * p.ntn;
    const int kcin = p.Cin >> 6;                            // 64-channel chunks of one tap
    const int kcn = p.k * p.k * kcin;                       // K chunks (tap, channel chunk), tap-major
    // the K split (the same on every CTA: it depends only on the tile count)
    int s = kCluster;
    // (a slice of nt / s columns: a power of two, at least 16)
    while (s > 1 && ((int64_t)units * s > (int64_t)gridDim.x || 8 * s > kcn || p.nt % (16 * s) ||
                     ((p.nt / s) & (p.nt / s - 1))))
        s >>= 1;
    const int per = kCluster / s;                           // units a cluster takes at a time
    const int rank = (int)cluster_rank();
    const int sub = rank / s, split = rank - sub * s, base = sub * s;
    const int u_first = (int)(blockIdx.x / kCluster) * per + sub;
    const int u_step = (int)(gridDim.x / kCluster) * per;
    const int c_lo = split * kcn / s, c_hi = (split + 1) * kcn / s;   // this CTA's K chunks (never empty)
    const int nck = c_hi - c_lo;
    const bool affine = p.gsc != nullptr;
    const bool transform = affine || p.silu;
    const bool relay = transform || !p.tma_a;               // the rows warps stage or transform A

    if (threadIdx.x == 0) {
        for (int i = 0; i < kAStages; ++i) {
            mbar_init(a_full(i), kRows);
            mbar_init(a_empty(i), 1);
            mbar_init(a_land(i), 1);
        }
        for (int i = 0; i < kWStages; ++i) {
            mbar_init(w_full(i), 1);
            mbar_init(w_empty(i), 1);
        }
        mbar_init(bar + kBarAccFull, 1);
        mbar_init(bar + kBarAccEmpty, kRows);
        mbar_init(bar + kBarRecv, 1);                       // + the slices' bytes
        mbar_init(bar + kBarReady, (uint32_t)s);            // every CTA of the unit: MMAs done
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tw)) : "memory");
        if (p.tma_a)
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tx)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(bar + kTmemSlot),
                     "r"(p.tmem_cols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + kOffBar + kTmemSlot);
    // the peers' barriers are initialised before the first remote access: every
    // thread arrives here; the rows warps wait before their first push, the
    // others after their loops
    cluster_arrive();

    if (warp == 0) {
        // ---- weight stages: 64 input channels of one tap x the unit's output channels
        const uint32_t bytes = (uint32_t)p.nt * 128u;
        int it = 0;
        bool ok = true;
        for (int u = u_first; ok && u < units; u += u_step) {
            const int nt = u % p.ntn;
            TapPos tp = tap_at(c_lo, kcin, p.k, p.pad);
            for (int q = c_lo; q < c_hi; ++q, ++it, tap_next(tp, kcin, p.k, p.pad)) {
                const int st = it % kWStages;
                if (it >= kWStages &&
                    !mbar_wait_w(w_empty(st), ((it / kWStages) & 1) ^ 1, abort_flag, hdr, kSiteWEmpty)) {
                    ok = false;
                    break;
                }
                // (a transposed conv reads its taps in reverse order)
                const int wq = p.tstride ? (p.k * p.k - 1 - ((tp.dr + p.pad) * p.k + tp.dc + p.pad)) * kcin + tp.cc : q;
                tma_load_2d_w(sb + kOffW + st * kWBytes, &tw, w_full(st), bytes, wq * 64, nt * p.nt);
            }
        }
        cluster_wait();
    } else if (warp == 1) {
        // ---- D = A W^T, four K=16 steps per 64-channel chunk (128-byte
        // swizzle: 32 bytes per step)
        const uint32_t idesc = idesc_bf16(p.nt);
        int ia = 0, k = 0;
        bool ok = true;
        for (int u = u_first; ok && u < units; u += u_step, ++k) {
            if (k > 0 && !mbar_wait_w(bar + kBarAccEmpty, (k - 1) & 1, abort_flag, hdr, kSiteAccEmpty))
                break;
            for (int q = c_lo; q < c_hi; ++q, ++ia) {
                const int sa = ia % kAStages, sw = ia % kWStages;
                if (!mbar_wait_w(w_full(sw), (ia / kWStages) & 1, abort_flag, hdr, kSiteWFull) ||
                    !mbar_wait_w(relay ? a_full(sa) : a_land(sa), (ia / kAStages) & 1, abort_flag, hdr, kSiteAFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = desc_sw128(sb + kOffA + sa * kABytes), bd = desc_sw128(sb + kOffW + sw * kWBytes);
                for (int kk = 0; kk < 4; ++kk)
                    mma_w(tmem, ad + 2u * kk, bd + 2u * kk, idesc, (q > c_lo || kk > 0) ? 1u : 0u);
                tc_commit_w(a_empty(sa));
                tc_commit_w(w_empty(sw));
            }
            if (ok)
                tc_commit_w(bar + kBarAccFull);
        }
        cluster_wait();
    } else if (warp == 2 && p.tma_a) {
        // ---- A by TMA: per chunk, one box of 64 channels x b x b pixels per
        // (tile, item) of the unit (lane q: pair q) at the tile's origin
        // shifted by the chunk's tap, landing as that pair's b^2 swizzled rows;
        // zero outside the map.  Rows of pairs past the list stay as they
        // are: their outputs are not written.
        int ia = 0;
        bool ok = true;
        for (int u = u_first; ok && u < units; u += u_step) {
            const int blk = u / p.ntn;
            const int64_t T = (int64_t)blk * tpb + lane;
            const bool tv = lane < tpb && T < items;
            int n = 0, h0 = 0, w0 = 0;
            if (tv) {
                const int t = (int)(T / p.N);
                n = (int)(T - (int64_t)t * p.N);
                if (p.dense) {
                    h0 = (t / p.tiles_w) * p.b;
                    w0 = (t % p.tiles_w) * p.b;
                } else {
                    const int2 o = __ldg(reinterpret_cast<const int2 *>(p.idx) + t);
                    h0 = o.x;
                    w0 = o.y;
                }
            }
            const uint32_t bytes = (uint32_t)__popc(__ballot_sync(0xFFFFFFFFu, tv)) * (uint32_t)bb * 128u;
            TapPos tp = tap_at(c_lo, kcin, p.k, p.pad);
            for (int j = 0; j < nck; ++j, tap_next(tp, kcin, p.k, p.pad)) {
                const int g = ia + j, st = g % kAStages;
                if (g >= kAStages &&
                    !mbar_wait_w(a_empty(st), ((g / kAStages) - 1) & 1, abort_flag, hdr, kSiteAEmpty)) {
                    ok = false;
                    break;
                }
                if (lane == 0)
                    mbar_expect_tx(a_land(st), bytes);
                __syncwarp();
                if (tv)
                    tma4(sb + kOffA + st * kABytes + (uint32_t)(lane * bb) * 128u, &tx, a_land(st), tp.cc * 64,
                         w0 * p.s + tp.dc, h0 * p.s + tp.dr, n);
            }
            ia += nck;
        }
        cluster_wait();
    } else if (warp >= 4) {
        cluster_wait();
        // ---- pixel rows (A) and the epilogue; thread = slot r = TMEM lane r
        const int r = (warp & 3) * 32 + lane;
        const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const int w = p.nt / s;                             // output columns this CTA finishes per unit
        const int lw = 31 - __clz(w);                       // log2 w when s > 1
        // 16-byte chunk XOR of a received row (w / 4 chunks, a power of two
        // when s > 1), at most 8 ways
        const int xm = min(w / 4, 8) - 1;
        int ia = 0, k = 0;
        bool ok = true;
        for (int u = u_first; ok && u < units; u += u_step, ++k) {
            const int blk = u / p.ntn, nt = u % p.ntn;
            // this slot's output pixel (or none)
            const int64_t T = (int64_t)blk * tpb + r / bb;
            bool valid = r < tpb * bb && T < items;
            int n = 0, yy = 0, xx = 0;
            if (valid) {
                const int t = (int)(T / p.N);
                n = (int)(T - (int64_t)t * p.N);
                int h0, w0;
                if (p.dense) {
                    h0 = (t / p.tiles_w) * p.b;
                    w0 = (t % p.tiles_w) * p.b;
                } else {
                    const int2 o = __ldg(reinterpret_cast<const int2 *>(p.idx) + t);
                    h0 = o.x;
                    w0 = o.y;
                }
                const int sl = r % bb;
                yy = h0 + sl / p.b;
                xx = w0 + sl % p.b;
                valid = h0 >= 0 && w0 >= 0 && yy < p.Ho && xx < p.Wo;
            }
            const int64_t pix = ((int64_t)n * p.Ho + yy) * p.Wo + xx;
            // the slot's pixel shifted by a chunk's tap; false outside the map
            // (a zero row: the conv's padding)
            auto tap_in = [&](const TapPos &t, int64_t &ipix) -> bool {
                int yi = yy * p.s + t.dr, xi = xx * p.s + t.dc;
                if (p.tstride > 0) {
                    // the virtual input holds x[y / t][x / t] where both are
                    // multiples of t, zero elsewhere
                    if (yi < 0 || xi < 0)
                        return false;
                    if (p.tstride == 2) {
                        if ((yi | xi) & 1)
                            return false;
                        yi >>= 1;
                        xi >>= 1;
                    } else {
                        if (yi % p.tstride || xi % p.tstride)
                            return false;
                        yi /= p.tstride;
                        xi /= p.tstride;
                    }
                }
                ipix = ((int64_t)n * p.H + yi) * p.W + xi;
                return valid && yi >= 0 && yi < p.H && xi >= 0 && xi < p.W;
            };
            TapPos t_issue = tap_at(c_lo, kcin, p.k, p.pad), t_use = t_issue;
            // GroupNorm + SiLU of this slot's row of stage st in place
            auto transform_row = [&](int st, int cc) {
                const uint32_t row = sb + kOffA + st * kABytes + (uint32_t)r * 128u;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t a = row + ((uint32_t)(c ^ (r & 7)) << 4);
                    uint4 v;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                                 : "r"(a));
                    const int c0 = cc * 64 + c * 8;
                    v = transform16(v, SIGE_BF16, affine ? p.gsc + (int64_t)n * p.Cin + c0 : nullptr,
                                    affine ? p.gsh + (int64_t)n * p.Cin + c0 : nullptr, p.silu);
                    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z),
                                 "r"(v.w)
                                 : "memory");
                }
            };
            // chunk j (called in order of j) into ring stage (ia + j) mod
            // kAStages once the MMAs of the chunk kAStages back have released it
            auto issue = [&](int j) -> bool {
                const int g = ia + j, st = g % kAStages;
                if (g >= kAStages &&
                    !mbar_wait_w(a_empty(st), ((g / kAStages) - 1) & 1, abort_flag, hdr, kSiteAEmpty))
                    return false;
                int64_t ipix;
                const bool in = tap_in(t_issue, ipix);
                const uint8_t *src = in ? p.x + (ipix * p.Cin + t_issue.cc * 64) * 2 : p.x;
                tap_next(t_issue, kcin, p.k, p.pad);
                const uint32_t nbytes = in ? 16u : 0u;            // 0: the copy writes zeros
                const uint32_t dst = sb + kOffA + st * kABytes + (uint32_t)r * 128u;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    cp_async16(dst + ((uint32_t)(c ^ (r & 7)) << 4), in ? src + c * 16 : p.x, nbytes);
                return true;
            };
            // this warp's copy of the unit's bias (read from shared memory in
            // the epilogue rather than by global loads behind the tensor-memory
            // waits)
            {
                const uint32_t bw = sb + kOffBias + (uint32_t)(warp & 3) * (kMaxNT * 4);
                for (int c = lane; c < p.nt; c += 32)
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(bw + 4u * c),
                                 "f"(p.bias ? __ldg(p.bias + nt * p.nt + c) : 0.0f)
                                 : "memory");
                __syncwarp();
            }
            if (relay && p.tma_a) {
                for (int j = 0; ok && j < nck; ++j) {
                    // A landed by TMA: transform this row in place, then hand
                    // the stage to the MMAs
                    const int g = ia + j, st = g % kAStages;
                    if (!mbar_wait_w(a_land(st), (g / kAStages) & 1, abort_flag, hdr, kSiteAFull)) {
                        ok = false;
                        break;
                    }
                    int64_t ipix;
                    if (tap_in(t_use, ipix))
                        transform_row(st, t_use.cc);
                    tap_next(t_use, kcin, p.k, p.pad);
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_arrive(a_full(st));
                }
            } else if (relay) {
                for (int j = 0; j < kAStages - 1; ++j) {
                    if (j < nck && !issue(j)) {
                        ok = false;
                        break;
                    }
                    cp_async_commit();
                }
                for (int j = 0; ok && j < nck; ++j) {
                    // chunk j first (its group is the oldest of those in
                    // flight), then the refill of the stage the MMAs of chunk
                    // j - 1 release: chunk j never waits for an MMA
                    cp_async_wait<kAStages - 2>();
                    const int st = (ia + j) % kAStages;
                    int64_t ipix;
                    if (tap_in(t_use, ipix) && transform)
                        transform_row(st, t_use.cc);
                    tap_next(t_use, kcin, p.k, p.pad);
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_arrive(a_full(st));
                    const int jn = j + kAStages - 1;
                    if (jn < nck && !issue(jn)) {
                        ok = false;
                        break;
                    }
                    cp_async_commit();
                }
                cp_async_wait<0>();
            }
            if (!__all_sync(0xFFFFFFFFu, ok))
                break;
            ia += nck;
            if (!mbar_wait_w(bar + kBarAccFull, k & 1, abort_flag, hdr, kSiteAccFull)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int co0 = nt * p.nt;
            const float4 *bsm = reinterpret_cast<const float4 *>(smem + kOffBias + (warp & 3) * (kMaxNT * 4));
            if (s == 1) {
                // ---- epilogue from tensor memory, 32 output channels per wait
                // (the loads stay inside the allocation, a power of two >= 32)
                uint8_t *dst = p.y + (pix * p.Cout + co0) * 2;
                const uint8_t *res = p.residual ? p.residual + (pix * p.Cout + co0) * 2 : nullptr;
                for (int c0 = 0; c0 < p.nt; c0 += 32) {
                    float v[32];
                    ld32_split(t_row + (uint32_t)c0, v);
                    if (!valid)
                        continue;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int c = c0 + 16 * h;
                        if (c < p.nt) {
                            float part[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                part[e] = v[16 * h + e];
                            store_out16(part, bsm + c / 4, res ? res + c * 2 : nullptr, dst + c * 2);
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(bar + kBarAccEmpty);
                continue;
            }
            // ---- K split (this CTA's only unit).  The partial goes, column
            // slice i by column slice i, into a staging copy in this CTA's
            // weight stages ([slice][row][w floats]); once every CTA of the
            // unit has finished its MMAs (its A stages become the receive
            // buffer, [sender][row][w floats]), one bulk copy per slice moves
            // slice i to the unit's CTA i, counted on its receive barrier.  The
            // CTAs send in a rotated order, so that every CTA receives from one
            // sender at a time.
            if (warp == 4) {
                if (lane == 0)
                    mbar_expect_tx(bar + kBarRecv, (uint32_t)(s * kRows * w * 4));
                __syncwarp();
                if (lane < s)
                    mbar_arrive_peer_relaxed(map_peer(bar + kBarReady, (uint32_t)(base + lane)));
            }
            const uint32_t slice = (uint32_t)(kRows * w * 4);
            for (int c0 = 0; c0 < p.nt; c0 += 32) {
                float v[32];
                ld32_split(t_row + (uint32_t)c0, v);        // within the allocation (a power of two >= 32)
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int col = c0 + 4 * q;
                    if (col < p.nt) {
                        const int i = col >> lw, c = (col & (w - 1)) >> 2;   // slice, 16-byte chunk of its row
                        sts4(sb + kStage + (uint32_t)i * slice + (uint32_t)r * (uint32_t)w * 4u +
                                 ((uint32_t)(c ^ (r & xm)) << 4),
                             v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                    }
                }
            }
            tc_fence_before();
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            asm volatile("bar.sync 1, 128;" ::: "memory");   // the four rows warps: staging complete
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_cluster(bar + kBarReady, 0, abort_flag, hdr, kSiteReady))) {
                ok = false;
                break;
            }
            if (warp == 4 && lane < s) {
                const int i = (split + lane) & (s - 1);
                bulk_to_peer(map_peer(sb + kOffRecv + (uint32_t)split * slice, (uint32_t)(base + i)),
                             sb + kStage + (uint32_t)i * slice, slice, map_peer(bar + kBarRecv, (uint32_t)(base + i)));
            }
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_cluster(bar + kBarRecv, 0, abort_flag, hdr, kSiteRecv))) {
                ok = false;
                break;
            }
            // ---- this CTA's slice: the s partials summed in split order
            {
                const int cs = co0 + split * w;
                uint8_t *dst = p.y + (pix * p.Cout + cs) * 2;
                const uint8_t *res = p.residual ? p.residual + (pix * p.Cout + cs) * 2 : nullptr;
                for (int c0 = 0; c0 < w; c0 += 16) {
                    float v[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        v[e] = 0.0f;
                    for (int i = 0; i < s; ++i) {
                        const uint32_t row = sb + kOffRecv + (uint32_t)(i * kRows + r) * (uint32_t)w * 4u;
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 x4 = lds4(row + ((uint32_t)((c0 / 4 + q) ^ (r & xm)) << 4));
                            v[4 * q] += x4.x;
                            v[4 * q + 1] += x4.y;
                            v[4 * q + 2] += x4.z;
                            v[4 * q + 3] += x4.w;
                        }
                    }
                    if (valid)
                        store_out16(v, bsm + (split * w + c0) / 4, res ? res + c0 * 2 : nullptr, dst + c0 * 2);
                }
            }
        }
        cp_async_wait<0>();
    } else {
        cluster_wait();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols));
    }
    // no CTA leaves while a peer may still address its shared memory
    cluster_arrive();
    cluster_wait();
}

// ------------------------------------------------------------------ input transform pre-pass

// For a 3x3 layer with an input transform (GroupNorm affine, SiLU, or the
// GauGAN-style per-pixel modulation and LeakyReLU): the
// transform of every input pixel the listed tiles' taps read (the halo of
// each tile, or the whole map for a dense call) is written once into a
// scratch copy of the input, which the GEMM then reads untransformed, instead
// of transforming each tap's copy of a row (nine times the work).  Pixels of
// overlapping halos are written with the same value by every tile that
// covers them.
struct PreArgs {
    const uint8_t *x;          // NHWC bf16 [N][H][W][Cin]
    uint8_t *xt;               // the scratch copy, same layout
    const int32_t *idx, *count;
    int32_t cap, dense;
    int32_t N, H, W, Cin, b, s, pad, hb;   // hb: halo side (b - 1) s + 3
    const float *gsc, *gsh;
    int32_t silu;
    const uint8_t *sg, *sb;    // per-pixel modulation maps (input shape, NHWC bf16) or null
    int32_t leaky;             // LeakyReLU(0.2) instead of SiLU
    UDiv dvpp, dhb, dN, dW, dH;
};

__global__ void __launch_bounds__(256) k_tile_pretransform(const __grid_constant__ PreArgs p)
{
    pdl_wait();
    const uint32_t vpp = (uint32_t)(p.Cin / 8);
    const uint32_t per_tile = (uint32_t)(p.hb * p.hb) * vpp;
    const uint32_t total = p.dense ? (uint32_t)p.N * (uint32_t)p.H * (uint32_t)p.W * vpp
                                   : (uint32_t)max(0, min(__ldg(p.count), p.cap)) * (uint32_t)p.N * per_tile;
    for (uint32_t v = blockIdx.x * blockDim.x + threadIdx.x; v < total; v += gridDim.x * blockDim.x) {
        uint32_t q = udiv(v, p.dvpp);
        const uint32_t cv = v - q * vpp;
        int n, y, x;
        if (p.dense) {
            const uint32_t r = q;                               // pixel n H W + y W + x
            q = udiv(r, p.dW);
            x = (int)(r - q * (uint32_t)p.W);
            const uint32_t q2 = udiv(q, p.dH);
            y = (int)(q - q2 * (uint32_t)p.H);
            n = (int)q2;
        } else {
            uint32_t r = q;
            q = udiv(r, p.dhb);
            const int ww = (int)(r - q * (uint32_t)p.hb);
            r = q;
            q = udiv(r, p.dhb);
            const int hh = (int)(r - q * (uint32_t)p.hb);
            r = q;
            q = p.N == 1 ? r : udiv(r, p.dN);
            n = (int)(r - q * (uint32_t)p.N);
            const int2 o = __ldg(reinterpret_cast<const int2 *>(p.idx) + q);
            y = o.x * p.s - p.pad + hh;
            x = o.y * p.s - p.pad + ww;
            if (y < 0 || y >= p.H || x < 0 || x >= p.W)
                continue;
        }
        const int64_t e = (((int64_t)n * p.H + y) * p.W + x) * p.Cin + (int64_t)cv * 8;
        const uint4 in = ld_nc16(p.x + e * 2);
        const float *sc = p.gsc ? p.gsc + (int64_t)n * p.Cin + cv * 8 : nullptr;
        const float *sh = p.gsc ? p.gsh + (int64_t)n * p.Cin + cv * 8 : nullptr;
        uint4 out;
        if (p.sg || p.leaky) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            out = transform16_mod(in, sc, sh, p.sg != nullptr, p.sg ? ld_nc16(p.sg + e * 2) : z,
                                  p.sb ? ld_nc16(p.sb + e * 2) : z, p.silu, p.leaky);
        } else {
            // the 8 channels' scale and shift by four 16-byte loads (8 scalar
            // loads each throttled the memory pipe)
            float gsc8[8], gsh8[8];
            if (sc) {
                const float4 a0 = __ldg(reinterpret_cast<const float4 *>(sc)), a1 = __ldg(reinterpret_cast<const float4 *>(sc) + 1);
                const float4 b0 = __ldg(reinterpret_cast<const float4 *>(sh)), b1 = __ldg(reinterpret_cast<const float4 *>(sh) + 1);
                gsc8[0] = a0.x; gsc8[1] = a0.y; gsc8[2] = a0.z; gsc8[3] = a0.w;
                gsc8[4] = a1.x; gsc8[5] = a1.y; gsc8[6] = a1.z; gsc8[7] = a1.w;
                gsh8[0] = b0.x; gsh8[1] = b0.y; gsh8[2] = b0.z; gsh8[3] = b0.w;
                gsh8[4] = b1.x; gsh8[5] = b1.y; gsh8[6] = b1.z; gsh8[7] = b1.w;
            }
            out = transform16_bf16_reg(in, gsc8, gsh8, sc != nullptr, p.silu);
        }
        reinterpret_cast<uint4 *>(p.xt)[e / 8] = out;
    }
}

// ------------------------------------------------------------------ host

bool tile_gemm_supported(const sige_conv_desc *cd, int dtype, bool dense)
{
    if (!cd || dtype != SIGE_BF16 || cd->stride < 1 || cd->stride > 2 || cd->block < 1 ||
        cd->block * cd->block > tg::kRows ||
        cd->c_in < 64 || cd->c_in % 64 || cd->c_out < 16 || cd->c_out % 16)
        return false;
    if ((long long)cd->kernel * cd->kernel * cd->c_in >= (1ll << 31))
        return false;
    // 1x1 stride 1 (any tile size), or 3x3 padding 1, stride 1 or 2, on 4x4
    // or 8x8 tiles, whose tap-shifted (and strided) boxes the TMA fills.  On
    // other tile sizes the rows are copied per thread: a dense call (every
    // tile, many units) still gains (2.1x on the 1x1 / 2x2-tile layers), and
    // so do sparse calls on one-pixel tiles (128 tiles per unit; 10-12%), but
    // sparse calls on 2x2 tiles measured from 7% faster to 12% slower than
    // the general kernel, which keeps them.
    return (cd->kernel == 1 && cd->pad == 0 && cd->stride == 1) ||
           (cd->kernel == 3 && cd->pad == 1 &&
            (dense || cd->block == 1 || (cd->block * cd->block) % 8 == 0));
}

int launch_tile_gemm(const ConvParams &cp, cudaStream_t stream)
{
    auto encode = get_encode();
    if (!encode)
        return SIGE_ERR_CUDA;
    tg::Args a{};
    a.x = cp.src;
    a.idx = cp.idx;
    a.count = cp.count;
    a.cap = cp.cap;
    a.dense = cp.dense;
    a.tiles_w = cp.tiles_w;
    a.tiles_total = cp.tiles_total;
    a.N = cp.N;
    a.H = cp.H;
    a.W = cp.W;
    a.s = cp.s;
    a.tstride = cp.tstride;
    a.Ho = cp.Ho;
    a.Wo = cp.Wo;
    a.Cin = cp.Cin;
    a.Cout = cp.Cout;
    a.b = cp.b;
    a.k = cp.k;
    a.pad = cp.pad;
    // output channels per unit: all of them up to 128, else the largest of
    // 128, 64, 32, 16 that divides C_out
    a.nt = cp.Cout;
    if (a.nt > tg::kMaxNT) {
        a.nt = tg::kMaxNT;
        while (cp.Cout % a.nt)
            a.nt >>= 1;
    }
    a.ntn = cp.Cout / a.nt;
    a.gsc = cp.gsc;
    a.gsh = cp.gsh;
    a.silu = cp.silu;
    a.bias = cp.bias;
    a.residual = cp.residual;
    a.y = cp.y;
    a.hdr = reinterpret_cast<WsHeader *>(cp.ws);
    uint32_t tc = 32;
    while (tc < (uint32_t)a.nt)
        tc <<= 1;
    a.tmem_cols = tc;
    // weights [C_out][k][k][C_in] as a 2-d map {k k C_in, C_out}: a box of 64
    // input channels of one tap x the unit's output channels lands as 128-byte
    // rows with the 128-byte swizzle
    CUtensorMap tw;
    const uint64_t kdim = (uint64_t)cp.k * cp.k * cp.Cin;
    cuuint64_t dims[2] = {(cuuint64_t)kdim, (cuuint64_t)cp.Cout};
    cuuint64_t strides[1] = {(cuuint64_t)kdim * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)a.nt};
    cuuint32_t es[2] = {1, 1};
    if (encode(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint8_t *>(cp.w), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return SIGE_ERR_UNSUPPORTED;
    // the input [N][H][W][C_in] as a 4-d map: a box of 64 channels x b x b
    // pixels of one item lands as the tile's b^2 rows of 128 bytes, 128-byte
    // swizzle, zero outside the map (also at the negative coordinates of a
    // shifted tap).  Used when b^2 rows fill whole 1 KB swizzle atoms (b = 4
    // or 8), so that every box starts on an atom.
    CUtensorMap tx = tw;
    a.tma_a = 0;
    if ((cp.b * cp.b) % 8 == 0 && cp.tstride == 0) {
        cuuint64_t xd[4] = {(cuuint64_t)cp.Cin, (cuuint64_t)cp.W, (cuuint64_t)cp.H, (cuuint64_t)cp.N};
        cuuint64_t xs[3] = {(cuuint64_t)cp.Cin * 2, (cuuint64_t)cp.W * cp.Cin * 2, (cuuint64_t)cp.H * cp.W * cp.Cin * 2};
        // (stride s: a box of b s pixels per side read every s-th pixel, b per side)
        cuuint32_t xb[4] = {64, (cuuint32_t)(cp.b * cp.s), (cuuint32_t)(cp.b * cp.s), 1};
        cuuint32_t xe[4] = {1, (cuuint32_t)cp.s, (cuuint32_t)cp.s, 1};
        if (encode(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint8_t *>(cp.src), xd, xs, xb, xe,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            a.tma_a = 1;
        else
            tx = tw;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return SIGE_ERR_CUDA;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = tg::kCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(tg::kThreads);
    cfg.dynamicSmemBytes = tg::kSmem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static std::atomic<int> clusters_of[64];   // co-resident clusters, per device
    int ncl = clusters_of[dev].load(std::memory_order_acquire);
    if (ncl == 0) {
        if (cudaFuncSetAttribute(k_tile_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tg::kSmem) !=
            cudaSuccess)
            return SIGE_ERR_CUDA;
        prefer_max_shared(k_tile_gemm);
        cfg.gridDim = dim3(tg::kCluster * (device_sm_count() / tg::kCluster));
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, k_tile_gemm, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();
            return SIGE_ERR_CUDA;
        }
        ncl = n;
        clusters_of[dev].store(n, std::memory_order_release);
    }
    const int tpb = tg::kRows / (cp.b * cp.b);
    const int64_t pairs = (int64_t)(cp.dense ? cp.tiles_total : cp.cap) * cp.N;
    const int64_t units_max = (pairs + tpb - 1) / tpb * a.ntn;
    if (units_max > INT32_MAX / tg::kCluster)
        return SIGE_ERR_INVALID_ARG;
    // a unit needs at most one cluster (a K split of 4)
    cfg.gridDim = dim3((unsigned)(tg::kCluster * std::max<int64_t>(1, std::min<int64_t>(ncl, units_max))));
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, k_tile_gemm, a, tw, tx) != cudaSuccess)
        return SIGE_ERR_CUDA;
    count_launch();
    return launch_check();
}

size_t tile_gemm_scratch_bytes(const sige_conv_desc *cd, int batch, int in_h, int in_w)
{
    if (!cd || cd->kernel != 3)
        return 0;
    return ((size_t)batch * in_h * in_w * cd->c_in * 2 + 255) & ~(size_t)255;
}

int launch_tile_gemm_pre(const ConvParams &cp, uint8_t *scratch, cudaStream_t stream)
{
    PreArgs a{};
    a.x = cp.src;
    a.xt = scratch;
    a.idx = cp.idx;
    a.count = cp.count;
    a.cap = cp.cap;
    a.dense = cp.dense;
    a.N = cp.N;
    a.H = cp.H;
    a.W = cp.W;
    a.Cin = cp.Cin;
    a.b = cp.b;
    a.s = cp.s;
    a.pad = cp.pad;
    a.hb = (cp.b - 1) * cp.s + cp.k;
    a.gsc = cp.gsc;
    a.gsh = cp.gsh;
    a.silu = cp.silu;
    a.sg = cp.sg;
    a.sb = cp.sb;
    a.leaky = cp.leaky;
    a.dvpp = udiv_make((uint32_t)(cp.Cin / 8));
    a.dhb = udiv_make((uint32_t)a.hb);
    a.dN = udiv_make((uint32_t)cp.N);
    a.dW = udiv_make((uint32_t)cp.W);
    a.dH = udiv_make((uint32_t)cp.H);
    const int64_t work = cp.dense ? (int64_t)cp.N * cp.H * cp.W * (cp.Cin / 8)
                                  : (int64_t)cp.cap * cp.N * a.hb * a.hb * (cp.Cin / 8);
    if (work > 0xFFFFFFFFll)
        return SIGE_ERR_UNSUPPORTED;
    // (a sparse call's grid is sized for the capacity; its tiles are read on
    // the device, usually far fewer)
    const int grid = (int)std::max<int64_t>(
        1, std::min<int64_t>((work + 255) / 256, (int64_t)device_sm_count() * (cp.dense ? 8 : 2)));
    if (launch_pdl(k_tile_pretransform, dim3(grid), dim3(256), 0, stream, a) != cudaSuccess)
        return SIGE_ERR_CUDA;
    count_launch();
    int rc = launch_check();
    if (rc != SIGE_OK)
        return rc;
    ConvParams g = cp;
    g.src = scratch;
    g.gsc = nullptr;
    g.gsh = nullptr;
    g.silu = 0;
    g.sg = nullptr;
    g.sb = nullptr;
    g.leaky = 0;
    return launch_tile_gemm(g, stream);
}

} // namespace sige
