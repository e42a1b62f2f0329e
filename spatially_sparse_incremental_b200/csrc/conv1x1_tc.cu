// 1x1 stride-1 layers on a tile list (or every tile) as a GEMM over gathered
// pixels: y[pixel][co] = sum_ci W[co][ci] * t(x[pixel][ci]) + bias[co]
// (+ residual), one rounding to bf16, for the pixels under the listed tiles;
// every other pixel of y keeps its cached value.  (SIGE project page,
// "Overview": gather the active blocks, run the layer, scatter the results; a
// 1x1 conv needs no halo, so the gather is a row gather.)
//
// A unit is 128 pixel slots (slot s = pixel s mod b^2 of the (tile, batch
// item) pair s / b^2, 128 / b^2 pairs per unit; rows of clipped pixels are
// zero, slots past the list are computed and not written) times up to 128
// output channels:
//   * A, for b = 4 or 8: warp 2 loads one TMA box of 64 channels x b x b
//     pixels per (tile, item) and chunk, which lands as that pair's b^2 rows
//     of the 128-byte-swizzled K-major A layout (row = slot, 128 bytes = 64
//     channels; zero outside the map); other tile sizes: warps 4..7, one slot
//     per thread, copy their pixel's chunks with cp.async straight into the
//     same layout, seven of eight stages in flight;
//   * warps 4..7 apply GroupNorm + SiLU to their row in place when asked, hand
//     the stage to the MMAs, and run the epilogue from tensor memory (bias,
//     residual, bf16);
//   * warp 0 loads the weights [C_out][C_in] by TMA (64 channels x the unit's
//     output channels per stage, 128-byte swizzle), four stages;
//   * warp 1 issues D += A W^T (M 128 slots, N the unit's output channels,
//     K 16 per instruction) into tensor memory.
// Persistent CTAs over the units; the tile count is read on the device.
#include <algorithm>
#include <atomic>

#include "conv_tc.cuh"
#include "tc_ptx.cuh"
#include "transform.cuh"

namespace sige {
namespace g1 {

constexpr int kThreads = 256;        // warp 0 weights, warp 1 MMA, warps 4..7 pixel rows + epilogue
constexpr int kRows = 128;
constexpr int kAStages = 8, kWStages = 4;
constexpr int kMaxNT = 128;          // output channels per unit
constexpr uint32_t kABytes = kRows * 128;                 // 16 KB
constexpr uint32_t kWBytes = kMaxNT * 128;                // 16 KB at most
constexpr uint32_t kOffA = 0;
constexpr uint32_t kOffW = kOffA + kAStages * kABytes;
constexpr uint32_t kOffBias = kOffW + kWStages * kWBytes;  // per rows warp: the unit's bias (kMaxNT floats)
constexpr uint32_t kOffBar = kOffBias + 4 * kMaxNT * 4;
constexpr uint32_t kBarAFull = 0, kBarAEmpty = kBarAFull + 8 * kAStages, kBarALand = kBarAEmpty + 8 * kAStages,
                   kBarWFull = kBarALand + 8 * kAStages, kBarWEmpty = kBarWFull + 8 * kWStages,
                   kBarAccFull = kBarWEmpty + 8 * kWStages, kBarAccEmpty = kBarAccFull + 8,
                   kTmemSlot = kBarAccEmpty + 8, kAbort = kTmemSlot + 4;
static_assert(kAbort + 4 <= 512, "barrier block");
constexpr uint32_t kSmem = kOffBar + 512 + 1024;          // + alignment slack

enum : int { kSiteWEmpty = 301, kSiteWFull, kSiteAFull, kSiteAEmpty, kSiteAccFull, kSiteAccEmpty };

struct Args {
    const uint8_t *x;          // NHWC bf16 [N][H][W][Cin]
    const int32_t *idx;        // sparse: tile origins (h0, w0)
    const int32_t *count;
    int32_t cap, dense, tiles_w, tiles_total;
    int32_t N, H, W, Cin, Cout, b;
    int32_t nt, ntn;           // output channels per unit, units along C_out
    const float *gsc, *gsh;    // GroupNorm affine [N][Cin] (or null)
    int32_t silu;
    const float *bias;
    const uint8_t *residual;   // NHWC bf16 [N][H][W][Cout] (or null)
    uint8_t *y;                // NHWC bf16 [N][H][W][Cout]
    WsHeader *hdr;
    uint32_t tmem_cols;
    int32_t tma_a;             // A by one TMA per (tile, chunk) (b^2 rows fill whole 1 KB swizzle atoms)
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

__device__ __forceinline__ void ld16(uint32_t taddr, float (&v)[16])
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

// D (tensor memory) (+)= A (shared memory) B (shared memory), one elected lane.
__device__ __forceinline__ void mma_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n .reg .pred p, e;\n .reg .b32 l;\n elect.sync l|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
                 " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
                 "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
                 : "memory");
}

} // namespace g1

using namespace g1;

__global__ void __launch_bounds__(g1::kThreads, 1)
    k_conv1x1(const __grid_constant__ g1::Args p, const __grid_constant__ CUtensorMap tw,
              const __grid_constant__ CUtensorMap tx)
{
    extern __shared__ __align__(1024) uint8_t g1_raw[];
    const uint32_t raw = smem_u32(g1_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t *smem = g1_raw + (sb - raw);
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
    const int kcn = p.Cin / 64;

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

    if (warp == 0) {
        // ---- weight stages: 64 input channels x the unit's output channels
        const uint32_t bytes = (uint32_t)p.nt * 128u;
        int it = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
            const int nt = u % p.ntn;
            for (int kc = 0; kc < kcn; ++kc, ++it) {
                const int st = it % kWStages;
                if (it >= kWStages &&
                    !mbar_wait_w(w_empty(st), ((it / kWStages) & 1) ^ 1, abort_flag, hdr, kSiteWEmpty)) {
                    ok = false;
                    break;
                }
                tma_load_2d_w(sb + kOffW + st * kWBytes, &tw, w_full(st), bytes, kc * 64, nt * p.nt);
            }
        }
    } else if (warp == 1) {
        // ---- D = A W^T, four K=16 steps per 64-channel chunk (128-byte
        // swizzle: 32 bytes per step)
        const uint32_t idesc = idesc_bf16(p.nt);
        int ia = 0, k = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < units; u += gridDim.x, ++k) {
            if (k > 0 && !mbar_wait_w(bar + kBarAccEmpty, (k - 1) & 1, abort_flag, hdr, kSiteAccEmpty))
                break;
            for (int kc = 0; kc < kcn; ++kc, ++ia) {
                const int sa = ia % kAStages, sw = ia % kWStages;
                if (!mbar_wait_w(w_full(sw), (ia / kWStages) & 1, abort_flag, hdr, kSiteWFull) ||
                    !mbar_wait_w(a_full(sa), (ia / kAStages) & 1, abort_flag, hdr, kSiteAFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = desc_sw128(sb + kOffA + sa * kABytes), bd = desc_sw128(sb + kOffW + sw * kWBytes);
                for (int kk = 0; kk < 4; ++kk)
                    mma_w(tmem, ad + 2u * kk, bd + 2u * kk, idesc, (kc > 0 || kk > 0) ? 1u : 0u);
                tc_commit_w(a_empty(sa));
                tc_commit_w(w_empty(sw));
            }
            if (ok)
                tc_commit_w(bar + kBarAccFull);
        }
    } else if (warp == 2 && p.tma_a) {
        // ---- A by TMA: per chunk, one box of 64 channels x b x b pixels per
        // (tile, item) of the unit (lane q: pair q), landing as that pair's b^2
        // swizzled rows; zero outside the map.  Rows of pairs past the list
        // stay as they are: their outputs are not written.
        int ia = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
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
            for (int kc = 0; kc < kcn; ++kc) {
                const int g = ia + kc, st = g % kAStages;
                if (g >= kAStages &&
                    !mbar_wait_w(a_empty(st), ((g / kAStages) - 1) & 1, abort_flag, hdr, kSiteAEmpty)) {
                    ok = false;
                    break;
                }
                if (lane == 0)
                    mbar_expect_tx(a_land(st), bytes);
                __syncwarp();
                if (tv)
                    tma4(sb + kOffA + st * kABytes + (uint32_t)(lane * bb) * 128u, &tx, a_land(st), kc * 64, w0, h0, n);
            }
            ia += kcn;
        }
    } else if (warp >= 4) {
        // ---- pixel rows (A) and the epilogue; thread = slot r = TMEM lane r
        const int r = (warp & 3) * 32 + lane;
        const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const bool affine = p.gsc != nullptr;
        const bool transform = affine || p.silu;
        int ia = 0, k = 0;
        bool ok = true;
        for (int u = blockIdx.x; ok && u < units; u += gridDim.x, ++k) {
            const int blk = u / p.ntn, nt = u % p.ntn;
            // this slot's pixel (or none)
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
                const int s = r % bb;
                yy = h0 + s / p.b;
                xx = w0 + s % p.b;
                valid = h0 >= 0 && w0 >= 0 && yy < p.H && xx < p.W;
            }
            const int64_t pix = ((int64_t)n * p.H + yy) * p.W + xx;
            const uint8_t *src = p.x + pix * p.Cin * 2;
            const uint32_t nbytes = valid ? 16u : 0u;            // 0: the copy writes zeros
            // A chunk j of this unit into ring stage (ia + j) mod 8 once the MMAs
            // of the chunk eight back have released it
            auto issue = [&](int j) -> bool {
                const int g = ia + j, st = g % kAStages;
                if (g >= kAStages &&
                    !mbar_wait_w(a_empty(st), ((g / kAStages) - 1) & 1, abort_flag, hdr, kSiteAEmpty))
                    return false;
                const uint32_t dst = sb + kOffA + st * kABytes + (uint32_t)r * 128u;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    cp_async16(dst + ((uint32_t)(c ^ (r & 7)) << 4), valid ? src + j * 128 + c * 16 : p.x, nbytes);
                return true;
            };
            // this warp's copy of the unit's bias (read per output piece from
            // shared memory rather than by a global load behind each
            // tensor-memory wait)
            {
                const uint32_t bw = sb + kOffBias + (uint32_t)(warp & 3) * (kMaxNT * 4);
                for (int c = lane; c < p.nt; c += 32)
                    asm volatile("st.shared.f32 [%0], %1;" ::"r"(bw + 4u * c), "f"(p.bias ? __ldg(p.bias + nt * p.nt + c) : 0.0f)
                                 : "memory");
                __syncwarp();
            }
            for (int j = 0; !p.tma_a && j < kAStages - 1; ++j) {
                if (j < kcn && !issue(j)) {
                    ok = false;
                    break;
                }
                cp_async_commit();
            }
            for (int kc = 0; p.tma_a && ok && kc < kcn; ++kc) {
                // A landed by TMA: GroupNorm + SiLU of this row in place when
                // asked, then hand the stage to the MMAs
                const int g = ia + kc, st = g % kAStages;
                if (!mbar_wait_w(a_land(st), (g / kAStages) & 1, abort_flag, hdr, kSiteAFull)) {
                    ok = false;
                    break;
                }
                if (transform && valid) {
                    const uint32_t row = sb + kOffA + st * kABytes + (uint32_t)r * 128u;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t a = row + ((uint32_t)(c ^ (r & 7)) << 4);
                        uint4 v;
                        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                                     : "r"(a));
                        const int c0 = kc * 64 + c * 8;
                        v = transform16(v, SIGE_BF16, affine ? p.gsc + (int64_t)n * p.Cin + c0 : nullptr,
                                        affine ? p.gsh + (int64_t)n * p.Cin + c0 : nullptr, p.silu);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y),
                                     "r"(v.z), "r"(v.w)
                                     : "memory");
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(a_full(st));
            }
            for (int kc = 0; !p.tma_a && ok && kc < kcn; ++kc) {
                // chunk kc first (its group is the oldest of the seven in
                // flight), then the refill of the stage the MMAs of chunk kc - 1
                // release: chunk kc never waits for an MMA
                cp_async_wait<kAStages - 2>();                     // chunk kc has landed (this thread's copies)
                const int st = (ia + kc) % kAStages;
                if (transform && valid) {
                    const uint32_t row = sb + kOffA + st * kABytes + (uint32_t)r * 128u;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const uint32_t a = row + ((uint32_t)(c ^ (r & 7)) << 4);
                        uint4 v;
                        asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                     : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                                     : "r"(a));
                        const int c0 = kc * 64 + c * 8;
                        v = transform16(v, SIGE_BF16, affine ? p.gsc + (int64_t)n * p.Cin + c0 : nullptr,
                                        affine ? p.gsh + (int64_t)n * p.Cin + c0 : nullptr, p.silu);
                        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y),
                                     "r"(v.z), "r"(v.w)
                                     : "memory");
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                mbar_arrive(a_full(st));
                const int j = kc + kAStages - 1;
                if (j < kcn && !issue(j)) {
                    ok = false;
                    break;
                }
                cp_async_commit();
            }
            cp_async_wait<0>();
            if (!__all_sync(0xFFFFFFFFu, ok))
                break;
            ia += kcn;
            // epilogue: 16 output channels at a time
            if (!mbar_wait_w(bar + kBarAccFull, k & 1, abort_flag, hdr, kSiteAccFull)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int co0 = nt * p.nt;
            uint8_t *dst = p.y + (pix * p.Cout + co0) * 2;
            const uint8_t *res = p.residual ? p.residual + (pix * p.Cout + co0) * 2 : nullptr;
            const float4 *bsm = reinterpret_cast<const float4 *>(smem + kOffBias + (warp & 3) * (kMaxNT * 4));
            for (int c0 = 0; c0 < p.nt; c0 += 16) {
                float v[16];
                ld16(t_row + (uint32_t)c0, v);
                if (!valid)
                    continue;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const float4 bq = bsm[c0 / 4 + q];
                    v[4 * q] += bq.x;
                    v[4 * q + 1] += bq.y;
                    v[4 * q + 2] += bq.z;
                    v[4 * q + 3] += bq.w;
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t o[4];
                    if (res) {
                        const uint4 rq = __ldg(reinterpret_cast<const uint4 *>(res + c0 * 2) + h);
                        const uint32_t rw[4] = {rq.x, rq.y, rq.z, rq.w};
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            o[t] = pack_bf16x2(v[8 * h + 2 * t] + bf16_lo(rw[t]), v[8 * h + 2 * t + 1] + bf16_hi(rw[t]));
                    } else {
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            o[t] = pack_bf16x2(v[8 * h + 2 * t], v[8 * h + 2 * t + 1]);
                    }
                    reinterpret_cast<uint4 *>(dst + c0 * 2)[h] = make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
            tc_fence_before();
            mbar_arrive(bar + kBarAccEmpty);
        }
        cp_async_wait<0>();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols));
    }
}

// ------------------------------------------------------------------ host

bool conv1x1_supported(const sige_conv_desc *cd, int dtype)
{
    return cd && dtype == SIGE_BF16 && cd->kernel == 1 && cd->stride == 1 && cd->pad == 0 && cd->block >= 1 &&
           cd->block * cd->block <= g1::kRows && cd->c_in >= 64 && cd->c_in % 64 == 0 && cd->c_out >= 16 &&
           cd->c_out % 16 == 0 && (cd->c_out <= g1::kMaxNT || cd->c_out % g1::kMaxNT == 0);
}

int launch_conv1x1(const ConvParams &cp, cudaStream_t stream)
{
    auto encode = get_encode();
    if (!encode)
        return SIGE_ERR_CUDA;
    g1::Args a{};
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
    a.Cin = cp.Cin;
    a.Cout = cp.Cout;
    a.b = cp.b;
    a.nt = std::min(cp.Cout, g1::kMaxNT);
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
    // weights [C_out][C_in] as a 2-d map: a box of 64 input channels x the
    // unit's output channels lands as 128-byte rows with the 128-byte swizzle
    CUtensorMap tw;
    cuuint64_t dims[2] = {(cuuint64_t)cp.Cin, (cuuint64_t)cp.Cout};
    cuuint64_t strides[1] = {(cuuint64_t)cp.Cin * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)a.nt};
    cuuint32_t es[2] = {1, 1};
    if (encode(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint8_t *>(cp.w), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return SIGE_ERR_UNSUPPORTED;
    // the input [N][H][W][C_in] as a 4-d map: a box of 64 channels x b x b
    // pixels of one item lands as the tile's b^2 rows of 128 bytes, 128-byte
    // swizzle, zero outside the map.  Used when b^2 rows fill whole 1 KB
    // swizzle atoms (b = 4 or 8), so that every box starts on an atom.
    CUtensorMap tx = tw;
    a.tma_a = 0;
    if ((cp.b * cp.b) % 8 == 0) {
        cuuint64_t xd[4] = {(cuuint64_t)cp.Cin, (cuuint64_t)cp.W, (cuuint64_t)cp.H, (cuuint64_t)cp.N};
        cuuint64_t xs[3] = {(cuuint64_t)cp.Cin * 2, (cuuint64_t)cp.W * cp.Cin * 2, (cuuint64_t)cp.H * cp.W * cp.Cin * 2};
        cuuint32_t xb[4] = {64, (cuuint32_t)cp.b, (cuuint32_t)cp.b, 1};
        cuuint32_t xe[4] = {1, 1, 1, 1};
        if (encode(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<uint8_t *>(cp.src), xd, xs, xb, xe,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            a.tma_a = 1;
        else
            tx = tw;
    }
    static std::atomic<int> attr_set[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return SIGE_ERR_CUDA;
    if (!attr_set[dev].load(std::memory_order_acquire)) {
        if (cudaFuncSetAttribute(k_conv1x1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)g1::kSmem) !=
            cudaSuccess)
            return SIGE_ERR_CUDA;
        prefer_max_shared(k_conv1x1);
        attr_set[dev].store(1, std::memory_order_release);
    }
    const int tpb = g1::kRows / (cp.b * cp.b);
    const int64_t pairs = (int64_t)(cp.dense ? cp.tiles_total : cp.cap) * cp.N;
    const int64_t units_max = (pairs + tpb - 1) / tpb * a.ntn;
    if (units_max > INT32_MAX)
        return SIGE_ERR_INVALID_ARG;
    const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(units_max, device_sm_count()));
    if (launch_pdl(k_conv1x1, dim3(grid), dim3(g1::kThreads), g1::kSmem, stream, a, tw, tx) != cudaSuccess)
        return SIGE_ERR_CUDA;
    count_launch();
    return launch_check();
}

} // namespace sige
