// Tensor-core form of the attention step with pruned queries
// (sige_attention_core): for every token under the active-tile list, per head,
// o = softmax(q K^T / sqrt(dh)) V over all keys, written at that token.  (The
// nubint.ai review of "Efficient Spatially Sparse Inference for Conditional
// GANs and Diffusion Models", "Proposed method": attention layers by pruning
// the query tokens of unedited regions; mer.dev notes on the same paper,
// abstract: attention for Stable Diffusion.)
//
// Work unit: 128 query slots of one (batch item, head).  Slot s of the list is
// pixel (s mod b^2) of tile s / b^2 (row-major inside the tile); slots of
// clipped pixels and past the list's end are padding rows, computed and not
// written.  The unit's keys are walked in chunks of 128:
//   * warp 0 loads the chunk's K and V head slices with one TMA each: 64
//     channels from the head's first x 128 keys, 128-byte rows with the
//     128-byte swizzle, which is the K-major operand K (keys x channels) of
//     the first MMA and the MN-major operand V (keys x channels) of the
//     second; keys past the end read as zero;
//   * warp 1 issues S = Q K^T (M 128 queries, N 128 keys, K = head width) into
//     tensor memory, then O += P V (M 128, N = value width, K 128 keys) with
//     P read from tensor memory;
//   * warps 2..5, one query row per thread, read S from tensor memory, keep the
//     running maximum and sum (fp32), store P = exp(S - max) as bf16 back into
//     tensor memory for the second MMA, and rescale the O row there when the
//     maximum has grown by more than a factor 2^8 (the sum and O share one
//     stale maximum otherwise, which the final division removes).
// S of chunk j + 1 is computed while chunk j's exponentials run: the softmax
// threads release S as soon as they have loaded it.  The TMA and MMA warps run
// converged and issue from one elected lane, so that descriptors and
// coordinates stay in uniform registers.
//
// Key splits: the CTAs of a cluster of 4 take 4 / s units at a time, s CTAs
// per unit, each over a contiguous share of the chunks; s is the largest power
// of two <= 4 with units * s <= the grid (the tile count is read on the
// device).  The s partial rows (O, max, sum) meet in distributed shared memory:
// CTA k of a unit owns the unit's rows k * 128 / s ..; every CTA pushes each
// of its rows to the owner, which sums them weighted by exp(max_i - max) and
// writes them.  No workspace, one launch.
#include "tc_ptx.cuh"

#include <algorithm>
#include <atomic>
#include <math.h>

namespace sige {
namespace attn {

constexpr int kThreads = 192;       // warp 0 TMA, warp 1 MMA, warps 2..5 softmax
constexpr int kRows = 128;          // query slots per unit (the MMAs' M)
constexpr int kKeys = 128;          // keys per chunk
constexpr int kMaxHead = 64;        // widest per-head q/k and v slice the kernel takes
constexpr int kCluster = 4;
constexpr int kStages = 4;          // K/V chunk ring

constexpr uint32_t kTile = kRows * 128;                  // 16 KB: Q, or one K or V stage (128-byte rows)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTile;
constexpr uint32_t kOffV = kOffK + kStages * kTile;
constexpr uint32_t kOStride = (kMaxHead + 4) * 4;        // a received fp32 O row, padded (bank spread)
constexpr uint32_t kOffO = kOffV + kStages * kTile;      // rows pushed here by the unit's splits
constexpr uint32_t kOffML = kOffO + kRows * kOStride;    // their (max, sum)
constexpr uint32_t kOffBar = kOffML + kRows * 8;
constexpr uint32_t kBarKvFull = 0;      // + 8 stage
constexpr uint32_t kBarKvEmpty = 32;    // + 8 stage
constexpr uint32_t kBarSFull = 64;
constexpr uint32_t kBarSFree = 72;
constexpr uint32_t kBarPFull = 80;      // + 8 buffer
constexpr uint32_t kBarPvDone = 96;
constexpr uint32_t kBarQFull = 104;
constexpr uint32_t kBarPeerO = 112;     // the 128 rows this CTA owns have been pushed
constexpr uint32_t kBarPeerRd = 120;    // every owner has merged what this CTA pushed
constexpr uint32_t kTmemSlot = 128;
constexpr uint32_t kAbort = 132;
constexpr uint32_t kSmem = kOffBar + 256 + 1024;         // + alignment slack
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kTmemP = 128;        // S: columns 0..127, P (bf16 pairs): two buffers of 64, O: 256..
constexpr uint32_t kTmemO = 256;

// wait sites (the detail of a recorded SIGE_ERR_TIMEOUT)
constexpr int kSiteKvEmpty = 201, kSiteKvFull = 202, kSiteSFree = 203, kSitePFull = 204, kSiteQFull = 205,
              kSiteSFull = 206, kSitePvDone = 207, kSitePeerO = 209, kSitePeerRd = 210;

static_assert(kSmem <= 227 * 1024, "shared memory");

struct Args {
    const __nv_bfloat16 *q;   // [N][H][W][D]
    __nv_bfloat16 *o;         // [N][H][W][Dv]
    const int32_t *idx;       // [cap][2] tile origins
    const int32_t *count;
    int32_t N, H, W, D, Dv, Lk, heads, dh, dvh, dhp, dvp, b, cap;
    float sc;                 // log2(e) / sqrt(dh): scores in base-2 exponent units
};

// The call's device-side error word (no workspace is passed to this call).
__device__ WsHeader g_hdr;

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Warp-wide forms: the converged warp calls them with identical arguments and
// one elected lane issues.
__device__ __forceinline__ void tma_kv_w(uint32_t dk, uint32_t dv, const CUtensorMap *mk, const CUtensorMap *mv,
                                         uint32_t bar, uint32_t bytes, int xk, int xv, int key, int n)
{
    asm volatile(
        "{\n .reg .pred e;\n .reg .b32 l;\n elect.sync l|e, 0xffffffff;\n"
        " @e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%4], %5;\n"
        " @e cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%2, {%6, %8, %9}], [%4];\n"
        " @e cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%1], [%3, {%7, %8, %9}], [%4];\n"
        "}\n" ::"r"(dk),
        "r"(dv), "l"(reinterpret_cast<uint64_t>(mk)), "l"(reinterpret_cast<uint64_t>(mv)), "r"(bar), "r"(bytes),
        "r"(xk), "r"(xv), "r"(key), "r"(n)
        : "memory");
}

// D (tensor memory) (+)= A (shared memory) B (shared memory)
__device__ __forceinline__ void mma_ss_w(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n .reg .pred p, e;\n .reg .b32 l;\n elect.sync l|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
                 " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
                 "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// D (tensor memory) (+)= A (tensor memory) B (shared memory)
__device__ __forceinline__ void mma_ts_w(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n .reg .pred p, e;\n .reg .b32 l;\n elect.sync l|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n"
                 " @e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
                 "r"(a), "l"(b), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// 32 columns of this warp's 32 tensor-memory lanes, no wait.
__device__ __forceinline__ void ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void st32(uint32_t taddr, const uint32_t *v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

__device__ __forceinline__ void st16(uint32_t taddr, const float (&v)[16])
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]), "f"(v[8]), "f"(v[9]),
        "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15])
        : "memory");
}

__device__ __forceinline__ void st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_peer_f32x2(uint32_t addr, float a, float b)
{
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}

__device__ __forceinline__ float2 lds_f2(uint32_t addr)
{
    float2 v;
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
    return v;
}

__device__ __forceinline__ float4 lds_f4(uint32_t addr)
{
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// Element offset of query slot `slot`'s pixel (n, y, x) in an [N][H][W][*]
// map with `ch` channels, or -1 for a padding slot.
__device__ __forceinline__ int64_t slot_pixel(const Args &p, int ntile, int slot, int n, int ch)
{
    const int bb = p.b * p.b;
    const int t = slot / bb;
    if (t >= ntile)
        return -1;
    const int w = slot - t * bb;
    const int2 org = __ldg(reinterpret_cast<const int2 *>(p.idx) + t);
    const int y = org.x + w / p.b, x = org.y + w % p.b;
    if (org.x < 0 || org.y < 0 || y >= p.H || x >= p.W)
        return -1;
    return (((int64_t)n * p.H + y) * p.W + x) * ch;
}

// 8 bf16 of o[8 g ..] * inv at dst
__device__ __forceinline__ void store8(__nv_bfloat16 *dst, const float *v, float inv)
{
    *reinterpret_cast<uint4 *>(dst) =
        make_uint4(pack_bf16x2(v[0] * inv, v[1] * inv), pack_bf16x2(v[2] * inv, v[3] * inv),
                   pack_bf16x2(v[4] * inv, v[5] * inv), pack_bf16x2(v[6] * inv, v[7] * inv));
}

} // namespace attn

using namespace attn;

__global__ void __launch_bounds__(attn::kThreads, 1)
    k_attn_tc(const __grid_constant__ attn::Args p, const __grid_constant__ CUtensorMap tk,
              const __grid_constant__ CUtensorMap tv)
{
    extern __shared__ __align__(1024) uint8_t attn_raw[];
    const uint32_t raw = smem_u32(attn_raw);
    const uint32_t sb = (raw + 1023u) & ~1023u;
    uint8_t *smem = attn_raw + (sb - raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t bar = sb + kOffBar;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffBar + kAbort);
    WsHeader *hdr = &g_hdr;

    // the launch's work: units = query blocks x batch x heads, keys split s ways
    const int ntile = max(0, min(__ldg(p.count), p.cap));
    const int qblocks = (ntile * p.b * p.b + kRows - 1) / kRows;
    const int units = qblocks * p.N * p.heads;
    const int nch = (p.Lk + kKeys - 1) / kKeys;
    int s = kCluster;
    while (s > 1 && ((int64_t)units * s > (int64_t)gridDim.x || s > nch))
        s >>= 1;
    const int per = kCluster / s;                      // units a cluster takes at a time
    const int cps = (nch + s - 1) / s;                 // chunks of one split
    const int rank = (int)cluster_rank();
    const int sub = rank / s, split = rank - sub * s;
    const int u_step = (int)(gridDim.x / kCluster) * per;
    const int u_first = (int)(blockIdx.x / kCluster) * per + sub;
    const int c_lo = split * cps;
    const int c_hi = min(nch, c_lo + cps);              // empty for a split past the last chunk
    const bool work = c_lo < c_hi;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(bar + kBarKvFull + 8u * i, 1);
            mbar_init(bar + kBarKvEmpty + 8u * i, 1);
        }
        mbar_init(bar + kBarSFull, 1);
        mbar_init(bar + kBarSFree, kRows);
        mbar_init(bar + kBarPFull, kRows);
        mbar_init(bar + kBarPFull + 8u, kRows);
        mbar_init(bar + kBarPvDone, 1);
        mbar_init(bar + kBarQFull, kRows);
        mbar_init(bar + kBarPeerO, kRows);                  // s senders x 128 / s rows
        mbar_init(bar + kBarPeerRd, (uint32_t)(kRows * s)); // s owners x 128 threads
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0 && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tk)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tv)) : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(bar + kTmemSlot),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    // the first unit's query row, fetched while the CTA sets up
    const int r = (warp & 3) * 32 + lane;   // softmax threads: query row = tensor-memory lane
    uint4 qrow[kMaxHead / 8];
    auto fetch_q = [&](int u) {
        const int qb = u % qblocks, rest = u / qblocks;
        const int head = rest % p.heads, n = rest / p.heads;
        const int64_t qo = slot_pixel(p, ntile, qb * kRows + r, n, p.D);
#pragma unroll
        for (int g = 0; g < kMaxHead / 8; ++g) {
            qrow[g] = make_uint4(0, 0, 0, 0);
            if (qo >= 0 && g < p.dh / 8)
                qrow[g] = ld_nc16(p.q + qo + head * p.dh + 8 * g);
        }
    };
    if (warp >= 2 && work && u_first < units)
        fetch_q(u_first);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem + kOffBar + kTmemSlot);
    // the peers' barriers are initialised before the first remote access:
    // every thread arrives here and waits before its first push (softmax) or
    // after its loop (TMA and MMA warps)
    cluster_arrive();
    bool joined = false;

    if (warp == 0) {
        // ---- K / V chunks by TMA, a four-stage ring
        int it = 0;
        bool ok = true;
        for (int u = u_first; ok && work && u < units; u += u_step) {
            const int rest = u / qblocks;
            const int head = rest % p.heads, n = rest / p.heads;
            for (int c = c_lo; c < c_hi; ++c, ++it) {
                const int st = it % kStages;
                if (it >= kStages && !mbar_wait_w(bar + kBarKvEmpty + 8u * st, ((it / kStages) & 1) ^ 1, abort_flag,
                                                  hdr, kSiteKvEmpty)) {
                    ok = false;
                    break;
                }
                tma_kv_w(sb + kOffK + st * kTile, sb + kOffV + st * kTile, &tk, &tv, bar + kBarKvFull + 8u * st,
                         2u * kTile, head * p.dh, head * p.dvh, c * kKeys, n);
            }
        }
    } else if (warp == 1) {
        // ---- the two MMAs per chunk
        const uint32_t id_s = idesc_bf16(kKeys);
        const uint32_t id_o = idesc_bf16(p.dvp) | (1u << 16);   // B (V) MN-major
        const int ks = p.dhp / 16;
        int it = 0, wu = 0;
        bool ok = true;
        // S = Q K_j^T into columns 0..127 once chunk j has landed and the
        // softmax threads have loaded S of chunk j - 1; K-major operands with
        // the 128-byte swizzle advance 32 bytes per 16-element step
        auto issue_s = [&](int j) -> bool {
            const int st = j % kStages;
            if (!mbar_wait_w(bar + kBarKvFull + 8u * st, (j / kStages) & 1, abort_flag, hdr, kSiteKvFull))
                return false;
            if (j > 0 && !mbar_wait_w(bar + kBarSFree, (j - 1) & 1, abort_flag, hdr, kSiteSFree))
                return false;
            tc_fence_after();
            const uint64_t qd = desc_sw128(sb + kOffQ), kd = desc_sw128(sb + kOffK + st * kTile);
            for (int kk = 0; kk < ks; ++kk)
                mma_ss_w(tmem, qd + 2u * kk, kd + 2u * kk, id_s, kk > 0);
            tc_commit_w(bar + kBarSFull);
            return true;
        };
        for (int u = u_first; ok && work && u < units; u += u_step, ++wu) {
            if (!mbar_wait_w(bar + kBarQFull, wu & 1, abort_flag, hdr, kSiteQFull) || !issue_s(it))
                break;
            for (int c = c_lo; c < c_hi; ++c, ++it) {
                if (c + 1 < c_hi && !issue_s(it + 1)) {
                    ok = false;
                    break;
                }
                const int pb = it & 1;
                if (!mbar_wait_w(bar + kBarPFull + 8u * pb, (it >> 1) & 1, abort_flag, hdr, kSitePFull)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // O += P V: 16 keys per step; P from tensor memory (8 columns
                // of bf16 pairs per step), V MN-major with the 128-byte
                // swizzle (two 8-key atoms of 1 KB per step)
                const int st = it % kStages;
                for (int kk = 0; kk < kKeys / 16; ++kk)
                    mma_ts_w(tmem + kTmemO, tmem + kTmemP + 64u * pb + 8u * kk,
                             desc_sw128(sb + kOffV + st * kTile + kk * 2048),
                             id_o, (c > c_lo) || kk > 0);
                tc_commit_w(bar + kBarPvDone);
                tc_commit_w(bar + kBarKvEmpty + 8u * st);
            }
        }
    } else {
        // ---- softmax: thread = query row r, tensor-memory lane r
        const uint32_t t_row = tmem + ((uint32_t)((warp & 3) * 32) << 16);
        const int base = sub * s;
        const int rows = kRows / s;   // rows a CTA of the unit owns in the merge
        int it = 0, nmerge = 0;
        bool ok = true, have_q = true;
        for (int u = u_first; ok && u < units; u += u_step) {
            const int qb = u % qblocks, rest = u / qblocks;
            const int head = rest % p.heads, n = rest / p.heads;
            float m_used = -INFINITY, l = 0.0f;
            float o[kMaxHead];   // written after the chunk loop only
            if (work) {
                // this row's query: one 128-byte row, 16-byte chunk g at
                // g ^ (r mod 8); the previous unit's S products have completed
                if (!have_q)
                    fetch_q(u);
                have_q = false;
#pragma unroll
                for (int g = 0; g < kMaxHead / 8; ++g)
                    sts128(sb + kOffQ + r * 128 + ((g ^ (r & 7)) << 4), qrow[g]);
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                tc_fence_before();
                mbar_arrive(bar + kBarQFull);
                for (int c = c_lo; c < c_hi; ++c, ++it) {
                    if (!mbar_wait_w(bar + kBarSFull, it & 1, abort_flag, hdr, kSiteSFull)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint32_t sr[4][32];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4)
                        ld32(t_row + 32u * q4, sr[q4]);
                    ld_wait();
                    tc_fence_before();
                    mbar_arrive(bar + kBarSFree);   // the next chunk's S may overwrite these columns
                    const int kvalid = min(kKeys, p.Lk - c * kKeys);
                    float sv[kKeys];
#pragma unroll
                    for (int k = 0; k < kKeys; ++k)
                        sv[k] = __uint_as_float(sr[k >> 5][k & 31]);
                    if (kvalid < kKeys) {
#pragma unroll
                        for (int k = 0; k < kKeys; ++k)
                            if (k >= kvalid)
                                sv[k] = -INFINITY;
                    }
                    float mx[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        mx[i] = sv[i];
#pragma unroll
                    for (int k = 8; k < kKeys; ++k)
                        mx[k & 7] = fmaxf(mx[k & 7], sv[k]);
                    const float t_max =
                        fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                        p.sc;
                    // the exponent base moves only when the maximum has grown by
                    // more than 8 (P <= 2^8 otherwise)
                    const bool grow = t_max > m_used + 8.0f;
                    const float m_new = grow ? t_max : m_used;
                    const float corr = ex2(m_used - m_new);   // 0 on the unit's first chunk, 1 when kept
                    const float nm = -m_new;
                    float ls[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        ls[i] = 0.0f;
                    // P of this chunk into buffer it mod 2 (its last reader, P V
                    // two chunks back, completed before this chunk's S), 64 keys
                    // at a time
                    const uint32_t t_p = t_row + kTmemP + 64u * (uint32_t)(it & 1);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        uint32_t pk[32];
#pragma unroll
                        for (int k = 0; k < 64; k += 2) {
                            const float p0 = ex2(fmaf(sv[64 * h + k], p.sc, nm));
                            const float p1 = ex2(fmaf(sv[64 * h + k + 1], p.sc, nm));
                            ls[(k >> 1) & 7] += p0 + p1;
                            pk[k >> 1] = pack_bf16x2(p0, p1);
                        }
                        st32(t_p + 32u * h, pk);
                    }
                    l = l * corr + (((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7])));
                    if (c > c_lo && __any_sync(0xFFFFFFFFu, grow)) {
                        // rescale this warp's O rows once the previous chunk's P V has landed
                        if (!mbar_wait_w(bar + kBarPvDone, (it - 1) & 1, abort_flag, hdr, kSitePvDone)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int pc = 0; pc < kMaxHead / 16; ++pc) {
                            if (pc * 16 < p.dvp) {
                                float v[16];
                                tmem_ld16(t_row + kTmemO + 16u * pc, v);
#pragma unroll
                                for (int i = 0; i < 16; ++i)
                                    v[i] *= corr;
                                st16(t_row + kTmemO + 16u * pc, v);
                            }
                        }
                    }
                    st_wait();
                    tc_fence_before();
                    mbar_arrive(bar + kBarPFull + 8u * (uint32_t)(it & 1));
                    m_used = m_new;
                }
                if (!ok)
                    break;
                // the unit's O row, once its last P V has landed
                if (!mbar_wait_w(bar + kBarPvDone, (it - 1) & 1, abort_flag, hdr, kSitePvDone)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int pc = 0; pc < kMaxHead / 16; ++pc) {
                    float v[16];
                    if (pc * 16 < p.dvp)
                        tmem_ld16(t_row + kTmemO + 16u * pc, v);
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        o[pc * 16 + i] = pc * 16 < p.dvp ? v[i] : 0.0f;
                }
                tc_fence_before();
            } else {
#pragma unroll
                for (int i = 0; i < kMaxHead; ++i)
                    o[i] = 0.0f;   // an empty split: weight 0 in the merge
            }
            if (s == 1) {
                const int64_t oo = slot_pixel(p, ntile, qb * kRows + r, n, p.Dv);
                if (oo >= 0) {
                    const float inv = 1.0f / l;
#pragma unroll
                    for (int g = 0; g < kMaxHead / 8; ++g)
                        if (g < p.dvh / 8)
                            store8(p.o + oo + head * p.dvh + 8 * g, o + 8 * g, inv);
                }
                continue;
            }
            // ---- merge of the unit's s splits: push this row to its owner
            if (!joined) {
                cluster_wait();
                joined = true;
            }
            // (the owner has merged the previous unit's rows)
            if (nmerge > 0 &&
                !__all_sync(0xFFFFFFFFu, mbar_wait_cluster(bar + kBarPeerRd, (nmerge - 1) & 1, abort_flag, hdr, kSitePeerRd))) {
                ok = false;
                break;
            }
            {
                const int owner = r / rows;
                const uint32_t slot = (uint32_t)(split * rows + (r - owner * rows));
                const uint32_t dst = map_peer(sb + kOffO + slot * kOStride, (uint32_t)(base + owner));
#pragma unroll
                for (int g = 0; g < kMaxHead / 8; ++g)
                    if (g < p.dvh / 8) {
                        st_peer_f32x4(dst + 32u * g, o[8 * g], o[8 * g + 1], o[8 * g + 2], o[8 * g + 3]);
                        st_peer_f32x4(dst + 32u * g + 16u, o[8 * g + 4], o[8 * g + 5], o[8 * g + 6], o[8 * g + 7]);
                    }
                st_peer_f32x2(map_peer(sb + kOffML + slot * 8u, (uint32_t)(base + owner)), m_used, l);
                mbar_arrive_peer(map_peer(bar + kBarPeerO, (uint32_t)(base + owner)));   // releases the pushes
            }
            if (!__all_sync(0xFFFFFFFFu, mbar_wait_cluster(bar + kBarPeerO, nmerge & 1, abort_flag, hdr, kSitePeerO))) {
                ok = false;
                break;
            }
            {
                // this CTA's rows split * rows .. of the unit: the s pushed
                // copies weighted by exp(max_i - max)
                const int ng = p.dvh / 8;
                for (int item = r; item < rows * ng; item += kRows) {
                    const int j = item / ng, g = item - j * ng;
                    float mi[kCluster], li[kCluster], mmax = -INFINITY;
#pragma unroll
                    for (int i = 0; i < kCluster; ++i) {
                        mi[i] = -INFINITY;
                        li[i] = 0.0f;
                        if (i < s) {
                            const float2 ml = lds_f2(sb + kOffML + (uint32_t)(i * rows + j) * 8u);
                            mi[i] = ml.x;
                            li[i] = ml.y;
                            mmax = fmaxf(mmax, ml.x);
                        }
                    }
                    float L = 0.0f, acc[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        acc[e] = 0.0f;
#pragma unroll
                    for (int i = 0; i < kCluster; ++i) {
                        if (i < s) {
                            const float w = ex2(mi[i] - mmax);   // 0 for an empty split
                            L = fmaf(li[i], w, L);
                            const uint32_t a = sb + kOffO + (uint32_t)(i * rows + j) * kOStride + 32u * g;
                            const float4 x0 = lds_f4(a), x1 = lds_f4(a + 16);
                            acc[0] = fmaf(w, x0.x, acc[0]);
                            acc[1] = fmaf(w, x0.y, acc[1]);
                            acc[2] = fmaf(w, x0.z, acc[2]);
                            acc[3] = fmaf(w, x0.w, acc[3]);
                            acc[4] = fmaf(w, x1.x, acc[4]);
                            acc[5] = fmaf(w, x1.y, acc[5]);
                            acc[6] = fmaf(w, x1.z, acc[6]);
                            acc[7] = fmaf(w, x1.w, acc[7]);
                        }
                    }
                    const int64_t oo = slot_pixel(p, ntile, qb * kRows + split * rows + j, n, p.Dv);
                    if (oo >= 0)
                        store8(p.o + oo + head * p.dvh + 8 * g, acc, 1.0f / L);
                }
            }
            // every sender may refill this CTA's rows (after its own wait)
            for (int i = 0; i < s; ++i)
                mbar_arrive_peer(map_peer(bar + kBarPeerRd, (uint32_t)(base + i)));
            ++nmerge;
        }
        // the owners' last "merged" arrivals have reached this CTA before it leaves
        if (ok && nmerge > 0)
            __all_sync(0xFFFFFFFFu, mbar_wait_cluster(bar + kBarPeerRd, (nmerge - 1) & 1, abort_flag, hdr, kSitePeerRd));
    }
    if (!joined)
        cluster_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
    }
    // no CTA leaves while a peer may still address its shared memory
    cluster_arrive();
    cluster_wait();
}

// ------------------------------------------------------------------ host

// K or V [N][Lk][C] as a 3-d map: a box of 64 channels (from the head's
// first) x 128 keys lands as 128-byte rows with the 128-byte swizzle, one
// contiguous read per key; zero past the last key and past channel C.  The
// channels past the head width belong to the next head: they meet zero query
// columns in S = Q K^T and give output columns that are not written in P V.
static bool encode_kv(CUtensorMap *map, const void *base, int N, int Lk, int C, PFN_cuTensorMapEncodeTiled_v12000 encode)
{
    cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)Lk, (cuuint64_t)N};
    cuuint64_t strides[2] = {(cuuint64_t)C * 2, (cuuint64_t)Lk * C * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)attn::kKeys, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool al16(const void *ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

bool attention_tc_scope(int dh, int dvh)
{
    return dh > 0 && dvh > 0 && dh % 8 == 0 && dvh % 8 == 0 && dh <= attn::kMaxHead && dvh <= attn::kMaxHead;
}

// The tensor-core attention step, or 1 when the call is outside its scope
// (head widths not multiples of 8 or above 64, unaligned buffers): the caller
// then runs the CUDA-core kernel.
int attention_core_tc(const void *q, const void *k, const void *v, void *o, const int32_t *idx, const int32_t *count,
                      int N, int H, int W, int D, int Dv, int Lk, int heads, int b, int cap, cudaStream_t stream)
{
    const int dh = D / heads, dvh = Dv / heads;
    if (!attention_tc_scope(dh, dvh))
        return 1;
    if (!al16(q) || !al16(k) || !al16(v) || !al16(o))
        return 1;
    const int64_t slots = (int64_t)cap * b * b;
    if (slots + attn::kRows > INT32_MAX / 2 || (slots + attn::kRows) / attn::kRows * N * heads > INT32_MAX / 16)
        return 1;
    const PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode();
    if (!encode)
        return 1;
    CUtensorMap tk, tv;
    if (!encode_kv(&tk, k, N, Lk, D, encode) || !encode_kv(&tv, v, N, Lk, Dv, encode))
        return 1;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
        return SIGE_ERR_CUDA;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = attn::kCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg{};
    cfg.blockDim = dim3(attn::kThreads);
    cfg.dynamicSmemBytes = attn::kSmem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static std::atomic<int> clusters_of[64];   // co-resident clusters, per device
    int ncl = clusters_of[dev].load(std::memory_order_acquire);
    if (ncl == 0) {
        if (cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)attn::kSmem) !=
            cudaSuccess) {
            cudaGetLastError();
            return 1;
        }
        cfg.gridDim = dim3(attn::kCluster * (device_sm_count() / attn::kCluster));
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, k_attn_tc, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();
            return 1;
        }
        ncl = n;
        clusters_of[dev].store(n, std::memory_order_release);
    }
    // every unit a launch can have needs at most one cluster
    const int64_t units_max = (slots + attn::kRows - 1) / attn::kRows * N * heads;
    cfg.gridDim = dim3((unsigned)(attn::kCluster * std::max<int64_t>(1, std::min<int64_t>(ncl, units_max))));
    attn::Args a{};
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.o = static_cast<__nv_bfloat16 *>(o);
    a.idx = idx;
    a.count = count;
    a.N = N; a.H = H; a.W = W; a.D = D; a.Dv = Dv; a.Lk = Lk; a.heads = heads;
    a.dh = dh; a.dvh = dvh; a.dhp = (dh + 15) / 16 * 16; a.dvp = (dvh + 15) / 16 * 16; a.b = b; a.cap = cap;
    a.sc = (float)(1.4426950408889634 / std::sqrt((double)dh));
    if (cudaLaunchKernelEx(&cfg, k_attn_tc, a, tk, tv) != cudaSuccess)
        return SIGE_ERR_CUDA;
    count_launch();
    return launch_check();
}

} // namespace sige
