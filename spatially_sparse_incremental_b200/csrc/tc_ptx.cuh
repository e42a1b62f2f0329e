// PTX wrappers shared by the tensor-core kernels of libsige: shared-memory
// addresses, mbarriers (bounded waits), TMA tile loads, tcgen05 fences,
// commits, MMA issue blocks and tensor-memory loads, cluster helpers, and the
// shared-memory matrix / instruction descriptors of tcgen05 (kind::f16).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "sige_internal.cuh"

namespace sige {

constexpr long long kWaitCycles = 1ll << 31;   // bound of every mbarrier wait, ~1.1 s at 1.9 GHz

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

// Bounded wait: false when the limit expired or another role gave up.  The
// polling loop is out of line so that the callers' loops stay compact.
static __device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, volatile int *abort_flag, WsHeader *hdr,
                                            int where)
{
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

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag, WsHeader *hdr,
                                          int where)
{
    return mbar_try(bar, parity) || mbar_wait_slow(bar, parity, abort_flag, hdr, where);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap *map, uint32_t bar, int c0, int c1, int c2,
                                            int c3, int c4)
{
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
        : "memory");
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// Cluster helpers (cluster launches).
__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_peer(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_peer_f32(uint32_t addr, float v)
{
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ void st_peer_f32x4(uint32_t addr, float a, float b, float c, float d)
{
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

// Arrive on an mbarrier of the peer; orders this thread's (and, through a
// preceding CTA barrier, the CTA's) earlier writes before the arrival.
__device__ __forceinline__ void mbar_arrive_peer(uint32_t addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

// The same with an arrival count.
__device__ __forceinline__ void mbar_arrive_peer_n(uint32_t addr, uint32_t n)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0], %1;" ::"r"(addr), "r"(n) : "memory");
}

__device__ __forceinline__ bool mbar_try_cluster(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

static __device__ __noinline__ bool mbar_wait_cluster_slow(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                    WsHeader *hdr, int where)
{
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_cluster(bar, parity))
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

__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                  WsHeader *hdr, int where)
{
    return mbar_try_cluster(bar, parity) || mbar_wait_cluster_slow(bar, parity, abort_flag, hdr, where);
}

// Relaxed: what the peer must see (the mbarrier initialisation) is released by
// the initialising thread's fence.mbarrier_init before it arrives.
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Warp-wide forms.  The whole converged warp calls them with identical
// arguments and one lane, chosen by elect.sync, issues the instruction.  The
// issuing loops then stay warp-uniform (their exits depend only on votes), so
// the compiler keeps descriptors, coordinates and stage counters in uniform
// registers, which is what the tensor-core and TMA instructions read.
__device__ __forceinline__ void tc_commit_w(uint32_t bar)
{
    asm volatile(
        "{\n .reg .pred e;\n .reg .b32 l;\n elect.sync l|e, 0xffffffff;\n"
        " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n}\n" ::"r"(bar)
        : "memory");
}

// The four K=16 steps of one 64-channel k-chunk (A advances 32 bytes per step,
// B by b_step) and the commit of the chunk's stage, from one elected lane.
__device__ __forceinline__ void tc_mma4_commit_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint64_t b_step,
                                                 uint32_t idesc, uint32_t accumulate, uint32_t bar)
{
    asm volatile(
        "{\n .reg .pred p, e, t;\n .reg .b32 l;\n .reg .b64 a1, a2, a3, b1, b2, b3;\n"
        " elect.sync l|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.eq.b32 t, 0, 0;\n"
        " add.s64 a1, %1, 2;\n add.s64 a2, %1, 4;\n add.s64 a3, %1, 6;\n"
        " add.s64 b1, %2, %5;\n add.s64 b2, b1, %5;\n add.s64 b3, b2, %5;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %3, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %3, t;\n"
        " @e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%6];\n}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "l"(b_step), "r"(bar)
        : "memory");
}

// The four K=16 steps of one 64-channel k-chunk into one accumulator block,
// from one elected lane (no commit).
__device__ __forceinline__ void tc_mma4_w(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint64_t b_step,
                                          uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p, e, t;\n .reg .b32 l;\n .reg .b64 a1, a2, a3, b1, b2, b3;\n"
        " elect.sync l|e, 0xffffffff;\n setp.ne.b32 p, %4, 0;\n setp.eq.b32 t, 0, 0;\n"
        " add.s64 a1, %1, 2;\n add.s64 a2, %1, 4;\n add.s64 a3, %1, 6;\n"
        " add.s64 b1, %2, %5;\n add.s64 b2, b1, %5;\n add.s64 b3, b2, %5;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a1, b1, %3, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a2, b2, %3, t;\n"
        " @e tcgen05.mma.cta_group::1.kind::f16 [%0], a3, b3, %3, t;\n}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "l"(b_step)
        : "memory");
}

// expect_tx on `bar` and the 2-D tile load that completes it, from one lane
__device__ __forceinline__ void tma_load_2d_w(uint32_t dst, const CUtensorMap *map, uint32_t bar, uint32_t bytes, int x,
                                              int y)
{
    asm volatile(
        "{\n .reg .pred e;\n .reg .b32 l;\n elect.sync l|e, 0xffffffff;\n"
        " @e mbarrier.arrive.expect_tx.shared::cta.b64 _, [%2], %3;\n"
        " @e cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%4, %5}], [%2];\n}\n"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(bytes), "r"(x), "r"(y)
        : "memory");
}

// Bounded wait by every lane of a warp; the outcome is the same in all lanes.
__device__ __forceinline__ bool mbar_wait_w(uint32_t bar, uint32_t parity, volatile int *abort_flag, WsHeader *hdr,
                                            int where)
{
    return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort_flag, hdr, where));
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

// cuTensorMapEncodeTiled from the driver, looked up once (no libcuda link).
PFN_cuTensorMapEncodeTiled_v12000 get_encode();

} // namespace sige
