// Internal definitions shared by the CUDA sources of libsige.
#pragma once

#include <atomic>
#include <utility>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "sige.h"

namespace sige {

constexpr int kNumSMs = 148;            // B200
constexpr int kMaxScales = SIGE_MAX_SCALES;
constexpr size_t kWsHeader = SIGE_WORKSPACE_HEADER_BYTES;

// Workspace header (first 256 bytes of every workspace).
struct WsHeader {
    int32_t error;        // first device error (a sige_status), 0 = none
    int32_t detail;       // call-specific detail of that error
    uint32_t arrive;      // "last CTA" arrival counter (self-resetting)
    uint32_t next;        // work counter of the mask's difference stream (self-resetting)
    uint32_t pad[60];
};
static_assert(sizeof(WsHeader) == kWsHeader, "header size");

__device__ __forceinline__ void record_error(WsHeader *h, int32_t code, int32_t detail)
{
    if (atomicCAS(&h->error, 0, code) == 0)
        atomicExch(&h->detail, detail);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Two floats -> packed bf16x2 (round to nearest even), low half = a.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&v);
}

// SiLU v * sigmoid(v) = v / (1 + e^-v); __fdividef returns 0 once the
// denominator overflows, which is the limit of SiLU for v -> -inf.
__device__ __forceinline__ float silu_f(float v) { return __fdividef(v, 1.0f + __expf(-v)); }

// 16-byte loads/stores.
__device__ __forceinline__ uint4 ld_stream16(const void *p)
{
    uint4 r;
    asm volatile("ld.global.cs.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}
__device__ __forceinline__ uint4 ld_nc16(const void *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

// Host-side helpers (sige_api.cu)
int launch_check();           // SIGE_OK or SIGE_ERR_CUDA after a launch
// Every kernel of the library asks for the largest shared-memory carveout, the
// configuration the tensor-core conv needs: consecutive launches then run
// without reconfiguring the SM's L1 / shared-memory split in between.
template <typename K>
inline void prefer_max_shared(K kernel)
{
    static std::atomic<int> done[64];   // per device; concurrent first calls both set the same attribute
    int d = 0;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64 || done[d].load(std::memory_order_acquire))
        return;
    cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
    cudaGetLastError();   // a refused preference is not an error of the call
    done[d].store(1, std::memory_order_release);
}
void count_launch();
int device_sm_count();
// Bound of the device-side waits that sige_set_wait_cycles() may shorten, for
// launches enqueued from now on: the value set there, or `dflt` when none is.
long long wait_cycles_or(long long dflt);
// The tensor-core attention step (attention_tc.cu): a sige_status, or 1 when
// the call is outside that kernel's scope and the CUDA-core kernel runs it.
int attention_core_tc(const void *q, const void *k, const void *v, void *o, const int32_t *idx, const int32_t *count,
                      int N, int H, int W, int D, int Dv, int Lk, int heads, int b, int cap, cudaStream_t stream);
// Head widths that kernel takes (with 16-byte aligned buffers).
bool attention_tc_scope(int dh, int dvh);

// Programmatic dependent launch.  A kernel launched this way may start while
// the kernel before it in the stream is still running: its CTAs take SMs as
// that kernel's CTAs leave.  It must call pdl_wait() before it touches any
// memory the previous kernel may write (pdl_wait returns once that kernel has
// completed and its writes are visible), and it calls pdl_trigger() to let the
// kernel after it start early in the same way.  Both are no-ops for a kernel
// launched without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... P, typename... A>
inline cudaError_t launch_pdl(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              A &&...args)
{
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<A>(args)...);
}

// Division of 32-bit values by a divisor fixed for a launch (or a unit): a
// multiply-high and two shifts (Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994, the unsigned case).  Exact
// for every n < 2^32 and 1 <= d <= 2^31.  A runtime division in a per-element
// loop costs tens of instructions; this costs four.
struct UDiv {
    uint32_t m, s1, s2;
};

__host__ __device__ inline UDiv udiv_make(uint32_t d)
{
    uint32_t l = 0;                                  // ceil(log2 d)
    while (l < 32 && (1ull << l) < d)
        ++l;
    const uint64_t m = ((((uint64_t)1 << l) - d) << 32) / d + 1;
    return UDiv{(uint32_t)m, l < 1 ? l : 1u, l > 1 ? l - 1 : 0u};
}

__device__ __forceinline__ uint32_t udiv(uint32_t n, UDiv f)
{
    const uint32_t t = __umulhi(n, f.m);
    return (t + ((n - t) >> f.s1)) >> f.s2;
}

} // namespace sige
