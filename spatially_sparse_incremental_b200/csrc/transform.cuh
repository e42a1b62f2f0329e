// Per-element input transform (GroupNorm affine + SiLU) and output epilogue
// (bias + residual, one rounding), shared by the gather, scatter and conv
// kernels so that the fused and the unfused paths round identically.
#pragma once

#include "sige_internal.cuh"

namespace sige {

// v -> v*scale + shift (when scale != nullptr) -> SiLU (when silu), in float.
__device__ __forceinline__ float transform1(float v, const float *sc, const float *sh, int k, int silu)
{
    if (sc)
        v = __fmaf_rn(v, __ldg(sc + k), __ldg(sh + k));
    if (silu)
        v = silu_f(v);
    return v;
}

// 16 bytes of a pixel's channels (8 bf16 or 4 f32) through the transform,
// stored back in the same dtype.  sc/sh point at the first channel.
__device__ __forceinline__ uint4 transform16(uint4 in, int dtype, const float *sc, const float *sh, int silu)
{
    if (!sc && !silu)
        return in;
    uint4 out;
    uint32_t *o = reinterpret_cast<uint32_t *>(&out);
    const uint32_t *w = reinterpret_cast<const uint32_t *>(&in);
    if (dtype == SIGE_BF16) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float a = transform1(bf16_lo(w[q]), sc, sh, 2 * q, silu);
            float b = transform1(bf16_hi(w[q]), sc, sh, 2 * q + 1, silu);
            o[q] = pack_bf16x2(a, b);
        }
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o[q] = __float_as_uint(transform1(__uint_as_float(w[q]), sc, sh, q, silu));
    }
    return out;
}

// transform16 for 8 bf16 channels whose affine parameters are in registers.
__device__ __forceinline__ uint4 transform16_bf16_reg(uint4 in, const float (&sc)[8], const float (&sh)[8],
                                                      bool affine, int silu)
{
    uint4 out;
    uint32_t *o = reinterpret_cast<uint32_t *>(&out);
    const uint32_t *w = reinterpret_cast<const uint32_t *>(&in);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float a = bf16_lo(w[q]), b = bf16_hi(w[q]);
        if (affine) {
            a = __fmaf_rn(a, sc[2 * q], sh[2 * q]);
            b = __fmaf_rn(b, sc[2 * q + 1], sh[2 * q + 1]);
        }
        if (silu) {
            a = silu_f(a);
            b = silu_f(b);
        }
        o[q] = pack_bf16x2(a, b);
    }
    return out;
}

// The GauGAN-style input transform of 8 bf16 channels of one pixel: the
// GroupNorm-style affine (when sc), the per-pixel modulation t * (1 + g) + b
// with g, b the same 8 channels of the modulation maps at that pixel (when
// mod), then SiLU or LeakyReLU(0.2); one rounding to bf16.
__device__ __forceinline__ uint4 transform16_mod(uint4 in, const float *sc, const float *sh, bool mod, uint4 g,
                                                 uint4 b, int silu, int leaky)
{
    uint4 out;
    uint32_t *o = reinterpret_cast<uint32_t *>(&out);
    const uint32_t *w = reinterpret_cast<const uint32_t *>(&in);
    const uint32_t *gw = reinterpret_cast<const uint32_t *>(&g);
    const uint32_t *bw = reinterpret_cast<const uint32_t *>(&b);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        float v[2] = {bf16_lo(w[q]), bf16_hi(w[q])};
        const float gg[2] = {bf16_lo(gw[q]), bf16_hi(gw[q])};
        const float bb[2] = {bf16_lo(bw[q]), bf16_hi(bw[q])};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            if (sc)
                v[e] = __fmaf_rn(v[e], __ldg(sc + 2 * q + e), __ldg(sh + 2 * q + e));
            if (mod)
                v[e] = __fmaf_rn(v[e], 1.0f + gg[e], bb[e]);
            if (silu)
                v[e] = silu_f(v[e]);
            else if (leaky)
                v[e] = v[e] >= 0.0f ? v[e] : 0.2f * v[e];
        }
        o[q] = pack_bf16x2(v[0], v[1]);
    }
    return out;
}

__device__ __forceinline__ float load_elem(const uint8_t *base, int64_t e, int dtype)
{
    if (dtype == SIGE_BF16)
        return __uint_as_float((uint32_t)(reinterpret_cast<const uint16_t *>(base)[e]) << 16);
    return reinterpret_cast<const float *>(base)[e];
}

// y[e .. e+3] = round(a + bias[0..3] + residual[e .. e+3]) in y's dtype.
__device__ __forceinline__ void store_out4(uint8_t *y, int64_t e, int dtype, float4 a, const float *bias,
                                           const uint8_t *residual)
{
    if (bias) {
        const float4 b = __ldg(reinterpret_cast<const float4 *>(bias));
        a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
    }
    if (dtype == SIGE_BF16) {
        if (residual) {
            const uint2 r = __ldg(reinterpret_cast<const uint2 *>(residual + e * 2));
            a.x += bf16_lo(r.x); a.y += bf16_hi(r.x); a.z += bf16_lo(r.y); a.w += bf16_hi(r.y);
        }
        *reinterpret_cast<uint2 *>(y + e * 2) = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
    } else {
        if (residual) {
            const float4 r = __ldg(reinterpret_cast<const float4 *>(residual + e * 4));
            a.x += r.x; a.y += r.y; a.z += r.z; a.w += r.w;
        }
        *reinterpret_cast<float4 *>(y + e * 4) = a;
    }
}

// Single-element form of store_out4.
__device__ __forceinline__ void store_out1(uint8_t *y, int64_t e, int dtype, float a, float bias,
                                           const uint8_t *residual)
{
    a += bias;
    if (residual)
        a += load_elem(residual, e, dtype);
    if (dtype == SIGE_BF16)
        reinterpret_cast<__nv_bfloat16 *>(y)[e] = __float2bfloat16_rn(a);
    else
        reinterpret_cast<float *>(y)[e] = a;
}

} // namespace sige
