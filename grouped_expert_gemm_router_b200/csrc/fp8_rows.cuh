// The per-vector e4m3 quantization shared by the row quantizer and the
// kernels that quantize rows on the way to another GPU (one definition, so
// their codes and scales are the same bits): a power-of-two scale per
// vector, s = 2^(c - 8) with c the smallest integer such that
// max|v| <= 2^c (s = 1 for an all-zero vector), codes = nearest e4m3 value of
// v / s, ties to even.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace moe {
namespace {

// The power-of-two scale of a vector of largest magnitude amax, s = 2^(c - 8),
// and the factor that divides by it: v / s = (v * p0) * p1 exactly, p0 * p1 =
// 2^(8 - c) split in two so that neither factor overflows (c can be as low as
// -133 for bf16 subnormals).  A product by a power of two is exact, or rounds
// once to nearest like the division would, so the codes equal those of v / s.
struct Fp8Scale {
    float s, p0, p1;
};
__device__ __forceinline__ Fp8Scale fp8_scale(float amax) {
    if (!(amax > 0.0f) || isinf(amax)) return {1.0f, 1.0f, 1.0f};
    int ex;
    const float m = frexpf(amax, &ex);  // amax = m * 2^ex, 0.5 <= m < 1
    const int c = (m == 0.5f) ? ex - 1 : ex;
    const int e = 8 - c;                // in [-119, 141]
    const int e0 = e > 64 ? 64 : e;
    return {ldexpf(1.0f, c - 8), ldexpf(1.0f, e0), ldexpf(1.0f, e - e0)};
}

// Two values / s to two e4m3 codes (low byte = first).  ONE: 1/s = p0 is a
// normal power of two (p1 == 1), one product per value (the common case).
template <bool ONE>
__device__ __forceinline__ uint32_t e4m3x2(float a, float b, const Fp8Scale &sc) {
    const float2 v = ONE ? make_float2(__fmul_rn(a, sc.p0), __fmul_rn(b, sc.p0))
                         : make_float2(__fmul_rn(__fmul_rn(a, sc.p0), sc.p1), __fmul_rn(__fmul_rn(b, sc.p0), sc.p1));
    return (uint32_t)__nv_cvt_float2_to_fp8x2(v, __NV_SATFINITE, __NV_E4M3);
}

// Eight bf16 values (one 16-byte vector) / s to eight codes.
template <bool ONE>
__device__ __forceinline__ uint2 quant8_t(const uint4 &v, const Fp8Scale &sc) {
    const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&v);
    uint32_t c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(b[i]);
        c[i] = e4m3x2<ONE>(f.x, f.y, sc);
    }
    return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}
__device__ __forceinline__ uint2 quant8(const uint4 &v, const Fp8Scale &sc) {
    return sc.p1 == 1.0f ? quant8_t<true>(v, sc) : quant8_t<false>(v, sc);
}

// Largest magnitude of eight bf16 values folded into m (packed bf16 max of
// the magnitudes: exact, NaN ignored as fmaxf ignores it).
__device__ __forceinline__ __nv_bfloat162 amax8(const uint4 &v, __nv_bfloat162 m) {
    const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) m = __hmax2(m, __habs2(b[i]));
    return m;
}
__device__ __forceinline__ float amax_of(__nv_bfloat162 m) {
    return fmaxf(__bfloat162float(m.x), __bfloat162float(m.y));
}

}  // namespace
}  // namespace moe
