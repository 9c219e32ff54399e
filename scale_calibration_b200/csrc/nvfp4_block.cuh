// One NVFP4 block (16 weights) quantised with its chosen scale: the fake-quantised
// values fp32(q * s), q = E2M1_RNE_sat(fp32(w / s)), and the packed 4-bit codes.
// Used by the fake-quant and packed-export kernel (internal header).
//
// "NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4 逐块权重缩放
// 算法实战指南" (xxmr.cn/news/266017), section "算法原理": Q(W, s) = Cast(W/s) * s.
#pragma once

#include <cuda_fp16.h>

#include "common.cuh"
#include "quant.cuh"

namespace lh {

template <typename T>
struct Vec16;

template <>
struct Vec16<uint16_t> {
    __device__ static void load(const uint16_t* p, float (&w)[16]) {
        const uint4* q = reinterpret_cast<const uint4*>(p);
        const uint4 a = __ldg(q), b = __ldg(q + 1);
        const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            w[2 * i] = __uint_as_float(v[i] << 16);
            w[2 * i + 1] = __uint_as_float(v[i] & 0xFFFF0000u);
        }
    }
    __device__ static void store(uint16_t* p, const float (&o)[16]) {
        uint32_t v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(o[2 * i], o[2 * i + 1]);  // RNE
            v[i] = *reinterpret_cast<const uint32_t*>(&h);
        }
        uint4* q = reinterpret_cast<uint4*>(p);
        q[0] = make_uint4(v[0], v[1], v[2], v[3]);
        q[1] = make_uint4(v[4], v[5], v[6], v[7]);
    }
};

template <>
struct Vec16<float> {
    __device__ static void load(const float* p, float (&w)[16]) {
        const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 t = __ldg(q + i);
            w[4 * i] = t.x; w[4 * i + 1] = t.y; w[4 * i + 2] = t.z; w[4 * i + 3] = t.w;
        }
    }
    __device__ static void store(float* p, const float (&o)[16]) {
        float4* q = reinterpret_cast<float4*>(p);
#pragma unroll
        for (int i = 0; i < 4; ++i) q[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
    }
};

// Two 4-bit OCP E2M1 codes at once (sign bit, 2 exponent bits with bias 1,
// 1 mantissa bit): round to nearest even with saturation at +-6, the hardware
// conversion (its first operand goes to the high nibble); and their exact
// values back.
__device__ __forceinline__ uint32_t e2m1x2_codes(float lo, float hi) {
    uint16_t r;
    asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.u16.u8 %0, t;\n}" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
__device__ __forceinline__ float2 e2m1x2_values(uint32_t codes) {
    uint32_t h2;
    asm("{\n .reg .b8 t;\n cvt.u8.u32 t, %1;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}" : "=r"(h2) : "r"(codes));
    const __half2 h = *reinterpret_cast<const __half2*>(&h2);
    return __half22float2(h);  // .x from the low nibble
}

// fp32(w / s) for the 16 weights, then the E2M1 codes and values. The quotient is
// formed from one correctly rounded reciprocal y = RN(1/s): q = RN(w y), r = w - s q
// (exact, one FMA), RN(q + r y) is the correctly rounded quotient (P. Markstein,
// IBM J. Res. Dev. 34(1), 1990) while s is normal and |w| >= 2^-100. With s in
// [2^-95, FLT_MAX] a weight below 2^-100 has |w / s| < 2^-5: the approximate quotient
// stays below 2^-4 as well, and both round to a zero of w's sign in E2M1, so one test
// of s per block covers every weight. Other blocks divide; s == 0 gives q = +-0 with
// the sign of w.
//
// The steps run on pairs (f32x2) with -y in place of y: a = RN(w (-y)) = -q,
// r = RN(a s + w), v = RN(r (-y) + a) = -RN(q + r y), so v is the negated quotient
// with the right sign even for w = +-0 (an FMA with a = -q keeps the zero's sign
// that q + r y would lose). Its E2M1 codes get their sign bits flipped, and their
// values are multiplied by -s.
template <bool kOut, bool kPack>
__device__ __forceinline__ void quantize_block(const float (&w)[16], float s, float (&o)[16], uint32_t (&word)[2]) {
    word[0] = word[1] = 0u;
    if (s >= 2.524355e-29f && s <= 3.4028235e38f) {  // 2^-95 <= s <= FLT_MAX
        const float ny = -__frcp_rn(s);
        const float2 ny2 = make_float2(ny, ny), s2 = make_float2(s, s), ns2 = make_float2(-s, -s);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const float2 w2 = make_float2(w[2 * p], w[2 * p + 1]);
            const float2 a = __fmul2_rn(w2, ny2);
            const float2 r = __ffma2_rn(a, s2, w2);
            const float2 v = __ffma2_rn(r, ny2, a);
            const uint32_t c2 = e2m1x2_codes(v.x, v.y);  // codes of -q, element 2p in the low nibble
            if constexpr (kOut) {
                const float2 q = __fmul2_rn(e2m1x2_values(c2), ns2);
                o[2 * p] = q.x;
                o[2 * p + 1] = q.y;
            }
            if constexpr (kPack) word[p >> 2] |= c2 << (8 * (p & 3));
        }
        word[0] ^= 0x88888888u;  // the sign bit of every nibble
        word[1] ^= 0x88888888u;
        return;
    }
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        float u[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const float wi = w[2 * p + h];
            u[h] = (s != 0.0f) ? __fdiv_rn(wi, s) : copysignf(0.0f, wi);
        }
        const uint32_t c2 = e2m1x2_codes(u[0], u[1]);
        if constexpr (kOut) {
            const float2 q = e2m1x2_values(c2);
            o[2 * p] = __fmul_rn(q.x, s);
            o[2 * p + 1] = __fmul_rn(q.y, s);
        }
        if constexpr (kPack) word[p >> 2] |= c2 << (8 * (p & 3));
    }
}

}  // namespace lh
