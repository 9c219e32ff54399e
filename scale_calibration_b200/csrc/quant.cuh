// NVFP4 format arithmetic on the device: E4M3 candidate values and exact
// E2M1 round-to-nearest-even.
//
// Format: "NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4 逐块
// 权重缩放算法实战指南" (xxmr.cn/news/266017), section "Local-Hessian 是什么":
// E2M1 weights in [-6, 6], one FP8 E4M3 scale per 16 weights, 126 positive
// non-zero finite E4M3 scale candidates.
#pragma once

#include <stdint.h>

namespace lh {

// Value of E4M3 code c in 1..126: subnormal c < 8 -> c * 2^-9, else
// (1 + (c & 7)/8) * 2^((c >> 3) - 7). Exact in FP32.
__device__ __forceinline__ float e4m3_value(int c) {
    const int e = c >> 3, f = c & 7;
    if (e == 0) return (float)f * 0.001953125f;  // 2^-9
    // (8 + f) * 2^(e - 10)
    return (float)(8 + f) * __int_as_float((e - 10 + 127) << 23);
}

// Rounds x >= 0 onto the E2M1 grid scaled by 2^k, {0, .5, 1, 1.5, 2, 3, 4, 6} * 2^k,
// round-to-nearest-even, saturating at 6 * 2^k. Exact for every FP32 input:
//   xc  = min(x, 6*2^k)                           (NaN -> 6*2^k)
//   sp  = grid spacing at xc: half the unit of the binade of max(xc, 2^k)
//   M   = 1.5 * 2^23 * sp  (an FP32 number whose ulp is sp; M/sp is even)
//   q   = (xc + M) - M     both additions IEEE round-to-nearest-even.
// Adding M rounds xc to a multiple of sp with ties to an even multiple,
// which is the E2M1 even mantissa; xc + M never leaves M's binade because
// xc < 4 sp there. `lim` = 6*2^k and `emin` = the FP32 exponent field of 2^k
// (as bits) are per-k constants.
__device__ __forceinline__ float e2m1_grid_round(float x, float lim, int emin_bits) {
    const float xc = fminf(x, lim);
    int e = __float_as_int(xc) & 0x7F800000;
    e = max(e, emin_bits);
    const float M = __int_as_float(e + 0x0B400000);  // exponent +22, mantissa .5
    return __fsub_rn(__fadd_rn(xc, M), M);
}

// Signed E2M1 RNE with saturation at +-6 of an FP32 value u (k = 0 grid).
__device__ __forceinline__ float e2m1_rne(float u) {
    const float q = e2m1_grid_round(fabsf(u), 6.0f, 127 << 23);
    return copysignf(q, u);
}

// E4M3 code of x >= 0: round to nearest even, saturating at 448 (the hardware
// conversion; both halves of the pair take x, the low byte is kept).
__device__ __forceinline__ int e4m3_rne_code(float x) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %1;" : "=h"(r) : "f"(x));
    return r & 0xFF;
}

}  // namespace lh
