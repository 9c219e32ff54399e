// Baseline block scalers: max scaling and four-over-six (the weight-MSE
// baseline is lh_sweep_scales with the identity H).
//
// "NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4 逐块权重缩放
// 算法实战指南" (xxmr.cn/news/266017), section "Local-Hessian 是什么": max
// scaling takes the block scale from the largest |w| of the 16 weights so that
// they fall inside the E2M1 range; four-over-six picks one of two candidate
// scales by the in-block error; the MSE method sweeps all 126 codes on the
// weight error. The pages give no formulas; the readings here:
//   max:           code = E4M3_RNE_sat(fp32(fp32(amax_b / 6) / g)), at least 1;
//   four-over-six: the codes of amax_b / 6 and amax_b / 4 the same way, keep the
//                  one with the smaller FP64 sum of dw^2 (the lower code on ties).
// One thread per block; W is streamed once.
#include "common.cuh"
#include "quant.cuh"

namespace lh {
namespace {

template <typename T>
__device__ __forceinline__ void load16(const T* p, float (&w)[16]);
template <>
__device__ __forceinline__ void load16<uint16_t>(const uint16_t* p, float (&w)[16]) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
    const uint4 a = __ldg(q), b = __ldg(q + 1);
    const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        w[2 * i] = __uint_as_float(v[i] << 16);
        w[2 * i + 1] = __uint_as_float(v[i] & 0xFFFF0000u);
    }
}
template <>
__device__ __forceinline__ void load16<float>(const float* p, float (&w)[16]) {
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 t = __ldg(q + i);
        w[4 * i] = t.x; w[4 * i + 1] = t.y; w[4 * i + 2] = t.z; w[4 * i + 3] = t.w;
    }
}

// FP64 sum of dw^2 for one candidate, in index order (no contraction).
__device__ double weight_error(const float (&w)[16], float s) {
    double e = 0.0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float q = (s != 0.0f) ? e2m1_rne(__fdiv_rn(w[i], s)) : 0.0f;
        const double d = __fma_rn((double)q, (double)s, -(double)w[i]);  // q s - w, exact
        e = __dadd_rn(e, __dmul_rn(d, d));
    }
    return e;
}

template <typename T, bool kFourOverSix>
__global__ void __launch_bounds__(256) baseline_kernel(const T* __restrict__ W, int64_t c_out, int64_t J, int64_t ld,
                                                       const float* __restrict__ gamax, float* __restrict__ best_amax,
                                                       uint8_t* __restrict__ best_code, int64_t n_blocks_total) {
    const int64_t per_mat = c_out * J;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < n_blocks_total;
         b += (int64_t)gridDim.x * blockDim.x) {
        const int64_t m = b / per_mat;
        const int64_t rj = b - m * per_mat;
        const int64_t r = rj / J, j = rj - r * J;
        const float g = __fdiv_rn(__ldg(gamax + m), 2688.0f);
        float w[16];
        load16<T>(W + (m * c_out + r) * ld + 16 * j, w);
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(w[i]));
        auto code_for = [&](float d) -> int {
            if (g == 0.0f) return 1;  // every scale is 0
            const int c = e4m3_rne_code(__fdiv_rn(__fdiv_rn(a, d), g));
            return c < 1 ? 1 : c;
        };
        int c = code_for(6.0f);
        if constexpr (kFourOverSix) {
            const int c4 = code_for(4.0f);
            if (c4 != c) {
                const double e6 = weight_error(w, __fmul_rn(e4m3_value(c), g));
                const double e4 = weight_error(w, __fmul_rn(e4m3_value(c4), g));
                if (e4 < e6 || (e4 == e6 && c4 < c)) c = c4;
            }
        }
        best_code[b] = (uint8_t)c;
        best_amax[b] = __fmul_rn(6.0f, __fmul_rn(e4m3_value(c), g));
    }
}

template <bool kFos>
void launch(const void* W, lh_dtype dt, int64_t c_out, int64_t J, int64_t ld, const float* gamax, float* best_amax,
            uint8_t* best_code, int64_t nb, unsigned grid, cudaStream_t st) {
    if (dt == LH_BF16)
        baseline_kernel<uint16_t, kFos><<<grid, 256, 0, st>>>((const uint16_t*)W, c_out, J, ld, gamax, best_amax,
                                                               best_code, nb);
    else
        baseline_kernel<float, kFos><<<grid, 256, 0, st>>>((const float*)W, c_out, J, ld, gamax, best_amax,
                                                            best_code, nb);
}

}  // namespace
}  // namespace lh

extern "C" lh_status lh_baseline_scales(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out, int64_t c_in,
                                        int64_t ld_w, const float* global_amax, lh_scaler method, float* best_amax,
                                        uint8_t* best_code, void* stream) {
    using namespace lh;
    clear_error();
    if (method == LH_SCALE_MSE)
        return lh_sweep_scales(W, w_dtype, n_mats, c_out, c_in, ld_w, global_amax, nullptr, best_amax, best_code,
                               stream);
    if (method != LH_SCALE_MAX && method != LH_SCALE_FOUR_OVER_SIX)
        return fail(LH_ERR_UNSUPPORTED, "unknown scaler %d", (int)method);
    if (!valid_dtype(w_dtype)) return fail(LH_ERR_UNSUPPORTED, "w_dtype %d is not LH_BF16 or LH_F32", (int)w_dtype);
    if (!W || !global_amax || !best_amax || !best_code) return fail(LH_ERR_INVALID_ARG, "null pointer argument");
    if (n_mats < 1 || c_out < 0 || c_in < 0) return fail(LH_ERR_INVALID_ARG, "n_mats must be >= 1, sizes >= 0");
    if (c_in % 16 != 0) return fail(LH_ERR_UNSUPPORTED, "c_in=%lld is not a multiple of 16", (long long)c_in);
    if (ld_w < c_in) return fail(LH_ERR_INVALID_ARG, "ld_w=%lld < c_in=%lld", (long long)ld_w, (long long)c_in);
    if (!aligned16(W) || (ld_w * elem_bytes(w_dtype)) % 16 != 0)
        return fail(LH_ERR_ALIGNMENT, "W must be 16-byte aligned with 16-byte aligned rows");
    const int64_t J = c_in / 16;
    const int64_t nb = n_mats * c_out * J;
    if (nb == 0) return LH_OK;
    const int sms = sm_count();
    if (sms <= 0) return fail(LH_ERR_CUDA, "no CUDA device");
    int64_t blocks = (nb + 255) / 256;
    if (blocks > (int64_t)sms * 16) blocks = (int64_t)sms * 16;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (method == LH_SCALE_MAX)
        launch<false>(W, w_dtype, c_out, J, ld_w, global_amax, best_amax, best_code, nb, (unsigned)blocks, st);
    else
        launch<true>(W, w_dtype, c_out, J, ld_w, global_amax, best_amax, best_code, nb, (unsigned)blocks, st);
    return cuda_status(cudaGetLastError(), "baseline_kernel launch");
}
