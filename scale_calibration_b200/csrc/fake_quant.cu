// Fake quantisation with the chosen block scales, and the global abs-max.
//
// "NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4 逐块权重缩放
// 算法实战指南" (xxmr.cn/news/266017), section "算法原理": Q(W, s) = Cast(W/s) * s
// with the per-block FP8 scale s and the global FP32 amax of the tensor.
//
// Both kernels stream W once from HBM: one thread per 16-weight block
// (32 or 64 contiguous bytes, 16-byte vector loads and stores).
#include "nvfp4_block.cuh"

namespace lh {
namespace {

// kOut: write the fake-quantised W; kPack: write the packed NVFP4 nibbles (two
// per byte, even column in the low nibble) and the block scale bytes.
// One thread per block, the 16 weights in one fused pass (quotient, E2M1
// rounding, product, packing) so few values stay live and more CTAs fit an SM.
template <typename Tin, typename Tout, bool kOut, bool kPack>
__global__ void __launch_bounds__(256, 4) fake_quant_kernel(const Tin* __restrict__ W, int64_t c_out, int64_t J,
                                                            int64_t ld, const float* __restrict__ gamax,
                                                            const uint8_t* __restrict__ codes,
                                                            Tout* __restrict__ out, uint8_t* __restrict__ packed,
                                                            uint8_t* __restrict__ scales, int64_t n_blocks_total) {
    const int64_t per_mat = c_out * J;
    const bool dense = ld == 16 * J;  // W rows back to back: block b starts at element 16 b
    int64_t m_cached = -1;
    float g = 0.0f;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < n_blocks_total;
         b += (int64_t)gridDim.x * blockDim.x) {
        int64_t m = 0, src = 16 * b;
        if (dense) {
            if (per_mat != n_blocks_total) m = b / per_mat;
        } else {
            m = b / per_mat;
            const int64_t rj = b - m * per_mat;
            const int64_t r = rj / J, j = rj - r * J;
            src = (m * c_out + r) * ld + 16 * j;
        }
        if (m != m_cached) {
            g = __fdiv_rn(__ldg(gamax + m), 2688.0f);
            m_cached = m;
        }
        const uint8_t code = __ldg(codes + b);
        const float s = __fmul_rn(e4m3_value(code), g);
        float w[16];
        Vec16<Tin>::load(W + src, w);
        float o[16];
        uint32_t word[2];
        quantize_block<kOut, kPack>(w, s, o, word);
        if constexpr (kOut) Vec16<Tout>::store(out + 16 * b, o);
        if constexpr (kPack) {
            *reinterpret_cast<uint2*>(packed + 8 * b) = make_uint2(word[0], word[1]);
            if (scales) scales[b] = code;
        }
    }
}

__global__ void global_scale_kernel(const float* __restrict__ gamax, float* __restrict__ gs, int64_t n) {
    for (int64_t m = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; m < n; m += (int64_t)gridDim.x * blockDim.x)
        gs[m] = __fdiv_rn(gamax[m], 2688.0f);
}

template <typename T>
__global__ void __launch_bounds__(256) absmax_kernel(const T* __restrict__ W, int64_t rows, int64_t cols,
                                                     int64_t ld, unsigned int* __restrict__ out) {
    const int64_t m = blockIdx.y;
    const T* base = W + m * rows * ld;
    constexpr int V = 16 / sizeof(T);  // elements per 16-byte vector
    const int64_t nv = cols / V;
    const int warps = blockDim.x >> 5;
    const int lane = threadIdx.x & 31;
    float mx = 0.0f;
    for (int64_t r = (int64_t)blockIdx.x * warps + (threadIdx.x >> 5); r < rows; r += (int64_t)gridDim.x * warps) {
        const T* row = base + r * ld;
        const uint4* rv = reinterpret_cast<const uint4*>(row);
        auto fold = [&](const uint4& t) {
            const uint32_t u[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if (sizeof(T) == 2) {
                    mx = fmaxf(mx, fabsf(__uint_as_float(u[i] << 16)));
                    mx = fmaxf(mx, fabsf(__uint_as_float(u[i] & 0xFFFF0000u)));
                } else {
                    mx = fmaxf(mx, fabsf(__uint_as_float(u[i])));
                }
            }
        };
        int64_t v = lane;
        for (; v + 96 < nv; v += 128) {  // four independent 16-byte loads in flight per lane
            const uint4 t0 = __ldg(rv + v), t1 = __ldg(rv + v + 32), t2 = __ldg(rv + v + 64), t3 = __ldg(rv + v + 96);
            fold(t0); fold(t1); fold(t2); fold(t3);
        }
        for (; v < nv; v += 32) fold(__ldg(rv + v));
        for (int64_t c = nv * V + lane; c < cols; c += 32) {
            const float x = sizeof(T) == 2 ? bf16_bits_to_float(reinterpret_cast<const uint16_t*>(row)[c])
                                           : reinterpret_cast<const float*>(row)[c];
            mx = fmaxf(mx, fabsf(x));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    __shared__ float red[32];
    if (lane == 0) red[threadIdx.x >> 5] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
        float v = 0.0f;
        for (int i = 0; i < warps; ++i) v = fmaxf(v, red[i]);
        // launched as a programmatic dependent of absmax_init_kernel: the loads above
        // overlap it, the atomics wait for its zeros
        asm volatile("griddepcontrol.wait;" ::: "memory");
        atomicMax(out + m, __float_as_uint(v));  // non-negative floats order like their bits
    }
}

__global__ void absmax_init_kernel(unsigned int* __restrict__ out, int64_t n) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = 0u;
}

template <bool kOut, bool kPack>
void launch_fake_quant(const void* W, lh_dtype w_dtype, int64_t c_out, int64_t J, int64_t ld,
                       const float* gamax, const uint8_t* codes, void* out, lh_dtype out_dtype, uint8_t* packed,
                       uint8_t* scales, int64_t nb, unsigned grid, cudaStream_t st) {
    if (w_dtype == LH_BF16 && out_dtype == LH_BF16)
        fake_quant_kernel<uint16_t, uint16_t, kOut, kPack><<<grid, 256, 0, st>>>(
            (const uint16_t*)W, c_out, J, ld, gamax, codes, (uint16_t*)out, packed, scales, nb);
    else if (w_dtype == LH_BF16)
        fake_quant_kernel<uint16_t, float, kOut, kPack><<<grid, 256, 0, st>>>(
            (const uint16_t*)W, c_out, J, ld, gamax, codes, (float*)out, packed, scales, nb);
    else if (out_dtype == LH_BF16)
        fake_quant_kernel<float, uint16_t, kOut, kPack><<<grid, 256, 0, st>>>(
            (const float*)W, c_out, J, ld, gamax, codes, (uint16_t*)out, packed, scales, nb);
    else
        fake_quant_kernel<float, float, kOut, kPack><<<grid, 256, 0, st>>>(
            (const float*)W, c_out, J, ld, gamax, codes, (float*)out, packed, scales, nb);
}

}  // namespace
}  // namespace lh

extern "C" lh_status lh_fake_quant(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out, int64_t c_in,
                                   int64_t ld_w, const float* global_amax, const uint8_t* codes, void* W_out,
                                   lh_dtype out_dtype, void* stream) {
    using namespace lh;
    clear_error();
    if (!valid_dtype(w_dtype) || !valid_dtype(out_dtype)) return fail(LH_ERR_UNSUPPORTED, "unknown dtype");
    if (!W || !global_amax || !codes || !W_out) return fail(LH_ERR_INVALID_ARG, "null pointer argument");
    if (n_mats < 1 || c_out < 0 || c_in < 0) return fail(LH_ERR_INVALID_ARG, "n_mats must be >= 1, sizes >= 0");
    if (c_in % 16 != 0) return fail(LH_ERR_UNSUPPORTED, "c_in=%lld is not a multiple of 16", (long long)c_in);
    if (ld_w < c_in) return fail(LH_ERR_INVALID_ARG, "ld_w < c_in");
    if (!aligned16(W) || (ld_w * elem_bytes(w_dtype)) % 16 != 0 || !aligned16(W_out))
        return fail(LH_ERR_ALIGNMENT, "W and W_out must be 16-byte aligned with 16-byte aligned rows");
    if (W == W_out) return fail(LH_ERR_INVALID_ARG, "W_out must not alias W");
    const int64_t J = c_in / 16;
    const int64_t nb = n_mats * c_out * J;
    if (nb == 0) return LH_OK;
    const int sms = sm_count();
    if (sms <= 0) return fail(LH_ERR_CUDA, "no CUDA device");
    int64_t blocks = (nb + 255) / 256;
    if (blocks > (int64_t)sms * 32) blocks = (int64_t)sms * 32;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const unsigned gb = (unsigned)blocks;
    launch_fake_quant<true, false>(W, w_dtype, c_out, J, ld_w, global_amax, codes, W_out, out_dtype, nullptr, nullptr,
                                   nb, gb, st);
    return cuda_status(cudaGetLastError(), "fake_quant_kernel launch");
}

extern "C" lh_status lh_quantize_nvfp4(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out,
                                       int64_t c_in, int64_t ld_w, const float* global_amax, const uint8_t* codes,
                                       uint8_t* packed, uint8_t* block_scales, float* global_scale, void* W_out,
                                       lh_dtype out_dtype, void* stream) {
    using namespace lh;
    clear_error();
    if (!valid_dtype(w_dtype) || (W_out && !valid_dtype(out_dtype))) return fail(LH_ERR_UNSUPPORTED, "unknown dtype");
    if (!W || !global_amax || !codes || !packed) return fail(LH_ERR_INVALID_ARG, "null pointer argument");
    if (n_mats < 1 || c_out < 0 || c_in < 0) return fail(LH_ERR_INVALID_ARG, "n_mats must be >= 1, sizes >= 0");
    if (c_in % 16 != 0) return fail(LH_ERR_UNSUPPORTED, "c_in=%lld is not a multiple of 16", (long long)c_in);
    if (ld_w < c_in) return fail(LH_ERR_INVALID_ARG, "ld_w < c_in");
    if (!aligned16(W) || (ld_w * elem_bytes(w_dtype)) % 16 != 0 || !aligned16(packed) || (W_out && !aligned16(W_out)))
        return fail(LH_ERR_ALIGNMENT, "W, packed and W_out must be 16-byte aligned, with 16-byte aligned rows of W");
    if (W == W_out || W == (const void*)packed) return fail(LH_ERR_INVALID_ARG, "outputs must not alias W");
    const int64_t J = c_in / 16;
    const int64_t nb = n_mats * c_out * J;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (global_scale) {
        global_scale_kernel<<<(unsigned)((n_mats + 255) / 256), 256, 0, st>>>(global_amax, global_scale, n_mats);
        lh_status s = cuda_status(cudaGetLastError(), "global_scale_kernel launch");
        if (s != LH_OK) return s;
    }
    if (nb == 0) return LH_OK;
    const int sms = sm_count();
    if (sms <= 0) return fail(LH_ERR_CUDA, "no CUDA device");
    int64_t blocks = (nb + 255) / 256;
    if (blocks > (int64_t)sms * 32) blocks = (int64_t)sms * 32;
    if (W_out)
        launch_fake_quant<true, true>(W, w_dtype, c_out, J, ld_w, global_amax, codes, W_out, out_dtype, packed,
                                      block_scales, nb, (unsigned)blocks, st);
    else
        launch_fake_quant<false, true>(W, w_dtype, c_out, J, ld_w, global_amax, codes, nullptr, LH_F32, packed,
                                       block_scales, nb, (unsigned)blocks, st);
    return cuda_status(cudaGetLastError(), "fake_quant_kernel launch");
}

extern "C" lh_status lh_absmax(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t rows, int64_t cols,
                               int64_t ld, float* out_amax, void* stream) {
    using namespace lh;
    clear_error();
    if (!valid_dtype(w_dtype)) return fail(LH_ERR_UNSUPPORTED, "unknown dtype");
    if (!W || !out_amax) return fail(LH_ERR_INVALID_ARG, "null pointer argument");
    if (n_mats < 1 || rows < 0 || cols < 0 || ld < cols) return fail(LH_ERR_INVALID_ARG, "bad sizes");
    if (n_mats > 65535) return fail(LH_ERR_UNSUPPORTED, "n_mats must be <= 65535");
    if (!aligned16(W) || (ld * elem_bytes(w_dtype)) % 16 != 0)
        return fail(LH_ERR_ALIGNMENT, "W must be 16-byte aligned with 16-byte aligned rows");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    absmax_init_kernel<<<(unsigned)((n_mats + 255) / 256), 256, 0, st>>>((unsigned int*)out_amax, n_mats);
    lh_status s = cuda_status(cudaGetLastError(), "absmax_init_kernel launch");
    if (s != LH_OK) return s;
    if (rows == 0 || cols == 0) return LH_OK;
    const int sms = sm_count();
    if (sms <= 0) return fail(LH_ERR_CUDA, "no CUDA device");
    int64_t per = (rows + 7) / 8;  // 8 warps per CTA, one row per warp per pass
    int64_t cap = ((int64_t)sms * 8) / n_mats;  // one wave of 8 CTAs per SM, none left over
    if (cap < 1) cap = 1;
    if (per > cap) per = cap;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)per, (unsigned)n_mats);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    unsigned int* o = (unsigned int*)out_amax;
    if (w_dtype == LH_BF16)
        s = cuda_status(cudaLaunchKernelEx(&cfg, absmax_kernel<uint16_t>, (const uint16_t*)W, rows, cols, ld, o),
                        "absmax_kernel launch");
    else
        s = cuda_status(cudaLaunchKernelEx(&cfg, absmax_kernel<float>, (const float*)W, rows, cols, ld, o),
                        "absmax_kernel launch");
    return s;
}
