// FP32 FMA throughput probe: the ceiling the sweep's roofline is measured
// against. The sweep is bound by FP32 CUDA-core arithmetic; its form uses
// packed two-lane FMAs (fma.rn.f32x2) and its other steps scalar ones, so the
// probe times both kinds on every SM: if the packed form retires two FMAs per
// lane per cycle, the FP32 ceiling is twice the scalar one. Diagnostics only;
// the calibration method has no counterpart.
#include "common.cuh"

namespace lh {
namespace {

constexpr int kProbeThreads = 256;
constexpr int kChains = 8;  // independent accumulator pairs per thread

// Each thread runs kChains independent chains of 2 FMAs per step (one packed
// f32x2 FMA, or two scalar FMAs issued through inline PTX so that they stay
// scalar), `iters` steps. The values stay finite (|a| < 1). The sum is stored
// only when it equals a value it never takes, so the work cannot be removed.
template <bool kPacked>
__global__ void __launch_bounds__(kProbeThreads) fma_probe_kernel(float* out, int iters, float a, float b) {
    float2 x[kChains];
#pragma unroll
    for (int c = 0; c < kChains; ++c) x[c] = make_float2(threadIdx.x * 1e-3f + c, blockIdx.x * 1e-3f - c);
    const float2 a2 = make_float2(a, a), b2 = make_float2(b, b);
#pragma unroll 1
    for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
#pragma unroll
            for (int c = 0; c < kChains; ++c) {
                if constexpr (kPacked) {
                    x[c] = __ffma2_rn(x[c], a2, b2);
                } else {
                    asm volatile("fma.rn.f32 %0, %0, %1, %2;" : "+f"(x[c].x) : "f"(a), "f"(b));
                    asm volatile("fma.rn.f32 %0, %0, %1, %2;" : "+f"(x[c].y) : "f"(a), "f"(b));
                }
            }
        }
    }
    float s = 0.0f;
#pragma unroll
    for (int c = 0; c < kChains; ++c) s += x[c].x + x[c].y;
    if (s == -1.2345e30f) out[0] = s;
}

}  // namespace
}  // namespace lh

extern "C" int64_t lh_probe_fma_flop(int64_t blocks, int64_t iters) {
    if (blocks < 1 || iters < 1) return 0;
    return blocks * lh::kProbeThreads * iters * 4 * lh::kChains * 2 * 2;  // 2 FMAs per chain step, 2 flop each
}

extern "C" lh_status lh_probe_fma(int packed, int64_t blocks, int64_t iters, float* out, void* stream) {
    using namespace lh;
    clear_error();
    if (!out) return fail(LH_ERR_INVALID_ARG, "null out");
    if (blocks < 1 || blocks > (1 << 20) || iters < 1 || iters > (1 << 24))
        return fail(LH_ERR_INVALID_ARG, "blocks must be in [1, 2^20] and iters in [1, 2^24]");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (packed)
        fma_probe_kernel<true><<<(unsigned)blocks, kProbeThreads, 0, st>>>(out, (int)iters, 0.999f, 1e-3f);
    else
        fma_probe_kernel<false><<<(unsigned)blocks, kProbeThreads, 0, st>>>(out, (int)iters, 0.999f, 1e-3f);
    return cuda_status(cudaGetLastError(), "fma_probe_kernel launch");
}
