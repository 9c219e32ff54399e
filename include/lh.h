/*
 * lh.h — C ABI of the Local-Hessian NVFP4 block-scale calibration library
 * (B200, sm_100a).
 *
 * The method ("NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4
 * 逐块权重缩放算法实战指南", xxmr.cn/news/266017, section "算法原理"): for a
 * linear layer Y = W X with W [C_out, C_in] and calibration activations X
 * (token-major here, [N tokens, C_in]), every NVFP4 block of 16 consecutive
 * weights w_b = W[r, 16j:16j+16] gets the FP8 E4M3 block scale s that
 * minimises the output-error proxy E_b(s) = dw^T H_j dw, where
 * dw = Cast_E2M1(w/s)*s - w and H_j = X_j X_j^T is the 16x16 local Hessian of
 * the block's 16 input channels. All 126 positive finite non-zero E4M3 codes
 * (0x01..0x7E) are tried as candidates s = fp8(c) * g, g = global_amax/(6*448).
 *
 * Conventions (all entry points):
 *   - Pointers marked "device" are caller-owned device memory of the current
 *     CUDA device; the library allocates nothing (the Hessian partial sums
 *     live in a caller-provided workspace).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream). Every call is asynchronous on that stream and returns without
 *     synchronising; a kernel fault surfaces at the caller's next sync.
 *   - Arguments are validated on the host before any launch. On an error
 *     status nothing was launched and no output was touched.
 *   - Matrices are row-major. Leading dimensions are in elements.
 *   - bf16 and f32 element pointers must be 16-byte aligned and leading
 *     dimensions must keep every row 16-byte aligned (LH_ERR_ALIGNMENT).
 *   - Outputs must not alias inputs.
 *   - Thread safety: calls are re-entrant; the only host state is a
 *     thread-local error message.
 */
#ifndef LH_H_
#define LH_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LH_API __attribute__((visibility("default")))
#else
#define LH_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LH_OK = 0,
    LH_ERR_INVALID_ARG = 1,   /* null pointer, negative size, ld < cols, ...      */
    LH_ERR_UNSUPPORTED = 2,   /* c_in not a multiple of 16, unknown dtype, no GPU */
    LH_ERR_ALIGNMENT = 3,     /* pointer or row not 16-byte aligned                */
    LH_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required        */
    LH_ERR_CUDA = 5,          /* a CUDA runtime call or launch failed              */
    LH_ERR_TIMEOUT = 6        /* a bounded in-kernel wait gave up (see lh_workspace_status) */
} lh_status;

typedef enum { LH_BF16 = 0, LH_F32 = 1 } lh_dtype;

/* Human-readable name of a status code (static string). */
LH_API const char* lh_status_string(lh_status s);

/* Detail of the last error returned on this host thread (e.g. the CUDA error
 * name and which argument failed). Empty string if none. */
LH_API const char* lh_last_error_message(void);

/* ------------------------------------------------------------------------
 * Global amax. "算法原理" (kernel contract): the sweep receives the global
 * FP32 amax of the weight tensor. out_amax[m] = max |W_m| over the matrix
 * [rows, cols] (leading dimension ld) of each of n_mats matrices stored back
 * to back (matrix stride rows*ld). Exact (a max is order-independent).
 *   W: device, bf16 or f32.  out_amax: device f32 [n_mats], overwritten.
 * ---------------------------------------------------------------------- */
LH_API lh_status lh_absmax(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t rows, int64_t cols,
                    int64_t ld, float* out_amax, void* stream);

/* ------------------------------------------------------------------------
 * Local Hessian accumulation. "算法原理": the local Hessian of block column j
 * is X_j X_j^T (16x16); "入口 API 与校准流程" Phase 2: H = sum X^T X over the
 * calibration tokens; kernel contract: H laid out [C_in/16, 16, 16].
 *
 *   H[g][j][a][b] += sum_{t in group g} x[t][16j+a] * x[t][16j+b]
 *
 * X: device bf16 [n_tokens_total, ld_x] (first c_in columns used), token-major.
 * offsets: device int64 [n_groups+1], non-decreasing, with the token range of
 *   each group (one per matrix / expert: tokens [offsets[g], offsets[g+1])), or
 *   NULL for a single group of all tokens (n_groups must then be 1). Offsets
 *   are clamped to [0, n_tokens_total]; tokens outside [offsets[0],
 *   offsets[n_groups]) belong to no group. Decreasing offsets make the call
 *   record LH_ERR_INVALID_ARG in the workspace (see lh_workspace_status); the
 *   kernel stays in bounds and H is then unspecified.
 * H: device f32 [n_groups][c_in/16][16][16], read and written (H += ...):
 *   accumulation can be split over batches and resumed across calls.
 * workspace: device, at least lh_hessian_workspace_bytes(...) bytes, 256-byte
 *   aligned, owned by the caller; it holds a status word, and the partial sums
 *   (with their ready flags) of the (slab, group) segments that several CTAs
 *   share.
 *   Its size depends on n_tokens_total and c_in only, is at most about 5.3 MB,
 *   and its contents need no clearing between calls; it must not be shared by
 *   calls in flight at the same time.
 * Work split: one kernel launch; each CTA (two per SM) reads an equal share of
 *   X whatever the group sizes. A CTA waits (bounded, 1 s) only for parts that
 *   CTAs with lower block indices publish, which the GPU has started before it.
 * Numerics: bf16 products are exact in FP32; tensor-core FP32 accumulation
 *   over at most 128 tokens, then FP64 accumulation, FP32 partial sums where a
 *   segment spans several CTAs, summed in a fixed order (deterministic), and
 *   one final rounding into H.
 * n_tokens_total == 0 is a no-op returning LH_OK.
 * ---------------------------------------------------------------------- */
LH_API size_t lh_hessian_workspace_bytes(int64_t n_tokens_total, int64_t c_in, int64_t n_groups);

LH_API lh_status lh_accumulate_hessian(const void* X, lh_dtype x_dtype, int64_t n_tokens_total, int64_t c_in,
                                int64_t ld_x, const int64_t* offsets, int64_t n_groups, float* H,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Status the last launch on `workspace` left there: LH_OK, LH_ERR_TIMEOUT when
 * a bounded wait inside lh_accumulate_hessian gave up, or LH_ERR_INVALID_ARG
 * when its group offsets decreased. Synchronises `stream`. Each launch stamps
 * the workspace with its own generation number, so an error of an earlier
 * launch is not reported again. */
LH_API lh_status lh_workspace_status(const void* workspace, void* stream);

/* Diagnostics; the pages have no counterpart. Runs on `stream` the bounded
 * wait that the Hessian kernel uses for its mbarriers, on a barrier that
 * nothing arrives on (arrive == 0) or that is completed first (arrive != 0),
 * with a limit of timeout_us microseconds (1 .. 1e6). A wait that runs out
 * records LH_ERR_TIMEOUT in the workspace header exactly as
 * lh_accumulate_hessian does, so lh_workspace_status(workspace) then returns
 * LH_ERR_TIMEOUT (LH_OK when arrive != 0). Lets callers exercise their
 * handling of an expired wait without a GPU fault; the context stays usable.
 * workspace: device, >= 256 bytes, 256-byte aligned. */
LH_API lh_status lh_debug_wait_timeout(void* workspace, size_t workspace_bytes, int64_t timeout_us, int arrive,
                                       void* stream);

/* Diagnostics; the pages have no counterpart. FP32 FMA throughput probe for
 * the sweep's roofline: launches `blocks` CTAs of 256 threads on `stream`, each
 * thread running `iters` steps of 64 FMAs over 16 independent accumulators, as
 * 32 packed two-lane FMAs (fma.rn.f32x2, packed != 0) or 64 scalar fma.rn.f32.
 * The caller times
 * the launch (CUDA events on `stream`); lh_probe_fma_flop(blocks, iters) is the
 * flop count of one launch (2 per FMA). out: device, >= 1 float, never written
 * in practice (it keeps the arithmetic from being removed).
 * LH_ERR_INVALID_ARG: null out, blocks outside [1, 2^20], iters outside [1, 2^24]. */
LH_API int64_t lh_probe_fma_flop(int64_t blocks, int64_t iters);
LH_API lh_status lh_probe_fma(int packed, int64_t blocks, int64_t iters, float* out, void* stream);

/* Diagnostics; the pages have no counterpart. Work counters of the sweep,
 * summed over the launches since the last clear: out[9] = {warp chunks of 32
 * rows, blocks, candidates quantised per warp, full quadratic forms evaluated
 * per warp, forms some lane needed (lane count), class-wide bound tests, blocks
 * re-swept in FP64 (all 126 codes), mantissa classes walked per warp, blocks
 * whose best two candidates were compared in FP64}. clear != 0 zeroes them
 * (out unused). Only a library built with -DLH_SWEEP_COUNTERS=1 (the
 * measurement build, liblh_counters.so) counts; the library itself returns
 * LH_ERR_UNSUPPORTED. Synchronous. */
LH_API lh_status lh_debug_sweep_counts(uint64_t* out, int clear);

/* ------------------------------------------------------------------------
 * Allocation-free variant of lh_accumulate_hessian. The pages have no
 * counterpart: this is a library convenience for callers that cannot
 * allocate device memory when they calibrate (serving processes that reserve
 * nearly all HBM for their own pools at start-up, plugins whose host owns
 * every device allocation, callers that avoid cudaMalloc/cudaFree because
 * those can synchronise the device). Same arguments and result as
 * lh_accumulate_hessian minus the workspace, which comes from a fixed 8 MiB
 * array compiled into the library; every GPU that loads the library holds it
 * until the process exits. Calls no cudaMalloc/cudaFree.
 *   - The largest Hessian workspace is about 5.3 MB, so every size fits; a
 *     size beyond the array would return LH_ERR_WORKSPACE without launching.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - Argument errors are the same, checked in the same order, as those of
 *     lh_accumulate_hessian.
 *   - All calls share the array (it keeps the last call's contents; nothing in
 *     it needs clearing between calls). Calls whose kernels overlap on the GPU
 *     race on it: serialise them (one stream, one thread at a time).
 *   - Errors the kernel finds (an expired bounded wait, decreasing group
 *     offsets) are written to the array's status word, not returned: read them
 *     with lh_noalloc_status after the call, before the next allocation-free
 *     call on that device.
 * ---------------------------------------------------------------------- */
LH_API lh_status lh_accumulate_hessian_noalloc(const void* X, lh_dtype x_dtype, int64_t n_tokens_total,
                                               int64_t c_in, int64_t ld_x, const int64_t* offsets,
                                               int64_t n_groups, float* H, void* stream);

/* Status the last lh_accumulate_hessian_noalloc call on the current device left
 * in the library's scratch array: LH_OK, LH_ERR_TIMEOUT or LH_ERR_INVALID_ARG
 * with the meaning lh_workspace_status gives them. Synchronises `stream` (pass
 * the stream of that call). The pages have no counterpart. */
LH_API lh_status lh_noalloc_status(void* stream);

/* ------------------------------------------------------------------------
 * FP8 block-scale sweep. "算法原理": per 16-weight block, all 126 FP8 E4M3
 * candidate scales are tried and the one minimising dw^T H dw is kept; the
 * kernel contract takes weights as [N_BLOCKS, 16] row-major over
 * (cout, cin/16), the global FP32 amax and H [cin/16, 16, 16], and returns
 * the per-block best amax. For every matrix m and block (r, j):
 *
 *   g     = fp32(global_amax[m] / 2688)
 *   s_c   = fp32(e4m3(c) * g),              c = 1..126
 *   q_i   = E2M1_RNE_sat(fp32(w_i / s_c))   (q = 0 when s_c == 0)
 *   E(c)  = dw^T H[m][j] dw,  dw = q*s_c - w
 *   best_code[m][r][j] = argmin_c E(c)  (lowest code on ties)
 *   best_amax[m][r][j] = fp32(6 * s_best)
 *
 * E is evaluated in FP32. When only the runner-up is within a proven bound on
 * the FP32 rounding error of the best, the two are compared in FP64; when a
 * third candidate is within it too, all 126 codes are re-evaluated in FP64. So
 * the chosen code is the exact argmin up to FP64 rounding.
 * W: device bf16 or f32 [n_mats][c_out][ld_w]. global_amax: device f32 [n_mats], finite
 *   and >= 0 (as lh_absmax writes it); 0 is defined (every block gets code 1 and amax 0);
 *   a NaN, infinite or negative value is not detected and gives unspecified codes.
 * H: device f32 [n_mats][c_in/16][16][16] (both triangles are read; E depends on the
 *   symmetric part (H + H^T)/2 only, so a symmetric H from lh_accumulate_hessian and any
 *   matrix with the same symmetric part give the same codes), or NULL for the identity
 *   (the weight-MSE sweep of the pages' MSE baseline).
 * best_amax: device f32 [n_mats][c_out][c_in/16]. best_code: device u8, same shape.
 * ---------------------------------------------------------------------- */
LH_API lh_status lh_sweep_scales(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out, int64_t c_in,
                          int64_t ld_w, const float* global_amax, const float* H, float* best_amax,
                          uint8_t* best_code, void* stream);

/* ------------------------------------------------------------------------
 * lh_sweep_scales with a caller-provided workspace; the same arguments, the
 * same results bit for bit. The workspace holds one 16-byte record per block
 * column and matrix: the pruning bounds of its H, computed once by a first
 * kernel instead of by every CTA of the column, which makes the call faster.
 * workspace: device, 16-byte aligned, at least
 *   lh_sweep_workspace_bytes(n_mats, c_in) = 16 * n_mats * (c_in / 16) bytes;
 *   its contents on entry do not matter and are overwritten; it must not be
 *   used by another call until this one has finished on `stream`.
 * Errors as lh_sweep_scales, plus LH_ERR_WORKSPACE (NULL or too small) and
 * LH_ERR_ALIGNMENT (workspace not 16-byte aligned).
 * ---------------------------------------------------------------------- */
LH_API size_t lh_sweep_workspace_bytes(int64_t n_mats, int64_t c_in);
LH_API lh_status lh_sweep_scales_ws(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out, int64_t c_in,
                                    int64_t ld_w, const float* global_amax, const float* H, float* best_amax,
                                    uint8_t* best_code, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Fake quantisation with the chosen codes. "算法原理": Q(W, s) = Cast(W/s)*s.
 *   W_out[m][r][c] = cast_out( fp32( E2M1_RNE_sat(fp32(w/s)) * s ) ),
 *   s = fp32(e4m3(codes[m][r][c/16]) * fp32(global_amax[m]/2688)).
 * W: device [n_mats][c_out][ld_w]. codes: device u8 [n_mats][c_out][c_in/16].
 * W_out: device [n_mats][c_out][c_in] (dense), bf16 (round to nearest even) or f32.
 * ---------------------------------------------------------------------- */
LH_API lh_status lh_fake_quant(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out, int64_t c_in,
                        int64_t ld_w, const float* global_amax, const uint8_t* codes, void* W_out,
                        lh_dtype out_dtype, void* stream);

/* ------------------------------------------------------------------------
 * Packed NVFP4 export, in the same pass as the fake quantisation. The pages
 * describe NVFP4 as a two-level scale (E2M1 data, an E4M3 block scale per 16
 * weights, an FP32 global scale) whose scales are computed once when the
 * checkpoint is made ("NVIDIA Model Optimizer Local-Hessian ..." sections
 * "Local-Hessian 是什么" and "仅更好的缩放，零运行时成本"; "GitHub推荐：NVIDIA
 * Model-Optimizer: NVFP4 + QAD ...", section "值得关注的理由"); they give no bit
 * layout. Layout here:
 *   packed[m][r][c/2]   u8: the 4-bit OCP E2M1 code of q for column c (sign bit,
 *                       2 exponent bits with bias 1, 1 mantissa bit), even c in
 *                       the low nibble, odd c in the high nibble;
 *                       q = E2M1_RNE_sat(fp32(w/s)) as in lh_fake_quant (q = +-0
 *                       with the sign of w when s == 0);
 *   block_scales[m][r][j] u8: the E4M3 code of the block scale (= codes);
 *   global_scale[m]     f32: g = fp32(global_amax[m] / 2688).
 * Decoding gives fp32(e2m1(nibble) * fp32(e4m3(scale byte) * g)), bit for bit
 * the value lh_fake_quant writes before its output cast.
 * W: device [n_mats][c_out][ld_w]. codes: device u8 [n_mats][c_out][c_in/16].
 * packed: device, 16-byte aligned, required. block_scales, global_scale and
 * W_out (the fake-quantised W as in lh_fake_quant, out_dtype) are optional
 * (NULL: not written). One read of W serves every output.
 * ---------------------------------------------------------------------- */
LH_API lh_status lh_quantize_nvfp4(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out, int64_t c_in,
                            int64_t ld_w, const float* global_amax, const uint8_t* codes, uint8_t* packed,
                            uint8_t* block_scales, float* global_scale, void* W_out, lh_dtype out_dtype,
                            void* stream);

/* ------------------------------------------------------------------------
 * Baseline block scalers the pages compare Local-Hessian with ("NVIDIA Model
 * Optimizer Local-Hessian ..." section "Local-Hessian 是什么": max scaling
 * from the block's largest |w|, four-over-six choosing one of two candidate
 * scales by the in-block error, and the MSE sweep of all 126 codes on the
 * weight error). The pages give no formulas; with g = fp32(global_amax/2688):
 *   LH_SCALE_MAX:           code = E4M3_RNE_sat(fp32(fp32(amax_b / 6) / g)),
 *                           at least 1 (code 1 when g == 0);
 *   LH_SCALE_FOUR_OVER_SIX: the codes of amax_b / 6 and amax_b / 4 the same
 *                           way; the one with the smaller FP64 sum of dw^2 over
 *                           the block is kept (the lower code on ties);
 *   LH_SCALE_MSE:           lh_sweep_scales with H = NULL (the identity).
 * Outputs as lh_sweep_scales: best_code u8 and best_amax = fp32(6 * s_code),
 * [n_mats][c_out][c_in/16]. W: device bf16 or f32 [n_mats][c_out][ld_w].
 * ---------------------------------------------------------------------- */
typedef enum { LH_SCALE_MAX = 0, LH_SCALE_FOUR_OVER_SIX = 1, LH_SCALE_MSE = 2 } lh_scaler;

LH_API lh_status lh_baseline_scales(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out, int64_t c_in,
                             int64_t ld_w, const float* global_amax, lh_scaler method, float* best_amax,
                             uint8_t* best_code, void* stream);

/* ------------------------------------------------------------------------
 * Amax multiplier search with the Hessian metric: the calibration's other
 * weight search ("NVIDIA Model Optimizer Local-Hessian ..." section
 * "入口 API 与校准流程": step_size 0.1, start_multiplier 0.25,
 * stop_multiplier 4.0 search the block amax when the FP8 scale sweep is off).
 * Readings: multipliers m_k = fp32(start + step * k) for k < n_mult (the pages'
 * values give start 0.25, step 0.1, n_mult 38: the stop is excluded); candidate
 * k of block b is the max-scaling code of the amax m_k * amax_b,
 *   code_k = E4M3_RNE_sat(fp32(fp32(fp32(m_k * amax_b) / 6) / g)), at least 1,
 * and the block keeps the candidate code with the smallest dw^T H dw (the
 * lowest code on ties), exactly as lh_sweep_scales does over all 126 codes.
 * Arguments and outputs as lh_sweep_scales (H may be NULL: the identity);
 * start > 0, step >= 0, 1 <= n_mult <= 4096.
 * ---------------------------------------------------------------------- */
LH_API lh_status lh_search_amax(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out, int64_t c_in,
                         int64_t ld_w, const float* global_amax, const float* H, double start, double step,
                         int64_t n_mult, float* best_amax, uint8_t* best_code, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* LH_H_ */
