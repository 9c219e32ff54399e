// Oracle for Local-Hessian NVFP4 block-scale calibration.
//
// TEST INFRASTRUCTURE ONLY. This file is the plain, slow, single-threaded
// CPU statement of what the calibration hot path computes, written in FP64
// wherever the method leaves the precision open. Only the test suite, the
// smoke check and the CPU-baseline leg of the benchmark may load it. It
// shares no code, header or table with the CUDA library.
//
// Sources (web pages, cited by title and section):
//   [LH]  "NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4
//         逐块权重缩放算法实战指南" (xxmr.cn/news/266017).
//         Sections: "Local-Hessian 是什么" (what it is: the NVFP4 format,
//         the 126-code FP8 sweep), "算法原理" (the error E(s), the local
//         Hessian X_b X_b^T, the per-block sweep and the kernel contract),
//         "入口 API 与校准流程" (Phase 2: H = sum X^T X).
//   [OV]  "NVIDIA Model Optimizer" overview (linlog.top/article/1517),
//         NVFP4 section: 16 weights share one FP8 E4M3 block scale, the
//         weights are E2M1.
// Readings where the pages are silent (global scale g = amax/(6*448), the
// E2M1 rounding mode, the tie rule of the argmin, the degenerate cases) are
// listed in the design notes and restated beside each function below.
//
// Parity status of each function: all are pinned by the CPU test suite
// (closed forms, brute force, library decoders, invariants); none is
// "parity unpinned".
//
// Build: g++ -O2 -std=c++17 -ffp-contract=off -fno-fast-math -shared -fPIC.
// -ffp-contract=off keeps every FP32 step a separately rounded IEEE op.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>

extern "C" {

// ---------------------------------------------------------------------------
// Formats
// ---------------------------------------------------------------------------

// Value of an FP8 E4M3 ("FN": no infinities, S.1111.111 is NaN) byte, as the
// OCP FP8 definition gives it: sign, 4 exponent bits (bias 7), 3 mantissa
// bits, subnormals at exponent field 0. [LH] "Local-Hessian 是什么": the 126
// positive non-zero finite codes 0x01..0x7E are the block-scale candidates.
double oracle_e4m3_value(int code) {
    const int b = code & 0xFF;
    const int sign = (b >> 7) & 1;
    const int e = (b >> 3) & 0xF;
    const int m = b & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return std::numeric_limits<double>::quiet_NaN();
    if (e == 0) v = std::ldexp((double)m, -9);          // m/8 * 2^(1-7)
    else        v = std::ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

// E2M1 round-to-nearest-even with saturation at +-6, as a function of the
// FP32 quotient u. The grid is {0, 0.5, 1, 1.5, 2, 3, 4, 6} (OCP FP4 E2M1;
// [OV] NVFP4 section, [LH] "Local-Hessian 是什么": range [-6, 6]). Values
// half-way between two grid points go to the one whose mantissa bit is 0
// (0, 1, 2, 4 are "even"; 0.5, 1.5, 3, 6 are "odd"); beyond 6 saturates.
// Written as the interval table of the grid's mid-points.
float oracle_e2m1_rne(float u) {
    const float x = std::fabs(u);
    float q;
    if (x <= 0.25f)      q = 0.0f;   // tie 0.25 -> 0
    else if (x < 0.75f)  q = 0.5f;   // tie 0.75 -> 1
    else if (x <= 1.25f) q = 1.0f;   // tie 1.25 -> 1
    else if (x < 1.75f)  q = 1.5f;   // tie 1.75 -> 2
    else if (x <= 2.5f)  q = 2.0f;   // tie 2.5  -> 2
    else if (x < 3.5f)   q = 3.0f;   // tie 3.5  -> 4
    else if (x <= 5.0f)  q = 4.0f;   // tie 5    -> 4
    else                 q = 6.0f;   // (5, inf) -> 6 (saturate)
    return std::signbit(u) ? -q : q;
}

// bfloat16 bits -> float (exact: bf16 is the top half of an FP32 word).
static float bf16_to_float(uint16_t h) {
    uint32_t b = (uint32_t)h << 16;
    float f;
    std::memcpy(&f, &b, 4);
    return f;
}

// float -> bfloat16 bits, round to nearest even (finite inputs).
uint16_t oracle_float_to_bf16(float f) {
    uint32_t b;
    std::memcpy(&b, &f, 4);
    if ((b & 0x7F800000u) == 0x7F800000u) return (uint16_t)((b >> 16) | ((b & 0xFFFF) ? 0x40 : 0));
    const uint32_t lsb = (b >> 16) & 1u;
    b += 0x7FFFu + lsb;
    return (uint16_t)(b >> 16);
}

// ---------------------------------------------------------------------------
// Global amax and scale ([LH] "算法原理": the kernel receives the global FP32
// amax). Reading: g = fp32(amax / (6 * 448)), one FP32 division; 6 is the
// E2M1 maximum and 448 the E4M3 maximum.
// ---------------------------------------------------------------------------

// max |W| over a [rows, cols] matrix with leading dimension ld (FP32, exact).
float oracle_absmax(const float* W, int64_t rows, int64_t cols, int64_t ld) {
    float a = 0.0f;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c) {
            const float x = std::fabs(W[r * ld + c]);
            if (x > a) a = x;
        }
    return a;
}

float oracle_global_scale(float amax) { return amax / 2688.0f; }

// Candidate block scale for code c: s_c = fp32(v(c) * g), one FP32 multiply.
float oracle_candidate_scale(int code, float g) {
    const float v = (float)oracle_e4m3_value(code);  // exact in FP32
    return v * g;
}

// ---------------------------------------------------------------------------
// Local Hessian ([LH] "算法原理": X_b X_b^T is the 16x16 local Hessian of
// block b; "入口 API 与校准流程" Phase 2: H accumulated as sum X^T X over the
// calibration tokens; kernel contract: H laid out [cin/16, 16, 16]).
//
// X: bf16 bits, token-major [n_tok, ld] (only the first c_in columns used).
// Tokens of group g are [offsets[g], offsets[g+1]); offsets == nullptr means
// one group of all tokens. H: [n_groups][c_in/16][16][16], overwritten.
// Every product of two bf16 values is exact in double; the sum runs in token
// order.
// ---------------------------------------------------------------------------
void oracle_hessian(const uint16_t* X, int64_t n_tok, int64_t c_in, int64_t ld,
                    const int64_t* offsets, int64_t n_groups, double* H) {
    const int64_t J = c_in / 16;
    const int64_t G = offsets ? n_groups : 1;
    std::memset(H, 0, sizeof(double) * (size_t)(G * J * 256));
    double xs[16];
    for (int64_t g = 0; g < G; ++g) {
        const int64_t t0 = offsets ? offsets[g] : 0;
        const int64_t t1 = offsets ? offsets[g + 1] : n_tok;
        for (int64_t j = 0; j < J; ++j) {
            double* Hj = H + (g * J + j) * 256;
            for (int64_t t = t0; t < t1; ++t) {
                for (int a = 0; a < 16; ++a) xs[a] = bf16_to_float(X[t * ld + 16 * j + a]);
                for (int a = 0; a < 16; ++a)
                    for (int b = 0; b < 16; ++b) Hj[a * 16 + b] += xs[a] * xs[b];
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Scale sweep ([LH] "算法原理": Q(W,s) = Cast(W/s)*s, the error
// Delta = Q - W, the block-diagonal error E_b(s_b) = Delta_b H_b Delta_b^T
// with H_b = X_b X_b^T of size 16x16, and the exhaustive sweep of the 126
// positive non-zero FP8 E4M3 scales per block; "Local-Hessian 是什么": the
// same 126-candidate sweep as the MSE method).
//
// For one block w[16] (FP32 values) with global scale g:
//   s_c  = fp32(v(c) * g)                    c = 1 .. 126
//   u_i  = fp32(w_i / s_c)                   IEEE FP32 division (Cast(W/s))
//   q_i  = E2M1_RNE_sat(u_i)                 (q_i = 0 when s_c == 0)
//   dw_i = q_i * s_c - w_i                   exact in double
//   E(c) = sum_a sum_b dw_a H_ab dw_b        double
// ---------------------------------------------------------------------------

// Error of one candidate code for one block; H256 is the block's 16x16 H.
double oracle_candidate_error(const float* w16, float g, int code, const double* H256) {
    const float s = oracle_candidate_scale(code, g);
    double dw[16];
    for (int i = 0; i < 16; ++i) {
        float q = 0.0f;
        if (s != 0.0f) {
            const float u = w16[i] / s;
            q = oracle_e2m1_rne(u);
        }
        dw[i] = (double)q * (double)s - (double)w16[i];
    }
    double E = 0.0;
    for (int a = 0; a < 16; ++a)
        for (int b = 0; b < 16; ++b) E += dw[a] * H256[a * 16 + b] * dw[b];
    return E;
}

// All 126 candidate errors of one block: err[c-1] = E(c).
void oracle_block_errors(const float* w16, float g, const double* H256, double* err126) {
    for (int c = 1; c <= 126; ++c) err126[c - 1] = oracle_candidate_error(w16, g, c, H256);
}

// Per-block argmin. Codes are scanned in ascending order with a strict '<',
// so the lowest code wins exact ties. Returns the code; writes the amax
// fp32(6 * s_c*) and the minimum error.
int oracle_block_argmin(const float* w16, float g, const double* H256, float* amax_out,
                        double* err_out) {
    int best = 1;
    double best_e = oracle_candidate_error(w16, g, 1, H256);
    for (int c = 2; c <= 126; ++c) {
        const double e = oracle_candidate_error(w16, g, c, H256);
        if (e < best_e) { best_e = e; best = c; }
    }
    if (amax_out) *amax_out = 6.0f * oracle_candidate_scale(best, g);
    if (err_out) *err_out = best_e;
    return best;
}

// Full sweep. W: FP32 values [n_mats][c_out][ld] (the caller widens bf16
// exactly). global_amax: [n_mats]. H: [n_mats][c_in/16][16][16] double.
// Outputs [n_mats][c_out][c_in/16]: code (u8), amax (f32), min error (f64,
// may be null).
void oracle_sweep(const float* W, int64_t n_mats, int64_t c_out, int64_t c_in, int64_t ld,
                  const float* global_amax, const double* H, uint8_t* code, float* amax,
                  double* err) {
    const int64_t J = c_in / 16;
    for (int64_t m = 0; m < n_mats; ++m) {
        const float g = oracle_global_scale(global_amax[m]);
        for (int64_t r = 0; r < c_out; ++r)
            for (int64_t j = 0; j < J; ++j) {
                const int64_t o = (m * c_out + r) * J + j;
                double e;
                float a;
                const int c = oracle_block_argmin(W + (m * c_out + r) * ld + 16 * j, g,
                                                  H + (m * J + j) * 256, &a, &e);
                code[o] = (uint8_t)c;
                amax[o] = a;
                if (err) err[o] = e;
            }
    }
}

// Sweep of an arbitrary list of blocks (mat, row, col) — the same arithmetic
// as oracle_sweep, for sampled parity checks at full sizes.
void oracle_sweep_blocks(const float* W, int64_t c_out, int64_t c_in, int64_t ld,
                         const float* global_amax, const double* H, const int64_t* mats,
                         const int64_t* rows, const int64_t* cols, int64_t n, uint8_t* code,
                         float* amax, double* err) {
    const int64_t J = c_in / 16;
    for (int64_t i = 0; i < n; ++i) {
        const int64_t m = mats[i], r = rows[i], j = cols[i];
        const float g = oracle_global_scale(global_amax[m]);
        double e;
        float a;
        code[i] = (uint8_t)oracle_block_argmin(W + (m * c_out + r) * ld + 16 * j, g,
                                               H + (m * J + j) * 256, &a, &e);
        amax[i] = a;
        if (err) err[i] = e;
    }
}

// ---------------------------------------------------------------------------
// Fake quantisation with chosen codes ([LH] "算法原理": Q(W,s) = Cast(W/s)*s).
// out = fp32(q * s) per element, q = E2M1_RNE_sat(fp32(w / s)), s = fp32(v(code) * g).
// Output either FP32 values or bf16 bits (RNE of the FP32 product).
// ---------------------------------------------------------------------------
static float fake_quant_one(float w, float s) {
    if (s == 0.0f) return 0.0f * w;  // keeps the sign of w: +-0
    const float q = oracle_e2m1_rne(w / s);
    return q * s;
}

void oracle_fake_quant_f32(const float* W, int64_t n_mats, int64_t c_out, int64_t c_in, int64_t ld,
                           const float* global_amax, const uint8_t* codes, float* out) {
    const int64_t J = c_in / 16;
    for (int64_t m = 0; m < n_mats; ++m) {
        const float g = oracle_global_scale(global_amax[m]);
        for (int64_t r = 0; r < c_out; ++r)
            for (int64_t c = 0; c < c_in; ++c) {
                const int code = codes[(m * c_out + r) * J + c / 16];
                const float s = oracle_candidate_scale(code, g);
                out[(m * c_out + r) * c_in + c] = fake_quant_one(W[(m * c_out + r) * ld + c], s);
            }
    }
}

void oracle_fake_quant_bf16(const float* W, int64_t n_mats, int64_t c_out, int64_t c_in, int64_t ld,
                            const float* global_amax, const uint8_t* codes, uint16_t* out) {
    const int64_t J = c_in / 16;
    for (int64_t m = 0; m < n_mats; ++m) {
        const float g = oracle_global_scale(global_amax[m]);
        for (int64_t r = 0; r < c_out; ++r)
            for (int64_t c = 0; c < c_in; ++c) {
                const int code = codes[(m * c_out + r) * J + c / 16];
                const float s = oracle_candidate_scale(code, g);
                out[(m * c_out + r) * c_in + c] =
                    oracle_float_to_bf16(fake_quant_one(W[(m * c_out + r) * ld + c], s));
            }
    }
}

// ---------------------------------------------------------------------------
// Packed NVFP4 export (the checkpoint form of the same quantisation; the pages
// describe NVFP4 as a two-level scale: E2M1 data with an E4M3 block scale on
// top of the FP32 global scale). Readings (the pages give no bit layout): each
// weight is the 4-bit OCP E2M1 code of q (1 sign bit, 2 exponent bits with
// bias 1, 1 mantissa bit; exponent field 0 is subnormal: value m * 0.5), two
// per byte with the even column in the low nibble; the block scale byte is
// the E4M3 code; the global scale is g. Decoding gives
// fp32(e2m1(nibble) * fp32(v(byte) * g)), the fake-quantised value.
// ---------------------------------------------------------------------------
static unsigned e2m1_code(float q) {
    const unsigned sign = std::signbit(q) ? 1u : 0u;
    const double a = std::fabs((double)q);
    unsigned e, m;
    if (a < 1.0) {  // subnormal: 0 or 0.5
        e = 0;
        m = (unsigned)(a / 0.5);
    } else {        // normal: a = 2^(e-1) * (1 + m/2)
        e = (unsigned)std::floor(std::log2(a)) + 1u;
        m = (unsigned)((a / std::ldexp(1.0, (int)e - 1) - 1.0) * 2.0);
    }
    return (sign << 3) | (e << 1) | m;
}

void oracle_pack_nvfp4(const float* W, int64_t n_mats, int64_t c_out, int64_t c_in, int64_t ld,
                       const float* global_amax, const uint8_t* codes, uint8_t* packed, uint8_t* scales,
                       float* gscale) {
    const int64_t J = c_in / 16;
    for (int64_t m = 0; m < n_mats; ++m) {
        const float g = oracle_global_scale(global_amax[m]);
        gscale[m] = g;
        for (int64_t r = 0; r < c_out; ++r) {
            for (int64_t j = 0; j < J; ++j) scales[(m * c_out + r) * J + j] = codes[(m * c_out + r) * J + j];
            for (int64_t c = 0; c < c_in; c += 2) {
                unsigned nib[2];
                for (int h = 0; h < 2; ++h) {
                    const int code = codes[(m * c_out + r) * J + (c + h) / 16];
                    const float s = oracle_candidate_scale(code, g);
                    const float w = W[(m * c_out + r) * ld + c + h];
                    const float q = (s == 0.0f) ? 0.0f * w : oracle_e2m1_rne(w / s);
                    nib[h] = e2m1_code(q);
                }
                packed[(m * c_out + r) * (c_in / 2) + c / 2] = (uint8_t)(nib[0] | (nib[1] << 4));
            }
        }
    }
}

// ---------------------------------------------------------------------------
// Baseline block scalers ([LH] "Local-Hessian 是什么": max scaling takes the
// block scale from the largest |w| of the 16 weights so they fall inside the
// E2M1 range; the MSE method sweeps all 126 codes on the weight error; the
// four-over-six method picks one of two candidate scales by the in-block
// error). Readings (the pages give no formulas):
//   max:          code = E4M3_RNE_sat(fp32(fp32(amax_b / 6) / g)), at least 1;
//   four-over-six: the codes of amax_b / 6 and amax_b / 4 the same way; keep the
//                 one with the smaller sum of dw^2 (FP64), the lower code on ties;
//   MSE:          the 126-code sweep with H = I (oracle_sweep with identity H).
// ---------------------------------------------------------------------------

// E4M3 code of x >= 0, round to nearest (ties to the even code), saturating at
// 448 (0x7E); written as a search over the 127 non-negative finite codes.
int oracle_e4m3_rne(float x) {
    const double v = (double)x;
    if (!(v > 0.0)) return 0;
    if (v >= 448.0) return 0x7E;
    int best = 0;
    double bd = std::fabs(v - oracle_e4m3_value(0));
    for (int c = 1; c <= 0x7E; ++c) {
        const double d = std::fabs(v - oracle_e4m3_value(c));
        if (d < bd || (d == bd && (c & 1) == 0)) { bd = d; best = c; }
    }
    return best;
}

static double weight_error(const float* w, float g, int code) {
    const float s = oracle_candidate_scale(code, g);
    double e = 0.0;
    for (int i = 0; i < 16; ++i) {
        const float q = (s != 0.0f) ? oracle_e2m1_rne(w[i] / s) : 0.0f;
        const double d = (double)q * (double)s - (double)w[i];
        e += d * d;
    }
    return e;
}

// method 0: max scaling; 1: four-over-six.
void oracle_baseline_scales(const float* W, int64_t n_mats, int64_t c_out, int64_t c_in, int64_t ld,
                            const float* global_amax, int method, uint8_t* code_out, float* amax_out) {
    const int64_t J = c_in / 16;
    for (int64_t m = 0; m < n_mats; ++m) {
        const float g = oracle_global_scale(global_amax[m]);
        for (int64_t r = 0; r < c_out; ++r)
            for (int64_t j = 0; j < J; ++j) {
                const float* w = W + (m * c_out + r) * ld + 16 * j;
                float a = 0.0f;
                for (int i = 0; i < 16; ++i) a = std::fmax(a, std::fabs(w[i]));
                auto code_for = [&](float d) {
                    if (g == 0.0f) return 1;  // every scale is 0
                    const int c = oracle_e4m3_rne((a / d) / g);
                    return c < 1 ? 1 : c;
                };
                int c = code_for(6.0f);
                if (method == 1) {
                    const int c4 = code_for(4.0f);
                    if (c4 != c) {
                        const double e6 = weight_error(w, g, c), e4 = weight_error(w, g, c4);
                        if (e4 < e6 || (e4 == e6 && c4 < c)) c = c4;
                    }
                }
                code_out[(m * c_out + r) * J + j] = (uint8_t)c;
                amax_out[(m * c_out + r) * J + j] = 6.0f * oracle_candidate_scale(c, g);
            }
    }
}

// ---------------------------------------------------------------------------
// Amax multiplier search ([LH] "入口 API 与校准流程": step_size 0.1,
// start_multiplier 0.25, stop_multiplier 4.0 are the amax search of the
// calibration when the FP8 scale sweep is switched off). Reading: multipliers
// m_k = fp32(start + step * k) for k < n_mult (the stop excluded: 38 values by
// default); candidate k is the block scale of the amax m_k * amax_b, rounded as
// in max scaling: code_k = E4M3_RNE_sat(fp32(fp32(fp32(m_k * amax_b) / 6) / g)),
// at least 1; the block keeps the candidate code with the smallest
// E = dw^T H dw (FP64, as in the sweep), the lowest code on ties.
// ---------------------------------------------------------------------------
void oracle_amax_search(const float* W, int64_t n_mats, int64_t c_out, int64_t c_in, int64_t ld,
                        const float* global_amax, const double* H, double start, double step, int64_t n_mult,
                        uint8_t* code_out, float* amax_out, double* err_out) {
    const int64_t J = c_in / 16;
    for (int64_t m = 0; m < n_mats; ++m) {
        const float g = oracle_global_scale(global_amax[m]);
        for (int64_t r = 0; r < c_out; ++r)
            for (int64_t j = 0; j < J; ++j) {
                const float* w = W + (m * c_out + r) * ld + 16 * j;
                const double* Hj = H + (m * J + j) * 256;
                float a = 0.0f;
                for (int i = 0; i < 16; ++i) a = std::fmax(a, std::fabs(w[i]));
                int best = 0;
                double be = 0.0;
                for (int64_t k = 0; k < n_mult; ++k) {
                    int c = 1;
                    if (g != 0.0f) {
                        const float mk = (float)(start + step * (double)k);
                        c = oracle_e4m3_rne(((mk * a) / 6.0f) / g);
                        if (c < 1) c = 1;
                    }
                    const double e = oracle_candidate_error(w, g, c, Hj);
                    if (best == 0 || e < be || (e == be && c < best)) { best = c; be = e; }
                }
                code_out[(m * c_out + r) * J + j] = (uint8_t)best;
                amax_out[(m * c_out + r) * J + j] = 6.0f * oracle_candidate_scale(best, g);
                err_out[(m * c_out + r) * J + j] = be;
            }
    }
}

}  // extern "C"
