// FP8 block-scale sweep: for every NVFP4 block, all 126 E4M3 candidate
// scales, keep the argmin of dw^T H dw.
//
// Method: "NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4 逐块
// 权重缩放算法实战指南" (xxmr.cn/news/266017), section "算法原理": the
// block-diagonal error E_b(s_b) = Delta_b (X_b X_b^T) Delta_b^T, swept over the
// 126 FP8 candidates per block; kernel contract: weights [N_BLOCKS, 16] in
// (cout, cin/16) order, global FP32 amax, H [cin/16, 16, 16], per-block best
// amax out.
//
// Design (B200, FP32 CUDA cores):
//  * One thread owns one block (row r, block column j). A CTA of 128 threads
//    takes a tile of 1024 rows of one block column (the last wave of tiles is
//    cut into 512- and 256-row pieces so the launch drains quickly), stages H_j once in
//    shared memory (read by broadcast), sorts the tile's rows by the largest
//    |w| over the heavy channels (to 1/16 of an octave), and hands out 32-row
//    chunks of the sorted order to its four warps.
//  * Candidate scales come in 8 mantissa classes (1 + f/8) * 2^x. Within a
//    class consecutive codes double the scale exactly, so fp32(w / s_c) is
//    fp32(w / s_c0) scaled by a power of two: 16 correctly rounded quotients
//    per class replace 16 per candidate, and each candidate rounds them onto
//    the E2M1 grid scaled by 2^k (exact: the quotients times 2^-k through the
//    hardware E2M1 conversions, round to nearest even with saturation).
//  * Per class a warp walks up and down from its max-scaling step. A lower
//    bound mu * sum_a H_aa dw_a^2 <= E skips the form for candidates that
//    cannot win, and class-wide bounds end each direction early; mu comes from
//    shifted Cholesky tests of the normalised H (per CTA, or once per column by
//    a first kernel when the caller gives a workspace).
//  * The survivors' E(c) is evaluated in FP32 with the symmetric form (136
//    FMA). Its error is at most rho * E with rho = 48 u nu / mu (nu bounds the
//    largest eigenvalue of |normalised H|), or an absolute bound when mu = 0.
//    When only the runner-up is within that bound of the best, the lane
//    compares the two in FP64; when a third candidate is too, the whole warp
//    re-sweeps the block in FP64. The result is the exact argmin (up to FP64
//    rounding), lowest code on ties.
#include <cmath>

#include "common.cuh"
#include "quant.cuh"
#include <cuda_fp16.h>

// Measurement build only (-DLH_SWEEP_COUNTERS=1): the work the walk does, summed
// over a launch; lh_debug_sweep_counts reads and clears it. Off in the library.
#ifndef LH_SWEEP_COUNTERS
#define LH_SWEEP_COUNTERS 0
#endif
#if LH_SWEEP_COUNTERS
// [0] warp chunks, [1] blocks, [2] candidates quantised (per warp), [3] full forms (per
// warp), [4] forms a lane needed (its bound did not exclude the candidate), [5] class-wide
// bound tests, [6] blocks re-swept in FP64, [7] classes walked (per warp), [8] blocks whose
// best two were compared in FP64
__device__ unsigned long long lh_sweep_counts[9];
#endif

#ifndef LH_SWEEP_UREGS
#define LH_SWEEP_UREGS false  // form coefficients read from shared memory (more warps per SM)
#endif

namespace lh {
namespace {

constexpr int kThreads = 128;        // threads per CTA (one block per thread at a time)
constexpr int kRowsPerThread = 8;    // rows each thread walks; a tile is 1024 rows of one block column

// packed upper-triangle index of (a, b), a <= b
__host__ __device__ constexpr int tri(int a, int b) { return a * 16 - (a * (a - 1)) / 2 + (b - a); }

template <typename T>
__device__ __forceinline__ void load_block(const T* p, float (&w)[16]);

template <>
__device__ __forceinline__ void load_block<uint16_t>(const uint16_t* p, float (&w)[16]) {
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
__device__ __forceinline__ void load_block<float>(const float* p, float (&w)[16]) {
    const float4* q = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 t = __ldg(q + i);
        w[4 * i] = t.x; w[4 * i + 1] = t.y; w[4 * i + 2] = t.z; w[4 * i + 3] = t.w;
    }
}

// E4M3 code of the value (1 + f/8) * 2^x (f in 0..7, x >= -9), or the
// subnormal code (8 + f) * 2^(x + 6) when x < -6.
__device__ __forceinline__ int class_code(int f, int x) {
    return x >= -6 ? 8 * (x + 7) + f : (8 + f) >> (-6 - x);
}

// Correctly rounded FP32 quotients a / b for positive normal b, two lanes at
// once, from y = RN(1/b) (correctly rounded reciprocal): q = RN(a y) is within
// one ulp of a/b, the remainder a - b q is exact with one FMA, and RN(q + r y)
// is RN(a/b) (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990, Theorem 1; see
// also Muller et al., Handbook of Floating-Point Arithmetic, ch. 4). Valid
// while the remainder a - b q cannot underflow, i.e. for a >= 2^-100 (or a = 0)
// and a normal b; blocks with a smaller non-zero |w| use IEEE division. The
// packed FP32 operations round each lane exactly as the scalar ones; nb = -b.
// Both values rounded to the nearest E2M1 value (ties to even, saturating at +-6),
// by the hardware conversions: to two E2M1 codes, and back through f16x2 (exact).
__device__ __forceinline__ float2 e2m1x2_round(float2 v) {
    uint32_t h2;
    asm("{\n .reg .b8 t;\n cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n cvt.rn.f16x2.e2m1x2 %0, t;\n}"
        : "=r"(h2) : "f"(v.y), "f"(v.x));
    const __half2 h = *reinterpret_cast<const __half2*>(&h2);
    return __half22float2(h);
}
__device__ __forceinline__ float2 div_by_recip2(float2 a, float2 nb, float2 y) {
    const float2 q = __fmul2_rn(a, y);
    const float2 r = __ffma2_rn(q, nb, a);
    return __ffma2_rn(r, y, q);
}

// IEEE quotients w_i / s0 for blocks holding a tiny non-zero weight (rare;
// kept out of line so the hot loop stays small).
__device__ __forceinline__ void quotients_ieee(const float (&w)[16], float s0, float2 (&u)[8]) {
#pragma unroll
    for (int p = 0; p < 8; ++p) u[p] = make_float2(__fdiv_rn(w[2 * p], s0), __fdiv_rn(w[2 * p + 1], s0));
}

// FP64 error of candidate code c for block w (definition order of the method:
// s = fp32(v(c) g), q = E2M1(fp32(w/s)), dw = q s - w exact, E = dw^T H dw),
// the form taken over the packed upper triangle Us (H_aa, H_ab + H_ba in FP64).
// w is read from shared memory, so no caller keeps its weights in local memory.
__device__ __noinline__ double candidate_error_f64(const float* w, float g, int c, const double* Us) {
    const float s = __fmul_rn(e4m3_value(c), g);
    const double sd = (double)s;
    double dw[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float q = (s != 0.0f) ? e2m1_rne(__fdiv_rn(w[i], s)) : 0.0f;
        dw[i] = fma((double)q, sd, -(double)w[i]);  // q s - w: q s has at most 27 significant bits
    }
    double E = 0.0;
#pragma unroll 1
    for (int a = 0; a < 16; ++a) {
        double t = 0.0;
#pragma unroll
        for (int b = 15; b >= a; --b) t = fma(Us[tri(a, b)], dw[b], t);
        E = fma(dw[a], t, E);
    }
    return E;
}

// Pair (U[a][2i], U[a][2i+1]) of row a of the symmetric form, in the order
// the form consumes them: rows a = 0..15, for row a the column pairs
// i = ceil(a/2)..7 (for even a the first pair starts on the diagonal; for odd
// a the diagonal is kept apart in Ud[a/2]). Every row's run of pairs starts
// on a 16-byte boundary so two pairs come in one 128-bit shared load.
__host__ __device__ constexpr int pair_first(int a) { return (a + 1) / 2; }
__host__ __device__ constexpr int pair_count(int a) { return 8 - pair_first(a); }
__host__ __device__ constexpr int pair_offset(int a) {
    int o = 0;
    for (int r = 0; r < a; ++r) o += 2 * ((pair_count(r) + 1) / 2);
    return o;
}
constexpr int kPairSlots = pair_offset(16);
static_assert(kPairSlots == 72, "72 padded pair slots");

constexpr int kTileRows = kThreads * kRowsPerThread;  // rows of one CTA, walked in sorted order

constexpr int kSortBuckets = 512;

// Work units of one launch, in launch order: the tiles (kTileRows rows of one block
// column, column-major over (m, j)); of the last wave of tiles, the first three
// quarters are cut into halves and the rest into quarters. CTAs start in launch
// order, so the pieces run last and the launch drains in a fraction of a tile's time.
// Large tiles sort more rows together (the warps of a tile agree more on where their
// walks start and stop) and spread the per-CTA set-up over more rows; pieces of
// fewer rows walk more slowly per row, so only the very end is cut finest.
struct Units {
    int64_t tiles_per_col;  // ceil(c_out / kTileRows)
    int64_t n_tiles;        // tiles_per_col * J * n_mats
    int64_t n_split;        // tiles cut into halves
    int64_t n_quart;        // tiles after those, cut into quarters (the last ones)
};

__device__ __forceinline__ void unit_of(const Units& U, int64_t J, int64_t c_out, int64_t u, int64_t& m, int64_t& j,
                                        int64_t& row0, int& nrows) {
    const int64_t whole = U.n_tiles - U.n_split - U.n_quart;
    int64_t t, r0, rn;
    if (u < whole) {
        t = u;
        r0 = 0;
        rn = kTileRows;
    } else if (u < whole + 2 * U.n_split) {
        const int64_t v = u - whole;
        t = whole + v / 2;
        r0 = (v % 2) * (kTileRows / 2);
        rn = kTileRows / 2;
    } else {
        const int64_t v = u - whole - 2 * U.n_split;
        t = whole + U.n_split + v / 4;
        r0 = (v % 4) * (kTileRows / 4);
        rn = kTileRows / 4;
    }
    const int64_t col = t / U.tiles_per_col;
    m = col / J;
    j = col - m * J;
    row0 = (t - col * U.tiles_per_col) * kTileRows + r0;
    const int64_t left = c_out - row0;
    nrows = left <= 0 ? 0 : (int)(left < rn ? left : rn);
}

// The pruning bounds of one block column (mu, nu below), computed once per column by
// sweep_bounds_kernel when the caller gives a workspace.
struct ColBounds {
    float mu, nu, pad0, pad1;
};
static_assert(sizeof(ColBounds) == 16, "16-byte column records");

struct SweepShared {
    // (bits of the heavy channels' max |w|) << 32 | local row; after the sort, 16 weights per
    // thread for the FP64 paths (kTileRows * 8 bytes = kThreads * 16 floats)
    unsigned long long key[kTileRows];
    unsigned long long order[kTileRows];  // the same, grouped by sort bucket
    uint32_t hist[kSortBuckets];
    double Us[136];                     // H_aa, H_ab + H_ba (a < b) in FP64, packed upper triangle
    float2 Up[kPairSlots];  // U pairs (U_ab = H_aa on the diagonal, H_ab + H_ba above it)
    float Ud[8];            // diagonals of the odd rows
    float Ua[136];          // |U| packed upper triangle, for the error bound
    float Hf[256];          // H as given, for the FP64 re-sweep
    __align__(16) float chol[8][32];  // the Cholesky tests' columns, per half-warp (column bounds)
    float2 dg[8];           // diagonal of H, pairs (for the lower bound)
    int pd[16];             // results of the shifted positive-definiteness tests
    uint32_t allow[4][kThreads];  // amax search: the codes each thread's current block may take
    float mu;               // mu <= lambda_min(D^-1/2 H D^-1/2), D = diag(H); 0 disables pruning
    float nu;               // nu >= lambda_max(|D^-1/2 H D^-1/2|) (largest absolute row sum)
    int next_chunk;         // next 32-row chunk of the sorted order to hand to a warp
    unsigned kmax;          // largest sort key of the tile
    // the CTA's unit, read back in the row loop rather than kept in registers
    unsigned long long wcol;  // address of W[m][tile0][16 j]
    long long ocol;           // index of output (m, tile0, j)
    int nrows;
};

// Is C - mu I positive definite? FP32 Cholesky by one half-warp, in registers:
// lane i (of 16) owns row i of C; the pivot of column k comes by a shuffle, and
// the multipliers L_bk through `col`, this half-warp's 2 x 16 floats of shared
// memory (one column per step, alternating, so one warp barrier a step suffices),
// read back as 128-bit broadcasts; true when every pivot is positive. Every lane
// of the warp calls it (the warp barriers).
__device__ __forceinline__ bool shifted_pd(const float (&crow)[16], float mu, int i, float* col) {
    float c[16];
#pragma unroll
    for (int b = 0; b < 16; ++b) c[b] = crow[b] - ((b == i) ? mu : 0.0f);
    bool ok = true;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const float d = __shfl_sync(0xFFFFFFFFu, c[k], k, 16);  // pivot, from lane k of this half
        ok = ok && (d > 0.0f);
        const float l = (i > k) ? c[k] * (d > 0.0f ? rsqrtf(d) : 1.0f) : 0.0f;  // L_ik
        float* lk = col + 16 * (k & 1);
        lk[i] = l;
        __syncwarp();
#pragma unroll
        for (int b4 = (k + 1) / 4 * 4; b4 < 16; b4 += 4) {
            const float4 v = *reinterpret_cast<const float4*>(lk + b4);
            const float lb[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (b4 + u > k) c[b4 + u] = __fmaf_rn(-l, lb[u], c[b4 + u]);
        }
    }
    return ok;
}

__device__ __forceinline__ float4 lds128(const void* p) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(p))));
    return v;
}

// E = sum_{a<=b} U_ab dw_a dw_b with packed FP32 FMAs: for every row a the
// pair (t.x, t.y) accumulates the even and odd columns b >= a, then
// E += dw_a (t.x + t.y). 64 paired FMAs, 8 products, 16 adds, 16 FMAs.
// Coefficients from registers.
__device__ __forceinline__ float quad_form_regs(const float2 (&dw)[8], const float2 (&Up)[kPairSlots],
                                                const float (&Ud)[8]) {
    float E0 = 0.0f, E1 = 0.0f;  // even and odd rows: two independent chains
#pragma unroll
    for (int a = 0; a < 16; ++a) {
        const float dwa = (a & 1) ? dw[a >> 1].y : dw[a >> 1].x;
        float2 t = (a & 1) ? make_float2(Ud[a >> 1] * dwa, 0.0f) : make_float2(0.0f, 0.0f);
#pragma unroll
        for (int i = pair_first(a); i < 8; ++i) t = __ffma2_rn(Up[pair_offset(a) + i - pair_first(a)], dw[i], t);
        if (a & 1) E1 = fmaf(dwa, t.x + t.y, E1);
        else E0 = fmaf(dwa, t.x + t.y, E0);
    }
    return E0 + E1;
}

// The same form with the coefficients streamed from shared memory on every
// call (volatile 128-bit broadcast loads: the compiler may not keep them).
__device__ __forceinline__ float quad_form_smem(const float2 (&dw)[8], const SweepShared& sm) {
    const float4 d0 = lds128(&sm.Ud[0]), d1 = lds128(&sm.Ud[4]);
    const float ud[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
    float E0 = 0.0f, E1 = 0.0f;  // even and odd rows: two independent chains
#pragma unroll
    for (int a = 0; a < 16; ++a) {
        const float dwa = (a & 1) ? dw[a >> 1].y : dw[a >> 1].x;
        float2 t = (a & 1) ? make_float2(ud[a >> 1] * dwa, 0.0f) : make_float2(0.0f, 0.0f);
#pragma unroll
        for (int i = pair_first(a); i < 8; i += 2) {
            const float4 c = lds128(&sm.Up[pair_offset(a) + i - pair_first(a)]);
            t = __ffma2_rn(make_float2(c.x, c.y), dw[i], t);
            if (i + 1 < 8) t = __ffma2_rn(make_float2(c.z, c.w), dw[i + 1], t);
        }
        if (a & 1) E1 = fmaf(dwa, t.x + t.y, E1);
        else E0 = fmaf(dwa, t.x + t.y, E0);
    }
    return E0 + E1;
}

// mu for the candidate lower bound E >= mu sum_a H_aa dw_a^2: the largest
// shift at which C - mu I passes an FP32 Cholesky test, C = D^-1/2 H_s D^-1/2
// (H_s = (H + H^T) / 2, D = diag(H), rows with H_aa = 0 replaced by identity
// rows). Two rounds of eight shifts (one per half-warp): 0.04 + 0.12 s, then
// nine steps up from the best of those. A completed factorisation is
// backward stable (|dC| <= 17 u |L||L^T| <= 17 u entrywise, so lambda_min(C)
// >= mu - 16 * 17 u, and forming C costs a few ulps more); 2^-14 is
// subtracted to cover it. mu = 0 (no pruning) when H has a zero diagonal
// entry with a non-zero off-diagonal entry in its row or a negative diagonal
// entry, or when mu would fall below 2^-8.
// Every thread of the CTA calls it (it holds __syncthreads); H is in sm.Hf. Sm is the
// sweep's shared state or the bounds kernel's smaller one (Hf, pd, mu, nu).
template <typename Sm>
__device__ __forceinline__ void column_bounds(Sm& sm, int tid) {
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int hl = lane >> 4, i = lane & 15;
    const int slot = 2 * warp + hl;  // 0..7
    const float hii = sm.Hf[i * 17];
    bool psd_rows = hii >= 0.0f;
    if (hii == 0.0f)
        for (int b = 0; b < 16; ++b)
            if (sm.Hf[i * 16 + b] != 0.0f || sm.Hf[b * 16 + i] != 0.0f) psd_rows = false;
    psd_rows = __all_sync(0xFFFFFFFFu, psd_rows);
    const float di = hii > 0.0f ? rsqrtf(hii) : 0.0f;
    float crow[16];
#pragma unroll
    for (int b = 0; b < 16; ++b) {
        const float hbb = sm.Hf[b * 17];
        const float db = __shfl_sync(0xFFFFFFFFu, di, b, 16);
        crow[b] = (hii > 0.0f && hbb > 0.0f) ? (0.5f * (sm.Hf[i * 16 + b] + sm.Hf[b * 16 + i])) * (di * db)
                                             : ((i == b) ? 1.0f : 0.0f);
    }
    // |C| is non-negative and symmetric, so its largest eigenvalue is at most its largest row
    // sum; the entries carry a few ulps of rounding (rsqrt, products), covered by 2^-16
    {
        float rs = 0.0f;
#pragma unroll
        for (int b = 0; b < 16; ++b) rs += fabsf(crow[b]);
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) rs = fmaxf(rs, __shfl_xor_sync(0xFFFFFFFFu, rs, off));
        if (tid == 0) sm.nu = rs * (1.0f + 1.5258789e-5f);
    }
    const float mu1 = 0.04f + 0.12f * (float)slot;
    float* const col = &sm.chol[slot][0];
    const bool ok1 = psd_rows && shifted_pd(crow, mu1, i, col);
    if (i == 0) sm.pd[slot] = ok1;
    __syncthreads();
    float lo = 0.0f;
    for (int q = 0; q < 8; ++q)
        if (sm.pd[q]) lo = fmaxf(lo, 0.04f + 0.12f * (float)q);
    const float step = (lo > 0.0f ? 0.12f : 0.04f) * (1.0f / 9.0f);
    const float mu2 = lo + step * (float)(slot + 1);
    __syncwarp();  // the last step's reads of col are done
    const bool ok2 = psd_rows && shifted_pd(crow, mu2, i, col);
    if (i == 0) sm.pd[8 + slot] = ok2;
    __syncthreads();
    float best = lo;
    for (int q = 0; q < 8; ++q)
        if (sm.pd[8 + q]) best = fmaxf(best, lo + step * (float)(q + 1));
    if (tid == 0) sm.mu = best >= 0.00390625f ? best - 6.1035156e-5f : 0.0f;  // - 2^-14
}

// Channels a with H_aa >= max_b H_bb / 10 (bit a); H is in sm.Hf.
__device__ __forceinline__ unsigned heavy_channels(const SweepShared& sm, int lane) {
    const float hii = sm.Hf[(lane & 15) * 17];
    float dmax = hii;
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) dmax = fmaxf(dmax, __shfl_xor_sync(0xFFFFFFFFu, dmax, off));
    return __ballot_sync(0xFFFFFFFFu, hii >= 0.1f * dmax) & 0xFFFFu;
}

// kMask: the amax multiplier search; each block may only take the codes of the
// amaxes m_k * amax_b, m_k = fp32(m_start + m_step * k), k < n_mult.
template <typename T, bool kURegs, bool kMask>
__global__ void __launch_bounds__(kThreads, kURegs ? 2 : 4)
sweep_kernel(const T* __restrict__ W, int64_t c_out, int64_t J, int64_t ld, int64_t mat_stride,
             const float* __restrict__ gamax, const float* __restrict__ H, float* __restrict__ best_amax,
             uint8_t* __restrict__ best_code, const ColBounds* __restrict__ cb, const Units U, double m_start,
             double m_step, int n_mult) {
    __shared__ __align__(16) SweepShared sm;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    int64_t m, j, tile0;
    int nrows;
    unit_of(U, J, c_out, (int64_t)blockIdx.x, m, j, tile0, nrows);
    if (nrows == 0) return;  // a quarter past the end of a ragged last tile (uniform over the CTA)
    if (tid == 0) {
        sm.wcol = reinterpret_cast<unsigned long long>(W + m * mat_stride + tile0 * ld + 16 * j);
        sm.ocol = (long long)((m * c_out + tile0) * J + j);
        sm.nrows = nrows;
    }

    const float* Hj = H ? H + (m * J + j) * 256 : nullptr;  // no H: the identity (the weight-MSE sweep)
    for (int i = tid; i < 256; i += kThreads) sm.Hf[i] = Hj ? Hj[i] : ((i % 17 == 0) ? 1.0f : 0.0f);
    for (int i = tid; i < kPairSlots; i += kThreads) sm.Up[i] = make_float2(0.0f, 0.0f);
    __syncthreads();
    if (tid < 8) sm.dg[tid] = make_float2(sm.Hf[(2 * tid) * 17], sm.Hf[(2 * tid + 1) * 17]);
    for (int i = tid; i < 256; i += kThreads) {
        const int a = i >> 4, b = i & 15;
        if (b < a) continue;
        const float u = (a == b) ? sm.Hf[i] : __fadd_rn(sm.Hf[i], sm.Hf[b * 16 + a]);  // H_ab + H_ba
        sm.Ua[tri(a, b)] = fabsf(u);
        sm.Us[tri(a, b)] = (a == b) ? (double)sm.Hf[i] : (double)sm.Hf[i] + (double)sm.Hf[b * 16 + a];  // exact
        if ((a & 1) && b == a) {
            sm.Ud[a >> 1] = u;  // odd rows keep their diagonal apart
        } else {
            // column b sits in pair b/2 of row a, as .x (even b) or .y (odd b)
            float* dst = reinterpret_cast<float*>(&sm.Up[pair_offset(a) + (b >> 1) - pair_first(a)]);
            dst[b & 1] = u;
        }
    }
    const unsigned heavy = heavy_channels(sm, lane);
    if (cb == nullptr) column_bounds(sm, tid);  // uniform over the CTA

    // Rows are walked in the order of their largest |w| over the heavy channels
    // (H_aa at least a tenth of the largest; all channels when those weights are
    // zero): the error is dominated by those channels, so their range sets where
    // the optimum lies; each class's walk starts at its max-scaling step. After
    // sorting, the 32 rows of a warp mostly agree on where to start, what to skip
    // and when to stop.
    // counting sort of the tile's rows by a 9-bit key: the octaves below the tile's
    // largest key (up to 30) and the first four mantissa bits of that largest |w|, so
    // rows within 1/16 of each other share a bucket; rows past c_out last
    for (int i = tid; i < kSortBuckets; i += kThreads) sm.hist[i] = 0;
    if (tid == 0) {
        sm.next_chunk = 0;
        sm.kmax = 0u;
    }
    __syncthreads();
    uint32_t kb[kRowsPerThread];
#pragma unroll
    for (int q = 0; q < kRowsPerThread; ++q) {
        const int p = q * kThreads + tid;
        const int64_t r = tile0 + p;
        uint32_t key = 0xFFFFFFFFu;
        if (p < nrows) {
            float wk[16];
            load_block<T>(W + m * mat_stride + r * ld + 16 * j, wk);
            float mx = 0.0f, mh = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                mx = fmaxf(mx, fabsf(wk[i]));
                mh = ((heavy >> i) & 1u) ? fmaxf(mh, fabsf(wk[i])) : mh;
            }
            key = __float_as_uint(mh > 0.0f ? mh : mx);
            atomicMax(&sm.kmax, key);  // non-negative floats order like their bits
        }
        kb[q] = key;
        sm.key[p] = ((unsigned long long)key << 32) | (unsigned)p;
    }
    __syncthreads();
    // buckets, largest keys first
    {
        const uint32_t emax = sm.kmax >> 23;
#pragma unroll
        for (int q = 0; q < kRowsPerThread; ++q) {
            const uint32_t key = kb[q];
            if (key == 0xFFFFFFFFu) {
                kb[q] = kSortBuckets - 1;
            } else {
                const uint32_t d = min(emax - min(key >> 23, emax), 30u);
                kb[q] = d * 16u + (15u - ((key >> 19) & 15u));
            }
            atomicAdd(&sm.hist[kb[q]], 1u);
        }
    }
    __syncthreads();
    if (tid < 32) {  // exclusive scan of the histogram by one warp
        uint32_t v[kSortBuckets / 32], run = 0;
#pragma unroll
        for (int i = 0; i < kSortBuckets / 32; ++i) { v[i] = sm.hist[tid * (kSortBuckets / 32) + i]; run += v[i]; }
        uint32_t incl = run;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
            if (tid >= off) incl += o;
        }
        uint32_t pos = incl - run;
#pragma unroll
        for (int i = 0; i < kSortBuckets / 32; ++i) { sm.hist[tid * (kSortBuckets / 32) + i] = pos; pos += v[i]; }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < kRowsPerThread; ++q) {
        const uint32_t pos = atomicAdd(&sm.hist[kb[q]], 1u);
        sm.order[pos] = sm.key[q * kThreads + tid];
    }
    __syncthreads();

    if (cb != nullptr) {
        // the bounds kernel before this one
        if (tid == 0) {
            const ColBounds c = cb[m * J + j];
            sm.mu = c.mu;
            sm.nu = c.nu;
        }
        __syncthreads();
    }

    // form coefficients: copied into registers, or read from shared memory (broadcast)
    float2 Ur[kPairSlots];
    float Udr[8];
    if constexpr (kURegs) {
#pragma unroll
        for (int i = 0; i < kPairSlots; ++i) Ur[i] = sm.Up[i];
#pragma unroll
        for (int i = 0; i < 8; ++i) Udr[i] = sm.Ud[i];
    }
    auto form = [&](const float2 (&d)[8]) -> float {
        if constexpr (kURegs) return quad_form_regs(d, Ur, Udr);
        else return quad_form_smem(d, sm);
    };

    const float A = gamax[m];  // m is not needed in the row loop
    const float g = __fdiv_rn(A, 2688.0f);
    // Power-of-two relation between the candidates of a class holds while
    // every candidate scale is a normal FP32 number: g * 2^-9 >= 2^-126.
    const bool fast = (g >= 1.2037062e-35f) && (g <= 1.0e30f);  // g >= 2^-116

    for (;;) {
        // warps take 32-row chunks of the sorted order as they finish the last one
        int chunk = 0;
        if (lane == 0) chunk = atomicAdd(&sm.next_chunk, 1);
        chunk = __shfl_sync(0xFFFFFFFFu, chunk, 0);
        if (chunk >= kTileRows / 32) break;
        const int pos = chunk * 32 + lane;
        const int lp = (int)(sm.order[pos] & 0xFFFFFFFFu);
        const bool active = lp < *reinterpret_cast<volatile int*>(&sm.nrows);
        if (__all_sync(0xFFFFFFFFu, !active)) break;  // rows past the unit sort last: so are all later chunks
        float w[16];
        if (active)
            load_block<T>(reinterpret_cast<const T*>(*reinterpret_cast<volatile unsigned long long*>(&sm.wcol)) +
                              (int64_t)lp * ld, w);
        else {
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = 0.0f;
        }

        const float hw = active ? __uint_as_float((uint32_t)(sm.order[pos] >> 32)) : 0.0f;  // the sort key
        if constexpr (kMask) {
            // the candidate codes of this block: max-scaling codes of m_k * amax_b
            uint32_t al[4] = {0u, 0u, 0u, 0u};
            float ab = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) ab = fmaxf(ab, fabsf(w[i]));
            for (int k = 0; k < n_mult; ++k) {
                int c = 1;
                if (g != 0.0f) {
                    const float mk = __double2float_rn(__dadd_rn(m_start, __dmul_rn(m_step, (double)k)));
                    c = max(1, e4m3_rne_code(__fdiv_rn(__fdiv_rn(__fmul_rn(mk, ab), 6.0f), g)));
                }
                al[c >> 5] |= 1u << (c & 31);
            }
            __syncwarp();  // the warp's earlier reads of the last block's codes are done
#pragma unroll
            for (int q = 0; q < 4; ++q) sm.allow[q][tid] = al[q];
            __syncwarp();
        }
        auto allowed = [&](int code, int t) -> bool {
            if constexpr (kMask) return (sm.allow[code >> 5][t] >> (code & 31)) & 1u;
            else return true;
        };
#if LH_SWEEP_COUNTERS
        unsigned cnt_cand = 0, cnt_form = 0, cnt_need = 0, cnt_below = 0, cnt_class = 0;
#endif
        float best_e = __int_as_float(0x7F800000), second_e = __int_as_float(0x7F800000);
        float third_e = __int_as_float(0x7F800000);  // the smallest FP32 error after the best two
        int best_fk = -1;    // 32 f + k of the best candidate (class f, step k); the code is formed at the end
        int second_fk = -1;  // the same for the runner-up
        bool flag = !fast;   // the whole block is re-swept in FP64
        bool pair = false;   // only the best two are within the FP32 error bound: they are compared in FP64
        if (g == 0.0f) flag = false;  // every s_c is 0: q = 0, all errors equal, code 1

        if (fast) {
            // With mu > 0 the FP32 error of the form becomes relative. With z_a = sqrt(H_aa) dw_a
            // and C = D^-1/2 H_s D^-1/2, T = sum |U_ab| |dw_a| |dw_b| = |z|^T |C| |z| <= nu |z|^2
            // and E = z^T C z >= mu |z|^2, so T <= (nu / mu) E and |E32 - E| <= rho E with
            // rho = 48 u nu / mu (nu <= 16; near 1 for weakly correlated channels), far tighter
            // than the Tw bound below for the candidates near the optimum. Thresholds then
            // follow from E in [E32 / (1 + rho), E32 / (1 - rho)]; closed forms are within 2u.
            const bool rel = sm.mu > 0.0f;
            const float rho = rel ? fminf(48.0f * 5.9604645e-8f * sm.nu / sm.mu * 1.001f, 0.25f) : 0.0f;
            const float up_fac = 1.0f / (1.0f - rho) * (1.0f + 4.0f * 5.9604645e-8f);  // E* <= E32 * up_fac
            // mu rounded down, less 32 u for the rounding of dw and of the bound's sum
            const float mu_lb = sm.mu * (1.0f - 32.0f * 5.9604645e-8f);
            // Without mu: Tw = sum_{a<=b} |U_ab| |w_a| |w_b| bounds sum |U_ab| |dw_a| |dw_b| for
            // every candidate, and |E32 - E| <= 30 u T <= 30 u Tw (48 u leaves slack for the
            // rounding of Tw itself).
            float margin = 0.0f;
            if (!rel) {
                float Tw = 0.0f;
#pragma unroll
                for (int a = 0; a < 16; ++a) {
                    float t = sm.Ua[tri(a, a)] * fabsf(w[a]);
#pragma unroll
                    for (int b = a + 1; b < 16; ++b) t = fmaf(sm.Ua[tri(a, b)], fabsf(w[b]), t);
                    Tw = fmaf(fabsf(w[a]), t, Tw);
                }
                margin = 2.0f * (48.0f * 5.9604645e-8f) * Tw;
            }
            float2 w2[8];
#pragma unroll
            for (int p = 0; p < 8; ++p) w2[p] = make_float2(w[2 * p], w[2 * p + 1]);
            // the upward bound loses at most 2^-22 H_aa w_a^2 per weight to the rounding of u;
            // 2^-20 mu sum_a H_aa w_a^2 covers it with room for the rounding of the sum
            float tail_corr;
            {
                float2 sw = make_float2(0.0f, 0.0f);
#pragma unroll
                for (int p = 0; p < 8; p += 2) {
                    const float4 d4 = lds128(&sm.dg[p]);
                    sw = __ffma2_rn(__fmul2_rn(w2[p], w2[p]), make_float2(d4.x, d4.y), sw);
                    sw = __ffma2_rn(__fmul2_rn(w2[p + 1], w2[p + 1]), make_float2(d4.z, d4.w), sw);
                }
                tail_corr = (sw.x + sw.y) * (sm.mu * 9.5367432e-7f);  // 2^-20 mu
            }
            // the reciprocal-based quotient needs every non-zero |w| >= 2^-100
            bool tiny_w = false;
#pragma unroll
            for (int i = 0; i < 16; ++i) tiny_w |= (w[i] != 0.0f) && (fabsf(w[i]) < 7.888609e-31f);

#pragma unroll 1
            for (int f = 0; f < 8; ++f) {
#if LH_SWEEP_COUNTERS
                ++cnt_class;
#endif
                const int tz = (f == 0) ? 3 : (f == 4) ? 2 : (f == 2 || f == 6) ? 1 : 0;
                const int x0 = -6 - tz;                  // smallest exponent of the class
                const int n = (f == 7 ? 7 : 8) - x0 + 1;  // codes in the class
                const float v0 = (float)(8 + f) * __int_as_float((x0 - 3 + 127) << 23);  // (1 + f/8) 2^x0
                const float s0 = __fmul_rn(v0, g);
                // signed quotients u = w / s0; candidate k of the class has the scale 2^k s0
                float2 u[8];
                float umax = 0.0f;  // max |u|
                if (tiny_w) {
                    quotients_ieee(w, s0, u);
                } else {
                    const float rs0 = __frcp_rn(s0);
                    const float2 ns02 = make_float2(-s0, -s0), rs02 = make_float2(rs0, rs0);
#pragma unroll
                    for (int p = 0; p < 8; ++p) u[p] = div_by_recip2(w2[p], ns02, rs02);
                }
#pragma unroll
                for (int p = 0; p < 8; ++p) umax = fmaxf(umax, fmaxf(fabsf(u[p].x), fabsf(u[p].y)));
                const float2 ns0 = make_float2(-s0, -s0);
                // One candidate; returns true (upward walk only) when every lane proves that no
                // later candidate of the upward walk can beat the incumbent.
                auto candidate = [&](int k, bool up) -> bool {
#if LH_SWEEP_COUNTERS
                    ++cnt_cand;
#endif
                    const float lim = __int_as_float(((129 + k) << 23) | 0x400000);  // 6 * 2^k
                    const unsigned mlo = ((unsigned)(127 + k) << 23) + 0x0B400000u;
                    float E;
                    bool stop = false, done = false;
                    if (!rel) {
                        // no pruning here, so whole-block shortcuts pay: every non-zero weight
                        // saturates (q = +-6) iff min |u| > 5 * 2^k; every q is 0 iff max |u| <= 2^k / 4
                        // (ties 5 -> 4 and 1/4 -> 0 round to even)
                        float umin = __int_as_float(0x7F800000);
#pragma unroll
                        for (int p = 0; p < 8; ++p) {
                            umin = (w2[p].x != 0.0f) ? fminf(umin, fabsf(u[p].x)) : umin;
                            umin = (w2[p].y != 0.0f) ? fminf(umin, fabsf(u[p].y)) : umin;
                        }
                        const bool sat = umin > __int_as_float(((129 + k) << 23) | 0x200000);  // 5 * 2^k
                        const bool zero = umax <= __int_as_float((125 + k) << 23);              // 2^k / 4
                        const bool all_sat = __all_sync(0xFFFFFFFFu, sat);
                        if (all_sat || __all_sync(0xFFFFFFFFu, zero)) {
                            // closed forms in FP64 with sigma = sign(w) (0 where w = 0): a saturated
                            // candidate has dw = 6 s_c sigma - w, so E = 36 s^2 sHs - 6 s (sHw + wHs) + wHw;
                            // an all-zero candidate has dw = -w, so E = wHw
                            double sHs = 0.0, sHw_wHs = 0.0, wHw = 0.0;
                            // the weights go through this thread's slot in shared memory (the loops
                            // index them at run time)
                            float* const wt = reinterpret_cast<float*>(sm.key) + 16 * tid;
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                *reinterpret_cast<float4*>(wt + 4 * i) =
                                    make_float4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
#pragma unroll 1
                            for (int a = 0; a < 16; ++a) {
                                const double wa = (double)wt[a];
                                const double sa = (wt[a] > 0.0f) ? 1.0 : (wt[a] < 0.0f ? -1.0 : 0.0);
                                double tw = 0.0, ts = 0.0;  // sum_{b >= a} Us_ab w_b, Us_ab sigma_b
                                for (int b = a; b < 16; ++b) {
                                    const double h = sm.Us[tri(a, b)];
                                    tw = fma(h, (double)wt[b], tw);
                                    ts = fma(h, (wt[b] > 0.0f) ? 1.0 : (wt[b] < 0.0f ? -1.0 : 0.0), ts);
                                }
                                wHw = fma(wa, tw, wHw);
                                sHs = fma(sa, ts, sHs);
                                sHw_wHs = fma(sa, tw, fma(wa, ts, sHw_wHs));
                            }
                            const double sc = (double)s0 * (double)__int_as_float((127 + k) << 23);  // s_c, exact
                            E = all_sat ? (float)fma(fma(36.0 * sHs, sc, -6.0 * sHw_wHs), sc, wHw) : (float)wHw;
                            done = true;
                        }
                    }
                    if (!done) {
                        // q = 2^k E2M1_RNE_sat(u 2^-k): u 2^-k is exact (a power of two), and the
                        // sm_100a conversions round it to nearest even on the E2M1 grid with
                        // saturation at +-6 (two values per conversion) and give the values back
                        // exactly through f16x2; dw takes the factor 2^k with -s0 2^k (exact).
                        const bool sat_any = __any_sync(0xFFFFFFFFu, umax > lim);
                        const float2 sck = make_float2(__int_as_float((127 - k) << 23), __int_as_float((127 - k) << 23));
                        const float nsk = -s0 * __int_as_float((127 + k) << 23);  // -s0 2^k, exact
                        const float2 nsk2 = make_float2(nsk, nsk);
                        float2 dw[8];
#pragma unroll
                        for (int p = 0; p < 8; ++p) {
                            const float2 uk = __fmul2_rn(u[p], sck);  // u 2^-k, exact
                            dw[p] = __ffma2_rn(e2m1x2_round(uk), nsk2, w2[p]);  // w - q_c s_c = -dw, one rounding
                        }
                        // E >= mu sum_a H_aa dw_a^2: skip the form when, for every lane, that bound
                        // (rounded down) exceeds the best so far by more than the FP32 error margin,
                        // so the candidate can neither be the argmin nor tie it
                        float2 lb2 = make_float2(0.0f, 0.0f), lb2b = make_float2(0.0f, 0.0f);  // two chains
#pragma unroll
                        for (int p = 0; p < 8; p += 2) {
                            const float4 d4 = lds128(&sm.dg[p]);
                            lb2 = __ffma2_rn(__fmul2_rn(dw[p], dw[p]), make_float2(d4.x, d4.y), lb2);
                            lb2b = __ffma2_rn(__fmul2_rn(dw[p + 1], dw[p + 1]), make_float2(d4.z, d4.w), lb2b);
                        }
                        lb2 = __fadd2_rn(lb2, lb2b);
                        // a candidate is out once its exact error provably exceeds the incumbent's
                        // (only when mu > 0: otherwise E may be negative and nothing is pruned)
                        const float thr = rel ? best_e * up_fac : __int_as_float(0x7F800000);
                        const float lbraw = lb2.x + lb2.y;
                        bool out = lbraw * mu_lb > thr;
                        if constexpr (kMask) out = out || !allowed(class_code(f, x0 + k), tid);
                        if (__all_sync(0xFFFFFFFFu, out)) {
                            E = __int_as_float(0x7F800000);
                            if (up) {
                                // Every larger scale of the class, 2^k' s0 with k' > k, has its grid
                                // points in U = {0, .5, 1, 1.5, 2, 3, 4, 6, 8, 12, 16, ...} 2^k, so each
                                // weight stays at least its distance to U away from it at every later
                                // step. Below 6 * 2^k the nearest point of U is q here; above 4 * 2^k U is
                                // the grid {1, 1.5} 2^m. When any weight saturates, the distances come
                                // from an unclamped rounding onto U: the magic constant
                                // M = 1.5 * 2^23 * spacing (spacing from the binade of |u|, at least that
                                // of 2^k) makes (u + M) - M the round-to-nearest-even onto U (the grid
                                // is symmetric, so the sign rides along), less 2^-23 |w| for the rounding
                                // of u.
                                float tail = lbraw;
                                if (sat_any) {
                                    float2 tl2 = make_float2(0.0f, 0.0f);
#pragma unroll
                                    for (int p = 0; p < 8; p += 2) {
                                        const float4 d4 = lds128(&sm.dg[p]);
                                        float2 du[2];
#pragma unroll
                                        for (int h = 0; h < 2; ++h) {
                                            const unsigned ex = (__float_as_uint(u[p + h].x) & 0x7F800000u) + 0x0B400000u;
                                            const unsigned ey = (__float_as_uint(u[p + h].y) & 0x7F800000u) + 0x0B400000u;
                                            const float2 M = make_float2(__uint_as_float(max(ex, mlo)), __uint_as_float(max(ey, mlo)));
                                            const float2 qu = __ffma2_rn(M, make_float2(-1.0f, -1.0f), __fadd2_rn(u[p + h], M));
                                            du[h] = __ffma2_rn(qu, ns0, w2[p + h]);
                                        }
                                        tl2 = __ffma2_rn(__fmul2_rn(du[0], du[0]), make_float2(d4.x, d4.y), tl2);
                                        tl2 = __ffma2_rn(__fmul2_rn(du[1], du[1]), make_float2(d4.z, d4.w), tl2);
                                    }
                                    tail = tl2.x + tl2.y;
                                }
                                stop = __all_sync(0xFFFFFFFFu, __fmaf_rn(tail, mu_lb, -tail_corr) > thr);
                            }
                        } else {
                            E = form(dw);
#if LH_SWEEP_COUNTERS
                            ++cnt_form;
                            cnt_need += __popc(__ballot_sync(0xFFFFFFFFu, !out && active));
#endif
                        }
                    }
                    if constexpr (kMask) {
                        if (!allowed(class_code(f, x0 + k), tid)) E = __int_as_float(0x7F800000);
                    }
                    if (E < best_e) {
                        third_e = second_e;
                        second_e = best_e;
                        second_fk = best_fk;
                        best_e = E;
                        best_fk = 32 * f + k;
                    } else if (E < second_e) {
                        third_e = second_e;
                        second_e = E;
                        second_fk = 32 * f + k;
                    } else {
                        third_e = fminf(third_e, E);
                    }
                    return stop;
                };
                // Every scale 2^k' s0 with k' < k1 quantises to at most 6 * 2^k' s0 <= 3 * 2^k1 s0, so a
                // weight with |w| > 3 * 2^k1 s0 keeps an error of at least |w| - 3 * 2^k1 s0 there: true
                // when, for every lane, that bound already exceeds the incumbent's error.
                auto below_excluded = [&](int k1) -> bool {
                    if (!rel) return false;
#if LH_SWEEP_COUNTERS
                    ++cnt_below;
#endif
                    const float thr = best_e * up_fac;
                    const float nc3 = -__int_as_float(((128 + k1) << 23) | 0x400000);  // -3 * 2^k1
                    float2 acc = make_float2(0.0f, 0.0f), acc2 = make_float2(0.0f, 0.0f);
#pragma unroll
                    for (int p = 0; p < 8; p += 2) {
                        const float4 d4 = lds128(&sm.dg[p]);
                        // max(|w| - 3 * 2^k1 s0, 0), one rounding: zero exactly when |w| <= 3 * 2^k1 s0
                        const float2 d0 = make_float2(fmaxf(__fmaf_rn(nc3, s0, fabsf(w2[p].x)), 0.0f),
                                                      fmaxf(__fmaf_rn(nc3, s0, fabsf(w2[p].y)), 0.0f));
                        const float2 d1 = make_float2(fmaxf(__fmaf_rn(nc3, s0, fabsf(w2[p + 1].x)), 0.0f),
                                                      fmaxf(__fmaf_rn(nc3, s0, fabsf(w2[p + 1].y)), 0.0f));
                        acc = __ffma2_rn(__fmul2_rn(d0, d0), make_float2(d4.x, d4.y), acc);
                        acc2 = __ffma2_rn(__fmul2_rn(d1, d1), make_float2(d4.z, d4.w), acc2);
                    }
                    acc = __fadd2_rn(acc, acc2);
                    return __all_sync(0xFFFFFFFFu, (acc.x + acc.y) * mu_lb > thr);
                };
                // start at the warp's mean max-scaling index of the heavy channels (6 * 2^k >= hw / s0)
                int kst = 0;
                {
                    const float x = __fdividef(hw, 6.0f * s0);
                    const int e = (int)((__float_as_uint(x) >> 23) & 0xFF) - 127;
                    kst = (x > 1.0f) ? e + ((__float_as_uint(x) & 0x7FFFFF) ? 1 : 0) : 0;
                    kst = max(0, min(n - 1, kst));
                }
                const int k0 = (int)((__reduce_add_sync(0xFFFFFFFFu, (unsigned)kst) + 16u) >> 5);
                // one loop for both directions keeps a single copy of the candidate code: up
                // from k0 until a candidate ends the upward walk, then down from k0 - 1 while
                // the candidates below are not excluded as a whole
                bool up = true;
                int k = k0;
#pragma unroll 1
                while (true) {
                    if (up && k >= n) { up = false; k = k0 - 1; }
                    if (!up && (k < 0 || below_excluded(k + 1))) break;
                    if (candidate(k, up)) { up = false; k = k0 - 1; continue; }
                    k += up ? 1 : -1;
                }
            }
            // A candidate whose FP32 error is clear of the best's by the error bound cannot be the
            // argmin or tie it; every candidate the bounds excluded cannot either. So when the
            // runner-up is not clear but all others are, the argmin is one of the best two, and
            // FP64 errors of those two decide it (exact FP32 ties included: the lowest-code rule);
            // when a third one is not clear either, the whole block is re-swept in FP64.
            auto clear = [&](float e) {
                return rel ? (e * (1.0f - 4.0f * 5.9604645e-8f) > best_e * up_fac * (1.0f + rho))
                           : (e - best_e > margin);
            };
            if (!clear(second_e)) {                                      // also catches NaN / inf
                if (clear(third_e) && best_fk >= 0 && second_fk >= 0) pair = true;
                else flag = true;
            }
        }
        auto fk_code = [](int fk) {
            const int f = fk >> 5;
            const int tz = (f == 0) ? 3 : (f == 4) ? 2 : (f == 2 || f == 6) ? 1 : 0;
            return class_code(f, -6 - tz + (fk & 31));
        };
        int best_c = best_fk >= 0 ? fk_code(best_fk) : 1;

        // the FP64 paths read the block's weights from this thread's slot in shared memory
        float* const wst = reinterpret_cast<float*>(sm.key);
        if ((pair || flag) && active) {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                *reinterpret_cast<float4*>(wst + 16 * tid + 4 * i) =
                    make_float4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
        __syncwarp();

        // the best two of a block whose other candidates are clear, in FP64 by its own lane
        if (__any_sync(0xFFFFFFFFu, pair && active)) {
            if (pair && active) {
                const int second_c = fk_code(second_fk);
                const double e1 = candidate_error_f64(wst + 16 * tid, g, best_c, sm.Us);
                const double e2 = candidate_error_f64(wst + 16 * tid, g, second_c, sm.Us);
                // lexicographic (error, code) minimum; a NaN error never wins
                if (e2 < e1 || (e2 == e1 && second_c < best_c) || (e1 != e1 && e2 == e2)) best_c = second_c;
            }
        }

        // FP64 re-sweep of flagged blocks, one block at a time across the warp.
        unsigned pending = __ballot_sync(0xFFFFFFFFu, flag && active);
#if LH_SWEEP_COUNTERS
        {
            const unsigned act = __ballot_sync(0xFFFFFFFFu, active);
            const unsigned prs = __ballot_sync(0xFFFFFFFFu, pair && active);
            if (lane == 0) {
                atomicAdd(&lh_sweep_counts[0], 1ull);
                atomicAdd(&lh_sweep_counts[1], (unsigned long long)__popc(act));
                atomicAdd(&lh_sweep_counts[2], (unsigned long long)cnt_cand);
                atomicAdd(&lh_sweep_counts[3], (unsigned long long)cnt_form);
                atomicAdd(&lh_sweep_counts[4], (unsigned long long)cnt_need);
                atomicAdd(&lh_sweep_counts[5], (unsigned long long)cnt_below);
                atomicAdd(&lh_sweep_counts[6], (unsigned long long)__popc(pending));
                atomicAdd(&lh_sweep_counts[7], (unsigned long long)cnt_class);
                atomicAdd(&lh_sweep_counts[8], (unsigned long long)__popc(prs));
            }
        }
#endif
        while (pending) {
            const int src = __ffs(pending) - 1;
            pending &= pending - 1;
            double be = 0.0;
            int bc = 127;
            const int src_tid = (tid & ~31) + src;
            for (int c = lane + 1; c <= 126; c += 32) {
                if (!allowed(c, src_tid)) continue;
                const double e = candidate_error_f64(wst + 16 * src_tid, g, c, sm.Us);
                if (bc == 127 || e < be) { be = e; bc = c; }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                const double oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
                const int oc = __shfl_xor_sync(0xFFFFFFFFu, bc, off);
                // lexicographic (error, code) minimum; NaN errors never win
                const bool take = (oc != 127) && (bc == 127 || oe < be || (oe == be && oc < bc) ||
                                                  (be != be && oe == oe));
                if (take) { be = oe; bc = oc; }
            }
            if (lane == src) best_c = (bc >= 1 && bc <= 126) ? bc : 1;
        }

        if (active) {
            const int64_t o = *reinterpret_cast<volatile long long*>(&sm.ocol) + (int64_t)lp * J;
            best_code[o] = (uint8_t)best_c;
            best_amax[o] = __fmul_rn(6.0f, __fmul_rn(e4m3_value(best_c), g));
        }
    }
}

// One CTA per block column (m, j): mu and nu of its H, the same computation the
// sweep kernel does inline when it has no workspace. Its shared state is only what
// the bounds need, so many CTAs fit an SM.
struct BoundsShared {
    float Hf[256];
    __align__(16) float chol[8][32];  // the Cholesky tests' columns, per half-warp
    int pd[16];
    float mu, nu;
};

__global__ void __launch_bounds__(kThreads) sweep_bounds_kernel(const float* __restrict__ H,
                                                                ColBounds* __restrict__ out) {
    __shared__ __align__(16) BoundsShared sm;
    const int64_t col = blockIdx.x;
    const float* Hj = H ? H + col * 256 : nullptr;
    for (int i = threadIdx.x; i < 256; i += kThreads) sm.Hf[i] = Hj ? Hj[i] : ((i % 17 == 0) ? 1.0f : 0.0f);
    __syncthreads();
    column_bounds(sm, threadIdx.x);
    if (threadIdx.x == 0) {
        ColBounds c;
        c.mu = sm.mu;
        c.nu = sm.nu;
        c.pad0 = 0.0f;
        c.pad1 = 0.0f;
        out[col] = c;
    }
}

}  // namespace
}  // namespace lh

namespace lh {
namespace {

template <typename T, bool kURegs, bool kMask>
lh_status launch_kernel(dim3 grid, cudaStream_t st, const T* w, int64_t c_out, int64_t J,
                        int64_t ld, int64_t mat_stride, const float* gamax, const float* H, float* best_amax,
                        uint8_t* best_code, const ColBounds* cb, const Units& U, double m_start, double m_step,
                        int n_mult) {
    sweep_kernel<T, kURegs, kMask><<<grid, kThreads, 0, st>>>(w, c_out, J, ld, mat_stride, gamax, H, best_amax,
                                                             best_code, cb, U, m_start, m_step, n_mult);
    return cuda_status(cudaGetLastError(), "sweep_kernel launch");
}

// Without a workspace every CTA computes its column's bounds; with one, a first kernel
// computes each column's bounds once and the sweep's CTAs read them. (Launching the
// sweep as a programmatic dependent of that kernel, so that its set-up overlaps it,
// measured 5-9 % slower over the whole sweep on B200 and is not done.)
lh_status launch_sweep(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out, int64_t c_in, int64_t ld_w,
                       const float* global_amax, const float* H, float* best_amax, uint8_t* best_code, bool masked,
                       double m_start, double m_step, int n_mult, void* workspace, size_t workspace_bytes,
                       void* stream) {
    if (!valid_dtype(w_dtype)) return fail(LH_ERR_UNSUPPORTED, "w_dtype %d is not LH_BF16 or LH_F32", (int)w_dtype);
    if (!W || !global_amax || !best_amax || !best_code) return fail(LH_ERR_INVALID_ARG, "null pointer argument");
    if (n_mats < 1 || c_out < 0 || c_in < 0) return fail(LH_ERR_INVALID_ARG, "n_mats must be >= 1, sizes >= 0");
    if (c_in % 16 != 0) return fail(LH_ERR_UNSUPPORTED, "c_in=%lld is not a multiple of 16", (long long)c_in);
    if (ld_w < c_in) return fail(LH_ERR_INVALID_ARG, "ld_w=%lld < c_in=%lld", (long long)ld_w, (long long)c_in);
    if (!aligned16(W) || (ld_w * elem_bytes(w_dtype)) % 16 != 0)
        return fail(LH_ERR_ALIGNMENT, "W must be 16-byte aligned with 16-byte aligned rows");
    const int64_t J = c_in / 16;
    if (J > 65535 || n_mats > 65535) return fail(LH_ERR_UNSUPPORTED, "c_in/16 and n_mats must be <= 65535");
    const bool with_ws = workspace != nullptr || workspace_bytes != 0;
    if (with_ws) {
        const size_t need = sizeof(ColBounds) * (size_t)n_mats * (size_t)J;
        if (need > 0 && (!workspace || workspace_bytes < need))
            return fail(LH_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                        workspace ? workspace_bytes : (size_t)0);
        if (workspace && !aligned16(workspace)) return fail(LH_ERR_ALIGNMENT, "workspace must be 16-byte aligned");
    }
    if (c_out == 0 || J == 0) return LH_OK;
    Units U;
    U.tiles_per_col = (c_out + kTileRows - 1) / kTileRows;
    U.n_tiles = U.tiles_per_col * J * n_mats;
    // one wave of tiles (4 resident CTAs per SM at 128 registers) cut into pieces: the
    // whole tiles started last end while the pieces still keep every SM busy
    const int64_t slots = 4 * (int64_t)sm_count();
    const int64_t n_cut = U.n_tiles < slots ? U.n_tiles : slots;
    U.n_quart = n_cut / 4;
    U.n_split = n_cut - U.n_quart;
    const int64_t n_units = U.n_tiles + U.n_split + 3 * U.n_quart;
    if (n_units > 0x7FFFFFFF)
        return fail(LH_ERR_UNSUPPORTED, "too many blocks: ceil(c_out/512) * c_in/16 * n_mats must be < 2^31");
    const dim3 grid((unsigned)n_units);
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int64_t mat_stride = c_out * ld_w;
    ColBounds* cb = nullptr;
    if (with_ws) {
        cb = static_cast<ColBounds*>(workspace);
        sweep_bounds_kernel<<<(unsigned)(n_mats * J), kThreads, 0, st>>>(H, cb);
        const lh_status s = cuda_status(cudaGetLastError(), "sweep_bounds_kernel launch");
        if (s != LH_OK) return s;
    }
    if (w_dtype == LH_BF16) {
        const uint16_t* w = static_cast<const uint16_t*>(W);
        return masked ? launch_kernel<uint16_t, false, true>(grid, st, w, c_out, J, ld_w, mat_stride,
                                                             global_amax, H, best_amax, best_code, cb, U, m_start,
                                                             m_step, n_mult)
                      : launch_kernel<uint16_t, LH_SWEEP_UREGS, false>(grid, st, w, c_out, J, ld_w,
                                                                       mat_stride, global_amax, H, best_amax,
                                                                       best_code, cb, U, 0.0, 0.0, 0);
    }
    const float* w = static_cast<const float*>(W);
    return masked ? launch_kernel<float, false, true>(grid, st, w, c_out, J, ld_w, mat_stride, global_amax,
                                                      H, best_amax, best_code, cb, U, m_start, m_step, n_mult)
                  : launch_kernel<float, LH_SWEEP_UREGS, false>(grid, st, w, c_out, J, ld_w, mat_stride,
                                                                global_amax, H, best_amax, best_code, cb, U, 0.0,
                                                                0.0, 0);
}

}  // namespace
}  // namespace lh

extern "C" lh_status lh_sweep_scales(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out,
                                     int64_t c_in, int64_t ld_w, const float* global_amax, const float* H,
                                     float* best_amax, uint8_t* best_code, void* stream) {
    lh::clear_error();
    return lh::launch_sweep(W, w_dtype, n_mats, c_out, c_in, ld_w, global_amax, H, best_amax, best_code, false, 0.0,
                            0.0, 0, nullptr, 0, stream);
}

extern "C" size_t lh_sweep_workspace_bytes(int64_t n_mats, int64_t c_in) {
    if (n_mats < 1 || c_in < 0 || c_in % 16 != 0) return 0;
    return sizeof(lh::ColBounds) * (size_t)n_mats * (size_t)(c_in / 16);
}

extern "C" lh_status lh_sweep_scales_ws(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out,
                                        int64_t c_in, int64_t ld_w, const float* global_amax, const float* H,
                                        float* best_amax, uint8_t* best_code, void* workspace,
                                        size_t workspace_bytes, void* stream) {
    lh::clear_error();
    if (!workspace) return lh::fail(LH_ERR_WORKSPACE, "null workspace");
    return lh::launch_sweep(W, w_dtype, n_mats, c_out, c_in, ld_w, global_amax, H, best_amax, best_code, false, 0.0,
                            0.0, 0, workspace, workspace_bytes, stream);
}

extern "C" lh_status lh_search_amax(const void* W, lh_dtype w_dtype, int64_t n_mats, int64_t c_out, int64_t c_in,
                                    int64_t ld_w, const float* global_amax, const float* H, double start, double step,
                                    int64_t n_mult, float* best_amax, uint8_t* best_code, void* stream) {
    using namespace lh;
    clear_error();
    if (!(start > 0.0) || !(step >= 0.0) || !std::isfinite(start) || !std::isfinite(step))
        return fail(LH_ERR_INVALID_ARG, "start must be > 0 and step >= 0, both finite");
    if (n_mult < 1 || n_mult > 4096) return fail(LH_ERR_INVALID_ARG, "n_mult must be in [1, 4096]");
    return launch_sweep(W, w_dtype, n_mats, c_out, c_in, ld_w, global_amax, H, best_amax, best_code, true, start, step,
                        (int)n_mult, nullptr, 0, stream);
}

extern "C" lh_status lh_debug_sweep_counts(uint64_t* out, int clear) {
    using namespace lh;
    clear_error();
#if LH_SWEEP_COUNTERS
    if (clear) {
        const unsigned long long z[9] = {};
        return cuda_status(cudaMemcpyToSymbol(lh_sweep_counts, z, sizeof(z)), "clear sweep counts");
    }
    if (!out) return fail(LH_ERR_INVALID_ARG, "null out");
    return cuda_status(cudaMemcpyFromSymbol(out, lh_sweep_counts, sizeof(unsigned long long) * 9), "read sweep counts");
#else
    (void)out;
    (void)clear;
    return fail(LH_ERR_UNSUPPORTED, "this library is built without the sweep's work counters");
#endif
}
