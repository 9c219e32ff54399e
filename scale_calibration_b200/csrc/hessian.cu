// Local Hessian accumulation on tcgen05 tensor cores.
//
// "NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4 逐块权重缩放
// 算法实战指南" (xxmr.cn/news/266017): section "算法原理" defines the local
// Hessian of a 16-channel block as X_b X_b^T (16x16); section
// "入口 API 与校准流程", Phase 2, accumulates H = sum X^T X over the calibration
// tokens; the kernel contract lays H out as [cin/16, 16, 16].
//
// Design (B200): one kernel launch per call, bound by the HBM read of X.
//  * Work split: the tokens are cut into equal bands and the CTAs of the grid
//    (about two per SM) form one team per band, one CTA per 128-channel slab
//    (or per run of slabs when the layer is wider than the grid). The CTAs of a
//    team start together on the same token rows and read them slab by slab,
//    so the whole width of each row is fetched from HBM at about the same
//    time, and every CTA reads the same number of bytes whatever the group
//    sizes. A CTA walks its band as pieces (one group's run of tokens) cut
//    into stages of at most 128 tokens that never cross a group's end.
//  * Per CTA: a TMA producer warp, an MMA warp and four epilogue warps. The
//    producer stages [tokens x 128 channels] bf16 tiles (two 64-channel boxes,
//    128-byte swizzle; 128-token boxes, or 16-token boxes for the short last
//    stage of a piece) in a 3-deep shared-memory ring. The tile is
//    channel-contiguous, so it is an MN-major operand for both A = tile^T and
//    B = tile: one tcgen05.mma (M = N = 128, K = 16, FP32 accumulate in TMEM)
//    per 16 tokens forms the 128x128 Gram block of the slab, of which the 8
//    diagonal 16x16 blocks are the local Hessians (the off-diagonal products
//    cost tensor-core time only). Token rows of the last 16-row step that lie
//    past the piece are zeroed in shared memory before the MMA.
//  * The epilogue warps read each stage's 8 diagonal blocks from one of two
//    TMEM buffers (tcgen05.ld) and add them into FP64 registers, so FP32
//    accumulation never spans more than 128 tokens. At the end of a piece:
//    if the group's tokens of that slab lie in this CTA's band alone, the CTA
//    is the only one to add to those entries of H and adds its sum with
//    vector reductions (red.global.add.v4.f32, no wait for H to load);
//    otherwise it stores the sum as its part of the (slab, group) segment in
//    the workspace. Each band but the segment's last publishes its part (per
//    epilogue warp: a fence, then a flag set to the launch's generation); the
//    last band, whose share of the segment is the first piece of its walk,
//    adds the parts in band order after the rest of its work, when the
//    earlier bands, which end with that segment, are done with it too, and
//    adds the sum to H with one reduction. The order of every sum is fixed,
//    so H is deterministic. A CTA waits only for CTAs of earlier bands (lower
//    block indices, which the GPU starts first), each wait bounded.
//  * Nothing in the workspace needs clearing between calls: the parts are
//    written before their flags are set, and the flags and the status word
//    carry the call's 48-bit generation, so a stale value from an earlier call
//    (or a fresh buffer) never matches it.
//  * Every wait is bounded (1 s of globaltimer); on expiry the kernel records
//    LH_ERR_TIMEOUT in the workspace status word and the CTA winds down.
//    Decreasing group offsets are recorded as LH_ERR_INVALID_ARG (the walk
//    stays in bounds, and waits for parts stop once an error is recorded).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <chrono>
#include <mutex>

#include "common.cuh"
#include "tcgen05.cuh"

namespace lh {
namespace {

constexpr int kSlab = 128;                       // channels per slab = MMA M = N
constexpr int kStageTok = 128;                   // tokens per full pipeline stage
constexpr int kSmallBox = 16;                    // token rows of the boxes for a short stage
constexpr int kStages = 3;
constexpr int kHalfBytes = kStageTok * 64 * 2;   // one 128-token, 64-channel TMA box: 16 KB
constexpr int kStageBytes = 2 * kHalfBytes;      // 32 KB
constexpr int kThreads = 192;                    // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kTmemCols = 256;                   // two 128x128 FP32 accumulators
constexpr int kMaxCtas = 320;                    // grid bound (two CTAs per SM, up to 160 SMs)
constexpr size_t kHeaderBytes = 256;
constexpr int kPartFloats = 8 * 256;             // one slab's 8 blocks of 16x16, FP32
constexpr unsigned long long kGenMask = (1ull << 48) - 1;

// Instruction descriptor of tcgen05.mma kind::f16: D = F32, A = B = BF16,
// both MN-major, N = 128, M = 128.
constexpr uint32_t kIdesc = (1u << 4)            // D format F32
                            | (1u << 7)          // A format BF16
                            | (1u << 10)         // B format BF16
                            | (1u << 15)         // A MN-major
                            | (1u << 16)         // B MN-major
                            | ((uint32_t)(kSlab >> 3) << 17)   // N >> 3
                            | ((uint32_t)(kSlab >> 4) << 24);  // M >> 4


// The grid: `bands` teams of `sgroups` CTAs. With at most `cap` CTAs: one CTA
// per slab and as many bands as fit, or, for layers with more slabs than CTAs,
// one band and runs of slabs. Bands start on whole 128-token tiles and hold at
// least kMinBandTiles tiles each (fewer, longer bands when the layer is short):
// a band of a few tiles pays the CTA's set-up and the sum of the parts for
// little streaming, and a band edge inside a tile costs a short extra stage.
constexpr int64_t kMinBandTiles = 4;
// Grouped X: a group's run costs about half a stage beyond its tokens (its short last
// stage and its flush), charged when the bands are cut.
constexpr int64_t kGroupCost = 64;
struct Grid {
    int64_t slabs, sgroups, bands;
    int64_t ctas() const { return sgroups * bands; }
};
constexpr Grid make_grid(int64_t n_tok, int64_t c_in, int64_t cap) {
    Grid gr{};
    gr.slabs = (c_in + kSlab - 1) / kSlab;
    gr.sgroups = gr.slabs < cap ? gr.slabs : cap;
    const int64_t tiles = (n_tok + kStageTok - 1) / kStageTok;
    int64_t bmax = cap / gr.sgroups;
    if (bmax > tiles) bmax = tiles;
    if (bmax < 1) bmax = 1;
    int64_t per = (tiles + bmax - 1) / bmax;  // tiles of the longest band
    if (per < kMinBandTiles) per = kMinBandTiles;
    gr.bands = (tiles + per - 1) / per;
    if (gr.bands < 1) gr.bands = 1;
    return gr;
}

// Workspace: [header: status word, generation of the last launch][flags:
// [bands][slabs][2][4 epilogue warps] u64][parts: [bands][slabs][2][8 blocks]
// [16][16] FP32]. Parts and flags exist only with several bands (a layer no
// wider than the grid), so their count is bounded by twice the grid size.
struct WsLayout {
    size_t flag_off, part_off, total;
};
constexpr WsLayout ws_layout(const Grid& gr) {
    WsLayout w{};
    const size_t pairs = gr.bands > 1 ? (size_t)gr.bands * (size_t)gr.slabs : 0;
    w.flag_off = kHeaderBytes;
    w.part_off = w.flag_off + (sizeof(unsigned long long) * 2 * 4 * pairs + 255) / 256 * 256;
    w.total = w.part_off + sizeof(float) * kPartFloats * 2 * pairs;
    return w;
}

using namespace lh::tc;

// Shared-memory matrix descriptor: MN-major operand, 128-byte swizzle,
// 64 channels per swizzle atom (atoms kHalfBytes apart), 8 token rows per
// atom (1024 bytes apart along K).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr) {
    uint64_t d = 0;
    d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((kHalfBytes >> 4) & 0x3FFF) << 16;  // leading byte offset: next 64 channels
    d |= (uint64_t)((1024 >> 4) & 0x3FFF) << 32;        // stride byte offset: next 8 tokens
    d |= (uint64_t)1 << 46;                              // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;                              // SWIZZLE_128B
    return d;
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
          "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
          "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
// A bounded mbarrier wait taken by a whole warp, with one answer for all its lanes.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort_flag));
}

struct KParams {
    int64_t N;           // tokens
    int64_t J;           // block columns (c_in / 16)
    int64_t G;           // groups (1 without offsets)
    int64_t slabs, sgroups, bands;  // the grid: bands x sgroups CTAs (see Grid)
    const int64_t* off;  // [G + 1] group offsets, or null: one group of all tokens
    float* H;            // [G][J][16][16], H +=
    unsigned long long* hdr;       // [0] status: gen << 16 | lh_status, written on error; [1] gen of the launch
    float* parts;                  // [bands][slabs][2][8][16][16]
    unsigned long long* flags;     // [bands][slabs][2][4]: gen << 1 once an epilogue warp's rows of that part are
                                   // written, gen << 1 | 1 when the band had no part to give (see combine_parts)
    unsigned long long gen;        // this launch's generation, < 2^48
    int64_t gcost;                 // grouped X: tokens' worth of work charged per group when cutting bands
    int64_t ctot;                  // N + gcost G: the total cost the bands share
};

// For two costs T[0] <= T[1]: the first g in [0, G) whose group end, with gcost
// charged for it and every group before it, reaches T[i]: hi_g + gcost (g + 1) >=
// T[i] (hi_g = offsets[g + 1] clamped to [0, N]); G when none. Both searches by the
// whole warp, step by step together (32 probes each per step, two steps for
// G <= 1024). Exact for non-decreasing offsets; bounded answers in [0, G] for any
// others.
__device__ void find_band_groups(const KParams& p, const int64_t (&T)[2], int64_t (&out)[2], int lane) {
    auto key = [&](int64_t g) { return min(max(__ldg(p.off + g + 1), (int64_t)0), p.N) + p.gcost * (g + 1); };
    int64_t lo[2] = {0, 0}, n[2] = {p.G, p.G};
    bool done[2] = {false, false};
    while (!(done[0] && done[1])) {
        int64_t ak[2];
        bool hit[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int64_t step = n[i] > 32 ? (n[i] + 31) / 32 : 1;
            ak[i] = min(lo[i] + (int64_t)(lane + 1) * step - 1, lo[i] + n[i] - 1);
            hit[i] = !done[i] && (n[i] > 32 || lane < n[i]) && key(ak[i]) >= T[i];  // loads of both in flight
        }
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const unsigned m = __ballot_sync(0xFFFFFFFFu, hit[i]);
            if (done[i]) continue;
            if (n[i] <= 32) {
                out[i] = m ? lo[i] + __ffs(m) - 1 : lo[i] + n[i];
                done[i] = true;
            } else if (m == 0) {
                out[i] = lo[i] + n[i];
                done[i] = true;
            } else {
                const int64_t step = (n[i] + 31) / 32;
                const int k = __ffs(m) - 1;
                const int64_t nlo = lo[i] + (int64_t)k * step;
                n[i] = min(lo[i] + (int64_t)(k + 1) * step - 1, lo[i] + n[i] - 1) - nlo + 1;
                lo[i] = nlo;
            }
        }
    }
}

// Cost threshold of band k's first token: T_k = floor(ctot k / bands).
__device__ __forceinline__ int64_t band_cost(const KParams& p, int64_t k) { return p.ctot * k / p.bands; }

// First token of bands k and k + 1 (warp-wide: every lane calls it), and a group at
// or before the one holding band k's first token. One group: the 128-token tiles of
// [0, N) split as evenly as integers allow (band k starts at tile floor(tiles k /
// bands)). Groups: each group's run ends in a short stage and a flush, so a group is
// charged gcost tokens' worth of work, and band k starts at the first token t whose
// cost, t + gcost (groups ending at or before t), reaches T_k; a band edge that falls
// on a group's end starts the next group whole.
__device__ void band_range(const KParams& p, int64_t k, int lane, int64_t& t0, int64_t& t1, int64_t& g0) {
    g0 = 0;
    if (!p.off) {
        const int64_t tiles = (p.N + kStageTok - 1) / kStageTok;
        t0 = k <= 0 ? 0 : min(p.N, kStageTok * (tiles * k / p.bands));
        t1 = k + 1 >= p.bands ? p.N : min(p.N, kStageTok * (tiles * (k + 1) / p.bands));
        return;
    }
    const int64_t T[2] = {band_cost(p, k), band_cost(p, k + 1)};
    int64_t g[2];
    find_band_groups(p, T, g, lane);
    int64_t t[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        if (g[i] >= p.G) {
            t[i] = T[i] - p.gcost * p.G;
        } else {
            // tokens of group g cost t + gcost g, and its end costs hi_g + gcost (g + 1) >= T
            const int64_t hi = min(max(__ldg(p.off + g[i] + 1), (int64_t)0), p.N);
            t[i] = min(T[i] - p.gcost * g[i], hi);
        }
        t[i] = min(max(t[i], (int64_t)0), p.N);
    }
    t0 = k <= 0 ? 0 : t[0];
    t1 = k + 1 >= p.bands ? p.N : t[1];
    g0 = k <= 0 ? 0 : min(g[0], p.G);
}
// The first band of the segment of group g that starts at token seg_lo (its first
// token, so the groups ending at or before it are g's predecessors): the last band
// whose T_k is at most the cost seg_lo + gcost g. Exact for non-decreasing offsets.
__device__ __forceinline__ int64_t first_band(const KParams& p, int64_t g, int64_t seg_lo) {
    if (!p.off) return 0;
    const int64_t c = seg_lo + p.gcost * g;
    return max((int64_t)0, min(p.bands - 1, ((c + 1) * p.bands - 1) / p.ctot));
}
// Part slot of band k in one slab: s = 0 for a segment that began in an earlier band
// (the band's first piece), s = 1 for one that begins in this band and goes on into
// the next (its last piece).
__device__ __forceinline__ int64_t part_slot(const KParams& p, int64_t k, int64_t slab, int s) {
    return (k * p.slabs + slab) * 2 + s;
}

// The flag of epilogue warp q for a part slot (see part_slot).
__device__ __forceinline__ unsigned long long* part_flag(const KParams& p, int64_t slot, int q) {
    return p.flags + slot * 4 + q;
}
__device__ __forceinline__ unsigned long long ld_acquire(const unsigned long long* a) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(a) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(unsigned long long* a, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(a), "l"(v) : "memory");
}
// Records `code` for this launch unless an error of this launch is there already.
__device__ void record_error(const KParams& p, int code) {
    unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(p.hdr);
    const unsigned long long v = (p.gen << 16) | (unsigned long long)code;
    while ((cur >> 16) != p.gen) {
        const unsigned long long prev = atomicCAS(p.hdr, cur, v);
        if (prev == cur) break;
        cur = prev;
    }
}
// The sum of a segment (group g, one slab) that bands b0..k share, formed by its
// last band k at the end of its work: this warp's 32 rows of each earlier band's
// part once that band has published them (band b0's in slot 1, the others' in slot
// 0; a band that held no tokens publishes an empty flag), then the parts added in
// band order in FP64 (this band's own, in slot 0, last) and the sum added to H with
// one reduction. Bands wait only for bands before them (lower block indices, running
// or done). False when a wait gave up; `stopped` then says it was not a timeout.
__device__ bool combine_parts(const KParams& p, int64_t g, int64_t slab, int64_t seg_lo, int64_t k, int q, int row,
                              volatile int* abort_flag, bool& stopped) {
    const int lane = threadIdx.x & 31;
    const int64_t b0 = first_band(p, g, seg_lo);
    double t[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) t[c] = 0.0;
    auto add_parts = [&](const int64_t (&kb)[4], int n) {
        float4 v[4][4];  // up to four parts' loads in flight, then added in band order
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (i < n) {
                const float4* src = reinterpret_cast<const float4*>(
                    p.parts + part_slot(p, kb[i], slab, kb[i] == b0 ? 1 : 0) * kPartFloats + row * 16);
#pragma unroll
                for (int c = 0; c < 4; ++c) v[i][c] = __ldcg(src + c);
            }
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (i < n) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    t[4 * c] += v[i][c].x;
                    t[4 * c + 1] += v[i][c].y;
                    t[4 * c + 2] += v[i][c].z;
                    t[4 * c + 3] += v[i][c].w;
                }
            }
    };
    // bands base .. base + 31 at a time: lane i waits for the flag of band base + i
    for (int64_t base = b0; base < k; base += 32) {
        const int64_t kb = base + lane;
        const unsigned long long* f =
            kb < k ? part_flag(p, part_slot(p, kb, slab, kb == b0 ? 1 : 0), q) : p.hdr + 1;
        const uint64_t t0 = global_ns();
        unsigned long long v = 0;
        for (uint32_t it = 0;; ++it) {
            if (kb < k) v = ld_acquire(f);
            if (__all_sync(0xFFFFFFFFu, kb >= k || (v >> 1) == p.gen)) break;
            if ((it & 15) == 15) {
                const bool stop =
                    *abort_flag || (*reinterpret_cast<volatile unsigned long long*>(p.hdr) >> 16) == p.gen;
                if (__any_sync(0xFFFFFFFFu, stop)) {
                    stopped = true;
                    return false;
                }
                if (__any_sync(0xFFFFFFFFu, global_ns() - t0 > kTimeoutNs)) {
                    stopped = false;
                    return false;
                }
            }
        }
        __syncwarp();  // the parts the other lanes acquired are visible to the whole warp from here
        unsigned have = __ballot_sync(0xFFFFFFFFu, kb < k && (v & 1ull) == 0);  // bands with a part
        while (have) {
            int64_t kbs[4];
            int n = 0;
            while (have && n < 4) {
                kbs[n++] = base + __ffs(have) - 1;
                have &= have - 1;
            }
            add_parts(kbs, n);
        }
    }
    {
        const int64_t own[4] = {k, k, k, k};
        add_parts(own, 1);
    }
    const int64_t jb = slab * 8 + (row >> 4);
    if (jb < p.J) {
        float* hrow = p.H + ((g * p.J + jb) * 16 + (row & 15)) * 16;
#pragma unroll
        for (int c = 0; c < 4; ++c)
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(hrow + 4 * c), "f"((float)t[4 * c]),
                         "f"((float)t[4 * c + 1]), "f"((float)t[4 * c + 2]), "f"((float)t[4 * c + 3])
                         : "memory");
    }
    return true;
}

// Token range of group g, clamped to [0, N]; an inverted range is empty.
__device__ __forceinline__ void group_range(const KParams& p, int64_t g, int64_t& lo, int64_t& hi) {
    if (!p.off) { lo = 0; hi = p.N; return; }
    lo = min(max(__ldg(p.off + g), (int64_t)0), p.N);
    hi = min(max(__ldg(p.off + g + 1), lo), p.N);
}

// One stage as the producer hands it to the MMA warp and, through it, to the
// epilogue.
struct StageDesc {
    int32_t ntok;     // tokens of the stage (1..128); 0 marks the end of the CTA's work
    int32_t flags;    // bit 0: last stage of its piece (flush); bits 1-2: the piece's role (kOwned ..
                      // kLastBand); on the end marker, bit 3: the band holds no token
    int32_t slab;
    int32_t g;
    int64_t seg_lo;   // the group's first token (clamped): its segment in this slab is
    int64_t seg_hi;   // [seg_lo, seg_hi)
};

// What the end of a piece does with its sum: the group's tokens of the slab lie in
// this band alone (add to H); the segment began in an earlier band and goes on into a
// later one (part in slot 0, published); it begins here and goes on (slot 1,
// published); it began earlier and ends here (slot 0; this band sums the parts).
enum PieceRole : int32_t { kOwned = 0, kMiddle = 1, kFirstBand = 2, kLastBand = 3 };

struct Smem {
    uint64_t full[kStages], empty[kStages], tfull[2], tempty[2], dfull[2];
    StageDesc sdesc[kStages];  // per ring slot, written before the slot's loads
    StageDesc edesc[2];        // per TMEM buffer, for the epilogue
    uint32_t tmem_slot;
    int abort_flag;
};

__global__ void __launch_bounds__(kThreads, 2) hessian_tc_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                 const __grid_constant__ CUtensorMap tmap16,
                                                                 const KParams p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzled tiles
    uint8_t* tiles_p = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Smem& S = *reinterpret_cast<Smem*>(tiles_p + kStages * kStageBytes);
    volatile int* abort_flag = &S.abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t tiles = smem_u32(tiles_p);
    const int64_t b = blockIdx.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_u32(&S.full[s]), 1);
            mbar_init(smem_u32(&S.empty[s]), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(smem_u32(&S.tfull[a]), 1);
            mbar_init(smem_u32(&S.tempty[a]), 4);
            mbar_init(smem_u32(&S.dfull[a]), 1);
        }
        S.abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 1) tmem_alloc(smem_u32(&S.tmem_slot), kTmemCols);
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem_base = S.tmem_slot;
    // the set-up above overlaps the kernel before (programmatic launch); X, the
    // offsets, H and the workspace are touched only after it has finished
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (threadIdx.x == 0 && b == 0) p.hdr[1] = p.gen;

    const int64_t band = b / p.sgroups, sg = b - band * p.sgroups;
    const int64_t sl0 = p.slabs * sg / p.sgroups, sl1 = p.slabs * (sg + 1) / p.sgroups;  // this CTA's slabs
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        // The whole warp walks the band (group look-ups are warp-wide); lane 0 issues.
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap16)) : "memory");
        int stage = 0;
        uint32_t phase = 0;
        int64_t bt0, bt1, gb;  // this band's tokens, and a group at or before the one holding bt0
        band_range(p, band, lane, bt0, bt1, gb);
        for (int64_t slab = sl0; ok && slab < sl1; ++slab) {
            int64_t t = bt0;
            int64_t g = gb;
            while (ok && t < bt1) {
                int64_t lo = 0, hi = 0;
                while (g < p.G) {
                    group_range(p, g, lo, hi);
                    if (hi > t) break;
                    ++g;
                }
                if (g >= p.G || lo >= bt1) break;  // no group holds the rest of the band
                t = max(t, lo);
                const int64_t t1 = min(hi, bt1);
                const int32_t role = lo >= bt0 ? (hi <= bt1 ? kOwned : kFirstBand) : (hi <= bt1 ? kLastBand : kMiddle);
                for (int64_t ts = t; ts < t1; ts += kStageTok) {
                    const int ntok = (int)min((int64_t)kStageTok, t1 - ts);
                    if (!warp_wait(smem_u32(&S.empty[stage]), phase ^ 1, abort_flag)) { ok = false; break; }
                    if (lane == 0) {
                        StageDesc& d = S.sdesc[stage];
                        d.ntok = ntok;
                        d.flags = ((ts + kStageTok >= t1) ? 1 : 0) | (role << 1);
                        d.slab = (int32_t)slab;
                        d.g = (int32_t)g;
                        d.seg_lo = lo;
                        d.seg_hi = hi;
                        const int x = (int)(slab * kSlab);
                        const int y = (int)ts;
                        const uint32_t dst = tiles + stage * kStageBytes;
                        const uint32_t fb = smem_u32(&S.full[stage]);
                        if (ntok == kStageTok) {
                            mbar_expect_tx(fb, kStageBytes);
                            tma_load_2d(dst, &tmap, x, y, fb);
                            tma_load_2d(dst + kHalfBytes, &tmap, x + 64, y, fb);
                        } else {
                            // the short last stage of a piece: only the 16-row boxes it needs
                            const int nb = (ntok + kSmallBox - 1) / kSmallBox;
                            mbar_expect_tx(fb, (uint32_t)(nb * 2 * kSmallBox * 128));
                            for (int i = 0; i < nb; ++i) {
                                tma_load_2d(dst + i * kSmallBox * 128, &tmap16, x, y + i * kSmallBox, fb);
                                tma_load_2d(dst + kHalfBytes + i * kSmallBox * 128, &tmap16, x + 64,
                                            y + i * kSmallBox, fb);
                            }
                        }
                    }
                    __syncwarp();
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
                t = t1;
            }
        }
        if (ok) {
            // end marker for the MMA warp: a stage of 0 tokens
            if (warp_wait(smem_u32(&S.empty[stage]), phase ^ 1, abort_flag)) {
                if (lane == 0) {
                    S.sdesc[stage].ntok = 0;
                    S.sdesc[stage].flags = bt0 >= bt1 ? 8 : 0;
                    mbar_arrive(smem_u32(&S.full[stage]));
                }
            } else {
                ok = false;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        while (ok) {
            if (!warp_wait(smem_u32(&S.full[stage]), phase, abort_flag)) { ok = false; break; }
            const StageDesc d = S.sdesc[stage];
            // the stage (or the end marker) goes to the epilogue with a free TMEM buffer
            if (!warp_wait(smem_u32(&S.tempty[acc]), acc_phase ^ 1, abort_flag)) { ok = false; break; }
            if (d.ntok == 0) {
                if (lane == 0) {
                    S.edesc[acc] = d;
                    mbar_arrive(smem_u32(&S.dfull[acc]));
                }
                break;
            }
            const int ksteps = (d.ntok + 15) >> 4;
            const int pad_end = ksteps * 16;
            if (d.ntok < pad_end) {
                // zero token rows [ntok, pad_end) of both 64-channel halves (128 bytes each)
                uint8_t* base = tiles_p + stage * kStageBytes;
                const int n16 = (pad_end - d.ntok) * 8;  // 16-byte chunks per half
                for (int i = lane; i < 2 * n16; i += 32) {
                    const int h = i / n16, rem = i - h * n16;
                    const int row = d.ntok + (rem >> 3), c = rem & 7;
                    *reinterpret_cast<uint4*>(base + h * kHalfBytes + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async();
            }
            __syncwarp();
            fence_after();
            if (lane == 0) {
                S.edesc[acc] = d;
                mbar_arrive(smem_u32(&S.dfull[acc]));
                const uint32_t a0 = tiles + stage * kStageBytes;
                for (int kk = 0; kk < ksteps; ++kk) {
                    const uint64_t sd = smem_desc(a0 + kk * 2048);  // 16 token rows of 128 bytes
                    mma_f16(tmem_base + acc * kSlab, sd, sd, kIdesc, kk > 0 ? 1u : 0u);
                }
                mma_commit(smem_u32(&S.empty[stage]));
                mma_commit(smem_u32(&S.tfull[acc]));
            }
            __syncwarp();
            if (++stage == kStages) { stage = 0; phase ^= 1; }
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = threadIdx.x - 64;    // 0..127
        const int q = warp & 3;              // TMEM lane quarter this warp may access
        const int row = 32 * q + lane;       // channel within the slab
        const int blk = row >> 4, a = row & 15;
        const bool hi16 = lane >= 16;
        // this CTA's slice of the offsets: no adjacent pair may decrease
        if (p.off) {
            const int64_t nct = p.bands * p.sgroups;
            const int64_t g0 = p.G * b / nct, g1 = p.G * (b + 1) / nct;
            bool bad = false;
            for (int64_t g = g0 + et; g < g1; g += 128) bad |= __ldg(p.off + g + 1) < __ldg(p.off + g);
            if (bad) atomicExch(p.hdr, (p.gen << 16) | (unsigned long long)LH_ERR_INVALID_ARG);
        }
        int acc = 0;
        uint32_t acc_phase = 0;
        double sum[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) sum[c] = 0.0;
        // a segment whose last band this is: its part is in slot 0, the bands before add theirs;
        // the sum is formed after this CTA's other work, when they are done with theirs. It is
        // the group holding the band's first token, the same in every slab of the CTA.
        bool pending = false;
        int32_t pend_g = 0;
        int64_t pend_lo = 0;
        bool seen_err = false;  // a wait stopped because the CTA aborts or an error of this launch is recorded
        bool empty_band = false;
        while (ok) {
            if (!warp_wait(smem_u32(&S.dfull[acc]), acc_phase, abort_flag)) { ok = false; break; }
            const StageDesc d = S.edesc[acc];
            if (d.ntok == 0) {
                empty_band = (d.flags & 8) != 0;
                break;
            }
            if (!warp_wait(smem_u32(&S.tfull[acc]), acc_phase, abort_flag)) { ok = false; break; }
            fence_after();
            uint32_t r[32];
            tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + acc * kSlab + 32 * q, r);
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&S.tempty[acc]));
#pragma unroll
            for (int c = 0; c < 16; ++c) sum[c] += (double)__uint_as_float(hi16 ? r[16 + c] : r[c]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
            if (!(d.flags & 1)) continue;

            // ---- end of a piece: add it to H, alone or through the parts
            const int64_t jb = (int64_t)d.slab * 8 + blk;
            const bool in_h = jb < p.J;
            float* hrow = p.H + (((int64_t)d.g * p.J + jb) * 16 + a) * 16;
            const int role = (d.flags >> 1) & 3;
            if (role == kOwned) {
                // the group's tokens of this slab are all in this band: no other CTA adds to
                // these entries of H, so a reduction is one ordered addition, H = fp32(H + fp32(sum))
                if (in_h) {
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(hrow + 4 * c),
                                     "f"((float)sum[4 * c]), "f"((float)sum[4 * c + 1]), "f"((float)sum[4 * c + 2]),
                                     "f"((float)sum[4 * c + 3])
                                     : "memory");
                }
            } else {
                // this band's part of a segment that several bands share
                const int64_t slot = part_slot(p, band, d.slab, role == kFirstBand ? 1 : 0);
                float4* part = reinterpret_cast<float4*>(p.parts + slot * kPartFloats + row * 16);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    __stcg(part + c, make_float4((float)sum[4 * c], (float)sum[4 * c + 1], (float)sum[4 * c + 2],
                                                 (float)sum[4 * c + 3]));
                if (role != kLastBand) {
                    // a later band adds it: publish this warp's rows of the part
                    __threadfence();
                    __syncwarp();
                    if (lane == 0) st_release(part_flag(p, slot, q), p.gen << 1);
                } else {
                    // the segment's last band: sum the parts at the end of this CTA's work
                    pending = true;
                    pend_g = d.g;
                    pend_lo = d.seg_lo;
                }
            }
#pragma unroll
            for (int c = 0; c < 16; ++c) sum[c] = 0.0;
        }
        // a band without tokens tells the segment that spans it that it has no part
        if (ok && empty_band && lane == 0)
            for (int64_t sl = sl0; sl < sl1; ++sl) st_release(part_flag(p, part_slot(p, band, sl, 0), q), (p.gen << 1) | 1);
        for (int64_t sl = sl0; ok && pending && sl < sl1; ++sl)
            ok = combine_parts(p, pend_g, sl, pend_lo, band, q, row, abort_flag, seen_err);
        if (!ok && seen_err) {
            ok = true;  // stopped for an error that is recorded already: no timeout to report
            *abort_flag = 1;
        }
    }

    if (!ok) {
        *abort_flag = 1;
        record_error(p, LH_ERR_TIMEOUT);
    }
    __syncthreads();
    if (*abort_flag) {
        // let copies and MMAs already issued by this CTA land before leaving
        const uint64_t t0 = global_ns();
        while (global_ns() - t0 < 200000ull) {
        }
    }
    fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// Diagnostics: the bounded wait of the kernel above, on an mbarrier that
// nothing arrives on (arrive == 0) or that thread 0 completes first
// (arrive != 0); a wait that runs out records LH_ERR_TIMEOUT in the workspace
// header as hessian_tc_kernel does.
__global__ void wait_timeout_kernel(unsigned long long* hdr, unsigned long long gen, uint64_t timeout_ns, int arrive) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        hdr[1] = gen;
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();
    if (arrive && threadIdx.x == 0) mbar_arrive(smem_u32(&bar));
    const bool ok = mbar_wait(smem_u32(&bar), 0u, &abort_flag, timeout_ns);
    if (!ok) atomicExch(hdr, (gen << 16) | (unsigned long long)LH_ERR_TIMEOUT);
}

// Generation of a launch: distinct for every call of the process (48 bits,
// never 0), starting from a value taken from the clock so that a workspace
// left by another process is unlikely to hold a matching stamp.
unsigned long long next_generation() {
    static std::atomic<unsigned long long> g{
        ((unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count() * 0x9E3779B97F4A7C15ull) >>
        16};
    for (;;) {
        const unsigned long long v = (g.fetch_add(1, std::memory_order_relaxed) + 1) & kGenMask;
        if (v != 0) return v;
    }
}

// Argument checks shared by the Hessian entry points (host side, before any launch).
lh_status validate_hessian_args(const void* X, lh_dtype x_dtype, int64_t n_tokens_total, int64_t c_in, int64_t ld_x,
                                const int64_t* offsets, int64_t n_groups, const float* H) {
    if (x_dtype != LH_BF16) return fail(LH_ERR_UNSUPPORTED, "X must be LH_BF16");
    if (!X || !H) return fail(LH_ERR_INVALID_ARG, "null X or H");
    if (n_tokens_total < 0 || c_in < 0 || n_groups < 1)
        return fail(LH_ERR_INVALID_ARG, "n_tokens_total, c_in must be >= 0 and n_groups >= 1");
    if (!offsets && n_groups != 1) return fail(LH_ERR_INVALID_ARG, "offsets == NULL requires n_groups == 1");
    if (c_in % 16 != 0) return fail(LH_ERR_UNSUPPORTED, "c_in=%lld is not a multiple of 16", (long long)c_in);
    if (ld_x < c_in) return fail(LH_ERR_INVALID_ARG, "ld_x < c_in");
    if (!aligned16(X) || (ld_x * 2) % 16 != 0)
        return fail(LH_ERR_ALIGNMENT, "X must be 16-byte aligned and ld_x a multiple of 8");
    if (n_tokens_total >= ((int64_t)1 << 31) || c_in >= ((int64_t)1 << 31) || n_groups > 65535)
        return fail(LH_ERR_UNSUPPORTED, "n_tokens_total and c_in must be < 2^31, n_groups <= 65535");
    return LH_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}


}  // namespace
}  // namespace lh

extern "C" size_t lh_hessian_workspace_bytes(int64_t n_tokens_total, int64_t c_in, int64_t n_groups) {
    using namespace lh;
    if (n_tokens_total < 0 || c_in <= 0 || n_groups < 1) return 0;
    // sized for the largest grid the launch uses on any GPU (it uses fewer CTAs on one with
    // under 160 SMs, and then fewer bands and parts)
    return ws_layout(make_grid(n_tokens_total, c_in, kMaxCtas)).total;
}

extern "C" lh_status lh_workspace_status(const void* workspace, void* stream) {
    using namespace lh;
    clear_error();
    if (!workspace) return fail(LH_ERR_INVALID_ARG, "null workspace");
    unsigned long long w[2] = {0, 0};
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    lh_status s = cuda_status(cudaMemcpyAsync(w, workspace, sizeof(w), cudaMemcpyDeviceToHost, st),
                              "read workspace status");
    if (s != LH_OK) return s;
    s = cuda_status(cudaStreamSynchronize(st), "synchronise");
    if (s != LH_OK) return s;
    if ((w[0] >> 16) != (w[1] & kGenMask)) return LH_OK;  // no error recorded by the last launch
    const int err = (int)(w[0] & 0xFFFFull);
    if (err == LH_ERR_TIMEOUT) return fail(LH_ERR_TIMEOUT, "a bounded wait in the Hessian kernel expired");
    if (err == LH_ERR_INVALID_ARG) return fail(LH_ERR_INVALID_ARG, "the group offsets decrease (overlapping ranges)");
    if (err != 0) return fail((lh_status)err, "the Hessian kernel recorded an error");
    return LH_OK;
}

extern "C" lh_status lh_debug_wait_timeout(void* workspace, size_t workspace_bytes, int64_t timeout_us,
                                           int arrive, void* stream) {
    using namespace lh;
    clear_error();
    if (!workspace || workspace_bytes < kHeaderBytes) return fail(LH_ERR_WORKSPACE, "workspace of 256 bytes needed");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(LH_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
    if (timeout_us < 1 || timeout_us > 1000000) return fail(LH_ERR_INVALID_ARG, "timeout_us must be in [1, 1e6]");
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    wait_timeout_kernel<<<1, 32, 0, st>>>(static_cast<unsigned long long*>(workspace), next_generation(),
                                          (uint64_t)timeout_us * 1000ull, arrive);
    return cuda_status(cudaGetLastError(), "wait_timeout_kernel launch");
}

extern "C" lh_status lh_accumulate_hessian(const void* X, lh_dtype x_dtype, int64_t n_tokens_total, int64_t c_in,
                                           int64_t ld_x, const int64_t* offsets, int64_t n_groups, float* H,
                                           void* workspace, size_t workspace_bytes, void* stream) {
    using namespace lh;
    clear_error();
    lh_status s = validate_hessian_args(X, x_dtype, n_tokens_total, c_in, ld_x, offsets, n_groups, H);
    if (s != LH_OK) return s;
    if (n_tokens_total == 0 || c_in == 0) return LH_OK;
    const WsLayout wl = ws_layout(make_grid(n_tokens_total, c_in, kMaxCtas));  // what the workspace is sized for
    if (!workspace || workspace_bytes < wl.total)
        return fail(LH_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", wl.total,
                    workspace ? workspace_bytes : (size_t)0);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(LH_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
    const int sms = sm_count();
    if (sms <= 0) return fail(LH_ERR_CUDA, "no CUDA device");
    auto encode = get_encode_fn();
    if (!encode) return fail(LH_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");

    CUtensorMap tmap, tmap16;
    const cuuint64_t dims[2] = {(cuuint64_t)c_in, (cuuint64_t)n_tokens_total};
    const cuuint64_t strides[1] = {(cuuint64_t)(ld_x * 2)};
    const cuuint32_t estr[2] = {1, 1};
    const cuuint32_t box[2] = {64, (cuuint32_t)kStageTok};
    const cuuint32_t box16[2] = {64, (cuuint32_t)kSmallBox};
    CUresult cr = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr == CUDA_SUCCESS)
        cr = encode(&tmap16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims, strides, box16, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(LH_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)cr);

    const int64_t cap = 2 * (int64_t)sms < kMaxCtas ? 2 * (int64_t)sms : kMaxCtas;  // two CTAs per SM
    const Grid gr = make_grid(n_tokens_total, c_in, cap);  // no more bands or slabs than sized for
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    KParams kp;
    kp.N = n_tokens_total;
    kp.J = c_in / 16;
    kp.G = offsets ? n_groups : 1;
    kp.slabs = gr.slabs;
    kp.sgroups = gr.sgroups;
    kp.bands = gr.bands;
    kp.off = offsets;
    kp.H = H;
    kp.hdr = reinterpret_cast<unsigned long long*>(ws);
    kp.parts = reinterpret_cast<float*>(ws + wl.part_off);
    kp.flags = reinterpret_cast<unsigned long long*>(ws + wl.flag_off);
    kp.gen = next_generation();
    kp.gcost = offsets ? kGroupCost : 0;
    kp.ctot = n_tokens_total + kp.gcost * kp.G;

    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    const size_t smem_bytes = (size_t)kStages * kStageBytes + 1024 + sizeof(Smem);
    std::call_once(attr_once, [&] {
        attr_err = cudaFuncSetAttribute(hessian_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes);
    });
    if (attr_err != cudaSuccess) return cuda_status(attr_err, "set shared memory size");
    // programmatic launch: the set-up of its CTAs overlaps the end of the kernel before
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)gr.ctas());
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem_bytes;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, hessian_tc_kernel, tmap, tmap16, kp), "hessian_tc_kernel launch");
}

// ---------------------------------------------------------------------------
// Allocation-free variant of lh_accumulate_hessian.
//
// Some callers cannot allocate device memory when they calibrate: serving
// processes that reserve nearly all HBM for their own pools at start-up,
// plugins whose host owns every device allocation and offers them no
// allocator, and latency-sensitive callers that avoid cudaMalloc/cudaFree
// because those calls can synchronise the whole device. This entry point
// takes the Hessian workspace from a fixed array compiled into the library
// instead of from the caller. Every GPU that loads the library holds the
// array (kNoAllocScratchBytes) until the process exits.
//
// In host code `lh_noalloc_scratch` names a host-side stand-in, not a device
// address; its device address is looked up once per device with
// cudaGetSymbolAddress on the first call made with that device current, and
// that lookup is the only set-up. Make the first call on each device before
// any stream capture. All calls share the one array: nothing in it needs
// clearing between calls (its parts are rewritten before they are read and its status word carries each call's
// generation), and calls whose kernels overlap on the GPU (different streams,
// or different host threads) race on the array and must be serialised by the
// caller.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;  // 8 MiB
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};
}  // namespace

static __device__ __align__(256) unsigned char lh_noalloc_scratch[kNoAllocScratchBytes];
// the largest workspace (parts of kMaxCtas (band, slab) pairs) fits: no call is turned away
static_assert(lh::ws_layout(lh::Grid{1, 1, lh::kMaxCtas}).total <= kNoAllocScratchBytes,
              "scratch holds the largest workspace");

// Device address of the scratch array for the current device, looked up on
// first use with that device current (the only set-up the entry point needs).
static lh_status noalloc_scratch(void** out) {
    using namespace lh;
    int dev = 0;
    lh_status s = cuda_status(cudaGetDevice(&dev), "cudaGetDevice");
    if (s != LH_OK) return s;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(LH_ERR_UNSUPPORTED, "device index %d too large", dev);
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        s = cuda_status(cudaGetSymbolAddress(&p, lh_noalloc_scratch), "cudaGetSymbolAddress(scratch)");
        if (s != LH_OK) return s;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return LH_OK;
}

extern "C" lh_status lh_accumulate_hessian_noalloc(const void* X, lh_dtype x_dtype, int64_t n_tokens_total,
                                                   int64_t c_in, int64_t ld_x, const int64_t* offsets,
                                                   int64_t n_groups, float* H, void* stream) {
    using namespace lh;
    clear_error();
    // the same argument checks, in the same order, as the workspace entry point
    lh_status s = validate_hessian_args(X, x_dtype, n_tokens_total, c_in, ld_x, offsets, n_groups, H);
    if (s != LH_OK) return s;
    if (n_tokens_total == 0 || c_in == 0) return LH_OK;
    const size_t need = lh_hessian_workspace_bytes(n_tokens_total, c_in, n_groups);
    if (need > kNoAllocScratchBytes)  // cannot happen (see the static_assert); kept as a guard
        return fail(LH_ERR_WORKSPACE,
                    "this Hessian needs %zu bytes of scratch but the allocation-free entry point has %zu "
                    "(8 MiB); call lh_accumulate_hessian with a caller-provided workspace instead",
                    need, kNoAllocScratchBytes);
    void* scratch = nullptr;
    s = noalloc_scratch(&scratch);
    if (s != LH_OK) return s;
    return lh_accumulate_hessian(X, x_dtype, n_tokens_total, c_in, ld_x, offsets, n_groups, H, scratch,
                                 kNoAllocScratchBytes, stream);
}

// Status the last allocation-free call on the current device left in the
// scratch array's header; the same words lh_workspace_status reads.
extern "C" lh_status lh_noalloc_status(void* stream) {
    using namespace lh;
    clear_error();
    void* scratch = nullptr;
    lh_status s = noalloc_scratch(&scratch);
    if (s != LH_OK) return s;
    return lh_workspace_status(scratch, stream);
}
