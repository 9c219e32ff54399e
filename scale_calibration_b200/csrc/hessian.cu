// Local Hessian accumulation on tcgen05 tensor cores.
//
// "NVIDIA Model Optimizer Local-Hessian: 基于局部 Hessian 的 NVFP4 逐块权重缩放
// 算法实战指南" (xxmr.cn/news/266017): section "算法原理" defines the local
// Hessian of a 16-channel block as X_b X_b^T (16x16); section
// "入口 API 与校准流程", Phase 2, accumulates H = sum X^T X over the calibration
// tokens; the kernel contract lays H out as [cin/16, 16, 16].
//
// Design (B200):
//  * Work item = (token chunk, 128-channel slab). A persistent grid of two CTAs
//    per SM walks the items; each CTA has a TMA producer warp, an MMA warp and
//    four epilogue warps, and two CTAs per SM keep more loads in flight and fill
//    each other's pipeline gaps.
//  * The producer stages [128 tokens x 128 channels] bf16 tiles (two 64-channel
//    TMA boxes, 128-byte swizzle) in a 3-deep shared-memory ring (96 KB).
//  * The tile is channel-contiguous, so it is an MN-major operand for both
//    A = tile^T (M = channels, K = tokens) and B = tile (K = tokens,
//    N = channels): one tcgen05.mma (M = N = 128, K = 16, FP32 accumulate in
//    TMEM) per 16 tokens forms the 128x128 Gram block of the slab, of which the
//    8 diagonal 16x16 blocks are the local Hessians. The off-diagonal products
//    cost tensor-core time only; the kernel stays bound by the HBM read of X.
//  * Each stage accumulates into one of two TMEM buffers; the epilogue warps
//    read the diagonal blocks (tcgen05.ld), free the buffer, and add them into
//    FP64 registers, so FP32 accumulation never spans more than 128 tokens.
//  * A chunk's sums go to the workspace; a second kernel adds the chunks of
//    each group in a fixed order (FP64) into H. No atomics: the result is
//    deterministic.
//  * Ragged ends (group boundaries inside a tile) are masked by zeroing the
//    token rows past the end inside the last 16-row MMA step; rows past the
//    tensor end arrive as zeros from TMA.
//  * Every mbarrier wait is bounded (1 s of globaltimer); on expiry the kernel
//    records LH_ERR_TIMEOUT in the workspace header and the CTA winds down.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "tcgen05.cuh"

namespace lh {
namespace {

constexpr int kSlab = 128;                       // channels per item = MMA M = N
constexpr int kStageTok = 128;                   // tokens per pipeline stage
constexpr int kStages = 3;
constexpr int kHalfBytes = kStageTok * 64 * 2;   // one 64-channel TMA box: 16 KB
constexpr int kStageBytes = 2 * kHalfBytes;      // 32 KB
constexpr int kThreads = 192;                    // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kTmemCols = 256;                   // two 128x128 FP32 accumulators
constexpr int kMinItems = 256;                   // work items wanted for one launch
constexpr int kMaxItems = 16384;
constexpr size_t kHeaderBytes = 256;

// Instruction descriptor of tcgen05.mma kind::f16: D = F32, A = B = BF16,
// both MN-major, N = 128, M = 128.
constexpr uint32_t kIdesc = (1u << 4)            // D format F32
                            | (1u << 7)          // A format BF16
                            | (1u << 10)         // B format BF16
                            | (1u << 15)         // A MN-major
                            | (1u << 16)         // B MN-major
                            | ((uint32_t)(kSlab >> 3) << 17)   // N >> 3
                            | ((uint32_t)(kSlab >> 4) << 24);  // M >> 4

struct Chunk {
    int64_t start;
    int32_t len;
    int32_t group;
};

struct WsLayout {
    size_t table_off, kfirst_off, partial_off, total;
    int64_t max_chunks;
};

struct Plan {
    int64_t chunk;       // tokens per chunk (multiple of kStageTok)
    int64_t n_slabs;
    int64_t max_chunks;  // bound on the number of chunks
    WsLayout ws;
};

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

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
__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t accumulate) {
    mma_f16(tmem_d, a, b, kIdesc, accumulate);
}
__device__ __forceinline__ void tc_fence_before() { fence_before(); }
__device__ __forceinline__ void tc_fence_after() { fence_after(); }
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

int64_t chunks_bound(int64_t n_tok, int64_t chunk, int64_t n_groups) {
    return (n_tok + chunk - 1) / chunk + (n_groups - 1);
}

Plan make_plan(int64_t n_tok, int64_t c_in, int64_t n_groups) {
    Plan p;
    p.n_slabs = (c_in + kSlab - 1) / kSlab;
    int64_t ch = 2048;
    while (ch > kStageTok && chunks_bound(n_tok, ch, n_groups) * p.n_slabs < kMinItems) ch /= 2;
    while (chunks_bound(n_tok, ch, n_groups) * p.n_slabs > kMaxItems && ch < ((int64_t)1 << 40)) ch *= 2;
    p.chunk = ch;
    p.max_chunks = chunks_bound(n_tok, ch, n_groups);
    const int64_t J = c_in / 16;
    p.ws.max_chunks = p.max_chunks;
    p.ws.table_off = kHeaderBytes;
    p.ws.kfirst_off = p.ws.table_off + align256(sizeof(Chunk) * (size_t)p.max_chunks);
    p.ws.partial_off = p.ws.kfirst_off + align256(sizeof(int32_t) * (size_t)(n_groups + 1));
    p.ws.total = p.ws.partial_off + sizeof(float) * 256 * (size_t)J * (size_t)p.max_chunks;
    return p;
}

struct KParams {
    int64_t n_tok;
    int64_t J;
    int64_t n_slabs;
    int64_t chunk;
    int64_t n_items_max;
    int grouped;
    const Chunk* table;
    const int32_t* n_chunks_dev;  // grouped: number of chunks (device)
    float* partial;               // [max_chunks][J][256]
    int* err;                     // workspace header word 0
};

__device__ __forceinline__ bool item_chunk(const KParams& p, int64_t item, int64_t n_chunks, int64_t& k,
                                           int64_t& sl, int64_t& start, int64_t& len) {
    k = item / p.n_slabs;
    sl = item - k * p.n_slabs;
    if (k >= n_chunks) return false;
    if (p.grouped) {
        const Chunk c = p.table[k];
        start = c.start;
        len = c.len;
    } else {
        start = k * p.chunk;
        len = min(p.chunk, p.n_tok - start);
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 2) hessian_tc_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                 const KParams p) {
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte alignment for the 128-byte-swizzled tiles
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    // bars: full[kStages], empty[kStages], tfull[2], tempty[2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t tiles = smem_u32(smem);
    auto full_bar = [&](int s) { return smem_u32(bars + s); };
    auto empty_bar = [&](int s) { return smem_u32(bars + kStages + s); };
    auto tfull_bar = [&](int a) { return smem_u32(bars + 2 * kStages + a); };
    auto tempty_bar = [&](int a) { return smem_u32(bars + 2 * kStages + 2 + a); };

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 4);
        }
        *abort_flag = 0;
        mbar_init_fence();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // set-up above overlaps the kernel before (programmatic launch); X, the chunk table
    // and the workspace header are read only after it has finished
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap)) : "memory");

    const int64_t n_chunks = p.grouped ? (int64_t)(*p.n_chunks_dev) : (p.n_tok + p.chunk - 1) / p.chunk;
    bool ok = true;

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            for (int64_t item = blockIdx.x; ok && item < p.n_items_max; item += gridDim.x) {
                int64_t k, sl, start, len;
                if (!item_chunk(p, item, n_chunks, k, sl, start, len)) break;
                const int n_st = (int)((len + kStageTok - 1) / kStageTok);
                for (int st = 0; st < n_st; ++st) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1, abort_flag)) { ok = false; break; }
                    mbar_expect_tx(full_bar(stage), kStageBytes);
                    const int y = (int)(start + (int64_t)st * kStageTok);
                    const int x = (int)(sl * kSlab);
                    tma_load_2d(tiles + stage * kStageBytes, &tmap, x, y, full_bar(stage));
                    tma_load_2d(tiles + stage * kStageBytes + kHalfBytes, &tmap, x + 64, y, full_bar(stage));
                    if (++stage == kStages) { stage = 0; phase ^= 1; }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        int stage = 0;
        uint32_t phase = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int64_t item = blockIdx.x; ok && item < p.n_items_max; item += gridDim.x) {
            int64_t k, sl, start, len;
            if (!item_chunk(p, item, n_chunks, k, sl, start, len)) break;
            const int n_st = (int)((len + kStageTok - 1) / kStageTok);
            for (int st = 0; st < n_st; ++st) {
                if (!mbar_wait(full_bar(stage), phase, abort_flag)) { ok = false; break; }
                const int nv = (int)min((int64_t)kStageTok, len - (int64_t)st * kStageTok);
                const int ksteps = (nv + 15) >> 4;
                const int pad_end = ksteps * 16;
                if (nv < pad_end) {
                    // zero token rows [nv, pad_end) of both 64-channel halves (128 bytes each)
                    uint8_t* base = smem + stage * kStageBytes;
                    const int n16 = (pad_end - nv) * 8;  // 16-byte chunks per half
                    for (int i = lane; i < 2 * n16; i += 32) {
                        const int h = i / n16, rem = i - h * n16;
                        const int row = nv + (rem >> 3), c = rem & 7;
                        *reinterpret_cast<uint4*>(base + h * kHalfBytes + row * 128 + c * 16) = make_uint4(0, 0, 0, 0);
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                }
                __syncwarp();
                if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1, abort_flag)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t a0 = tiles + stage * kStageBytes;
                    for (int kk = 0; kk < ksteps; ++kk) {
                        const uint64_t d = smem_desc(a0 + kk * 2048);  // 16 token rows of 128 bytes
                        mma_bf16(tmem_base + acc * kSlab, d, d, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(empty_bar(stage));
                    mma_commit(tfull_bar(acc));
                }
                __syncwarp();
                if (++stage == kStages) { stage = 0; phase ^= 1; }
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;              // TMEM lane quarter this warp may access
        const int row = 32 * q + lane;       // channel within the slab
        const int blk = row >> 4, a = row & 15;
        const bool hi = lane >= 16;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int64_t item = blockIdx.x; ok && item < p.n_items_max; item += gridDim.x) {
            int64_t k, sl, start, len;
            if (!item_chunk(p, item, n_chunks, k, sl, start, len)) break;
            const int n_st = (int)((len + kStageTok - 1) / kStageTok);
            double sum[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) sum[c] = 0.0;
            for (int st = 0; st < n_st; ++st) {
                if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) { ok = false; break; }
                tc_fence_after();
                uint32_t r[32];
                tmem_ld32(tmem_base + ((uint32_t)(32 * q) << 16) + acc * kSlab + 32 * q, r);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(tempty_bar(acc));
#pragma unroll
                for (int c = 0; c < 16; ++c) sum[c] += (double)__uint_as_float(hi ? r[16 + c] : r[c]);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            if (!ok) break;
            const int64_t jb = sl * 8 + blk;
            if (jb < p.J) {
                float4* dst = reinterpret_cast<float4*>(p.partial + ((size_t)k * p.J + jb) * 256 + a * 16);
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    dst[c] = make_float4((float)sum[4 * c], (float)sum[4 * c + 1], (float)sum[4 * c + 2],
                                         (float)sum[4 * c + 3]);
            }
        }
    }

    if (!ok) {
        *abort_flag = 1;
        atomicExch(p.err, (int)LH_ERR_TIMEOUT);
    }
    // the reduction may launch now; it waits for this grid to finish before reading
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __syncthreads();
    if (*abort_flag) {
        // let copies and MMAs already issued by this CTA land before leaving
        const uint64_t t0 = global_ns();
        while (global_ns() - t0 < 200000ull) {
        }
    }
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                     : "memory");
    }
}

// Diagnostics: the bounded wait of the kernels above, on an mbarrier that
// nothing arrives on (arrive == 0) or that thread 0 completes first
// (arrive != 0); a wait that runs out records LH_ERR_TIMEOUT in the workspace
// header like hessian_tc_kernel does.
__global__ void wait_timeout_kernel(int* err, uint64_t timeout_ns, int arrive) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        mbar_init_fence();
    }
    __syncthreads();
    if (arrive && threadIdx.x == 0) mbar_arrive(smem_u32(&bar));
    const bool ok = mbar_wait(smem_u32(&bar), 0u, &abort_flag, timeout_ns);
    if (!ok) atomicExch(err, (int)LH_ERR_TIMEOUT);
}

// Builds the chunk table of the grouped case: each group's token range split
// into chunks of `chunk` tokens; kfirst[g] = first chunk of group g.
__global__ void chunk_table_kernel(const int64_t* __restrict__ offsets, int64_t G, int64_t n_tok, int64_t chunk,
                                   int64_t max_chunks, Chunk* __restrict__ table, int32_t* __restrict__ kfirst,
                                   int32_t* __restrict__ n_chunks_out, int* __restrict__ status) {
    __shared__ int64_t scan[1024];
    __shared__ int64_t base_s;
    const int tid = threadIdx.x;
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");  // the main kernel may set up meanwhile
    if (tid == 0) base_s = 0;
    __syncthreads();
    for (int64_t g0 = 0; g0 < G; g0 += blockDim.x) {
        const int64_t g = g0 + tid;
        int64_t lo = 0, hi = 0, cnt = 0;
        if (g < G) {
            lo = min(max(offsets[g], (int64_t)0), n_tok);
            hi = min(max(offsets[g + 1], lo), n_tok);
            cnt = (hi - lo + chunk - 1) / chunk;
        }
        scan[tid] = cnt;
        __syncthreads();
        for (int off = 1; off < (int)blockDim.x; off <<= 1) {  // inclusive Hillis-Steele scan
            const int64_t v = tid >= off ? scan[tid - off] : 0;
            __syncthreads();
            scan[tid] += v;
            __syncthreads();
        }
        const int64_t base = base_s;
        const int64_t first = base + scan[tid] - cnt;
        if (g < G) {
            kfirst[g] = (int32_t)min(first, max_chunks);
            for (int64_t c = 0; c < cnt && first + c < max_chunks; ++c) {
                Chunk ch;
                ch.start = lo + c * chunk;
                ch.len = (int32_t)min(chunk, hi - ch.start);
                ch.group = (int32_t)g;
                table[first + c] = ch;
            }
        }
        __syncthreads();
        if (tid == (int)blockDim.x - 1) base_s = base + scan[tid];
        __syncthreads();
    }
    if (tid == 0) {
        const int64_t n = min(base_s, max_chunks);
        kfirst[G] = (int32_t)n;
        *n_chunks_out = (int32_t)n;
        // only overlapping (decreasing) offsets hold more chunks than the bound; the chunks
        // past it are dropped and the call reports it
        if (base_s > max_chunks) atomicExch(status, (int)LH_ERR_INVALID_ARG);
    }
}

// H[g][j][e] = fp32(H[g][j][e] + sum_{k in chunks of g} partial[k][j][e]) in FP64, chunk order.
// One block per group and `cols` (8) block columns: each thread keeps 8 independent
// sums, so the loads of a chunk are in flight together (many groups, few chunks each).
__global__ void __launch_bounds__(256) hessian_reduce_kernel(const float* __restrict__ partial,
                                                             const int32_t* __restrict__ kfirst, int64_t J,
                                                             int64_t n_chunks_plain, int cols,
                                                             float* __restrict__ H) {
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the partials of the kernel before
    const int64_t j0 = (int64_t)blockIdx.x * cols;
    const int64_t g = blockIdx.y;
    const int e = threadIdx.x;
    int64_t k0, k1;
    if (kfirst) { k0 = kfirst[g]; k1 = kfirst[g + 1]; }
    else { k0 = 0; k1 = n_chunks_plain; }
    if (k1 <= k0) return;
    const int nj = (int)min((int64_t)cols, J - j0);
    float* h = H + ((size_t)g * J + j0) * 256 + e;
    double hs[8], acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        hs[i] = i < nj ? (double)h[i * 256] : 0.0;
        acc[i] = 0.0;
    }
    for (int64_t k = k0; k < k1; ++k) {
        const float* src = partial + ((size_t)k * J + j0) * 256 + e;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i < nj) acc[i] += (double)src[i * 256];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (i < nj) h[i * 256] = (float)(hs[i] + acc[i]);
}


// The same with one block column per block (one group: enough blocks to fill the GPU).
__global__ void __launch_bounds__(256) hessian_reduce1_kernel(const float* __restrict__ partial,
                                                              const int32_t* __restrict__ kfirst, int64_t J,
                                                              int64_t n_chunks_plain, float* __restrict__ H) {
    asm volatile("griddepcontrol.wait;" ::: "memory");  // the partials of the kernel before
    const int64_t j = blockIdx.x;
    const int64_t g = blockIdx.y;
    const int e = threadIdx.x;
    int64_t k0, k1;
    if (kfirst) { k0 = kfirst[g]; k1 = kfirst[g + 1]; }
    else { k0 = 0; k1 = n_chunks_plain; }
    if (k1 <= k0) return;
    double s = 0.0;
    for (int64_t k = k0; k < k1; ++k) s += (double)partial[((size_t)k * J + j) * 256 + e];
    float* h = H + ((size_t)g * J + j) * 256 + e;
    *h = (float)((double)*h + s);
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
    if (n_tokens_total < 0 || c_in <= 0 || n_groups < 1) return 0;
    return lh::make_plan(n_tokens_total, c_in, n_groups).ws.total;
}

extern "C" lh_status lh_workspace_status(const void* workspace, void* stream) {
    using namespace lh;
    clear_error();
    if (!workspace) return fail(LH_ERR_INVALID_ARG, "null workspace");
    int err = 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    lh_status s = cuda_status(cudaMemcpyAsync(&err, workspace, sizeof(int), cudaMemcpyDeviceToHost, st),
                              "read workspace status");
    if (s != LH_OK) return s;
    s = cuda_status(cudaStreamSynchronize(st), "synchronise");
    if (s != LH_OK) return s;
    if (err == LH_ERR_TIMEOUT) return fail(LH_ERR_TIMEOUT, "a bounded wait in the Hessian kernel expired");
    if (err != 0)
        return fail((lh_status)err, "the group offsets overlap: their ranges hold more tokens than n_tokens_total");
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
    lh_status s = cuda_status(cudaMemsetAsync(workspace, 0, kHeaderBytes, st), "clear workspace header");
    if (s != LH_OK) return s;
    wait_timeout_kernel<<<1, 32, 0, st>>>(static_cast<int*>(workspace), (uint64_t)timeout_us * 1000ull, arrive);
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
    const Plan plan = make_plan(n_tokens_total, c_in, n_groups);
    if (!workspace || workspace_bytes < plan.ws.total)
        return fail(LH_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", plan.ws.total,
                    workspace ? workspace_bytes : (size_t)0);
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(LH_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
    const int sms = sm_count();
    if (sms <= 0) return fail(LH_ERR_CUDA, "no CUDA device");
    auto encode = get_encode_fn();
    if (!encode) return fail(LH_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");

    CUtensorMap tmap;
    const cuuint64_t dims[2] = {(cuuint64_t)c_in, (cuuint64_t)n_tokens_total};
    const cuuint64_t strides[1] = {(cuuint64_t)(ld_x * 2)};
    const cuuint32_t box[2] = {64, (cuuint32_t)kStageTok};
    const cuuint32_t estr[2] = {1, 1};
    CUresult cr = encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(X), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return fail(LH_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)cr);

    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    s = cuda_status(cudaMemsetAsync(ws, 0, kHeaderBytes, st), "clear workspace header");
    if (s != LH_OK) return s;

    const int64_t J = c_in / 16;
    KParams kp;
    kp.n_tok = n_tokens_total;
    kp.J = J;
    kp.n_slabs = plan.n_slabs;
    kp.chunk = plan.chunk;
    kp.n_items_max = plan.max_chunks * plan.n_slabs;
    kp.grouped = offsets != nullptr;
    kp.table = reinterpret_cast<const Chunk*>(ws + plan.ws.table_off);
    kp.n_chunks_dev = reinterpret_cast<const int32_t*>(ws + 4);
    kp.partial = reinterpret_cast<float*>(ws + plan.ws.partial_off);
    kp.err = reinterpret_cast<int*>(ws);
    int32_t* kfirst = reinterpret_cast<int32_t*>(ws + plan.ws.kfirst_off);

    if (offsets) {
        chunk_table_kernel<<<1, 1024, 0, st>>>(offsets, n_groups, n_tokens_total, plan.chunk, plan.max_chunks,
                                               reinterpret_cast<Chunk*>(ws + plan.ws.table_off), kfirst,
                                               reinterpret_cast<int32_t*>(ws + 4), reinterpret_cast<int*>(ws));
        s = cuda_status(cudaGetLastError(), "chunk_table_kernel launch");
        if (s != LH_OK) return s;
    }

    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    const size_t smem_bytes = (size_t)kStages * kStageBytes + 1024 + 256;
    std::call_once(attr_once, [&] {
        attr_err = cudaFuncSetAttribute(hessian_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes);
    });
    if (attr_err != cudaSuccess) return cuda_status(attr_err, "set shared memory size");
    int64_t grid = kp.n_items_max < 2 * sms ? kp.n_items_max : 2 * sms;  // two CTAs per SM
    {
        // programmatic launch: the set-up of its blocks overlaps the end of the kernel before
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem_bytes;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        s = cuda_status(cudaLaunchKernelEx(&cfg, hessian_tc_kernel, tmap, kp), "hessian_tc_kernel launch");
    }
    if (s != LH_OK) return s;

    const int64_t plain_chunks = (n_tokens_total + plan.chunk - 1) / plan.chunk;
    {
        // launched as a programmatic dependent of the main kernel: its blocks start while
        // that kernel drains and wait (griddepcontrol.wait) for its partial sums
        const int cols = (n_groups * ((J + 7) / 8) >= 4 * (int64_t)sms) ? 8 : 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)((J + cols - 1) / cols), (unsigned)n_groups);
        cfg.blockDim = dim3(256);
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const float* part = kp.partial;
        const int32_t* kf = offsets ? kfirst : nullptr;
        s = cols == 1 ? cuda_status(cudaLaunchKernelEx(&cfg, hessian_reduce1_kernel, part, kf, J, plain_chunks, H),
                                    "hessian_reduce1_kernel launch")
                      : cuda_status(cudaLaunchKernelEx(&cfg, hessian_reduce_kernel, part, kf, J, plain_chunks, cols, H),
                        "hessian_reduce_kernel launch");
    }
    return s;
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
// any stream capture. All calls share the one array: the header words that
// must start at zero are cleared by every call, and calls whose kernels
// overlap on the GPU (different streams, or different host threads) race on
// the array and must be serialised by the caller.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocScratchBytes = (size_t)16 << 20;  // 16 MiB
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};
}  // namespace

static __device__ __align__(256) unsigned char lh_noalloc_scratch[kNoAllocScratchBytes];

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
    if (need > kNoAllocScratchBytes)
        return fail(LH_ERR_WORKSPACE,
                    "this Hessian needs %zu bytes of scratch but the allocation-free entry point has %zu "
                    "(16 MiB); call lh_accumulate_hessian with a caller-provided workspace instead",
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
