// indexer.cu -- the sparse indexer that produces the decode's index lists:
// one score per context position on the tensor cores, then the top-k
// positions of each request.
//
// Page "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
// section "Four-bit caches make room": a sparse indexer picks the cache rows
// each token's attention reads and hands over a list of 2,048 positions.  The
// scoring form is a reading (the lightning indexer of DeepSeek sparse
// attention):
//   I[t, p] = sum_h w[t, h] * max(0, q[t, h, :] . k[slot(t, p), :])
// 64 heads x 128 dims, q and k E4M3, w FP32, slot(t, p) through the request's
// block table.  The list holds the top min(topk, ctx) positions (equal scores
// by increasing position) in increasing position order, padded with -1.
//
// Scores (indexer_score_kernel).  Context positions are the M dimension of
// an FP8 tcgen05 MMA (M = 128 positions per tile), heads the N dimension
// (N = 64), the 128 dims the K dimension (four K = 32 steps):
//   S^T[p, h] = K[p, 0:128] . Q[h, 0:128]      (E4M3 x E4M3 -> FP32 in TMEM)
// Key pages arrive by TMA (box = min(page, 128) rows x 128 bytes, 128-byte
// swizzle) into a 2-stage ring; the epilogue reads one TMEM lane (one
// position) per thread and folds the 64 heads with ReLU and the weights.
// The work is HBM-bound (128 key bytes per position against 16K FLOP), but
// each CTA's chain (copy -> MMA -> epilogue) handles about one tile per
// microsecond whatever its depth, so the keys stream best from many short
// pipelines: four CTAs per SM, each with a copy warp, an MMA warp and four
// epilogue warps and double-buffered accumulators (2 x 64 TMEM columns).
//
// Selection (indexer_topk_kernel): up to 8 CTAs share a request's score row.
// Each copies its part into shared memory, takes a threshold from a sample
// of it, marks the positions at or above it in one pass and publishes them
// in position order; the last CTA to arrive (an atomic counter, nobody
// waits) selects exactly among them and writes the list in increasing
// position order.  If a threshold missed, that CTA falls back to binned or
// radix passes over the whole row.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>

#include "common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace nvfp4mla {
namespace idx {

using namespace ptx;

constexpr int kHeads = NVFP4MLA_INDEX_HEADS;   // 64
constexpr int kDimI = NVFP4MLA_INDEX_DIM;      // 128 (bytes per key row)
constexpr int kTile = 128;                     // positions per tile (MMA M)
constexpr int kStages = 2;
constexpr int kThreads = 192;                  // warp 0 copies, warp 1 MMA + TMEM, warps 2-5 epilogue
constexpr int kCtasPerSm = 4;                  // 4 x 128 TMEM columns = all 512
constexpr int kStageBytes = kTile * kDimI;     // 16 KB
constexpr int kOffQ = 0;                       // 64 x 128 B
constexpr int kOffStage = 8192;
constexpr int kOffW = kOffStage + kStages * kStageBytes;
enum { BAR_FULL = 0, BAR_EMPTY = kStages, BAR_TFULL = 2 * kStages, BAR_TEMPTY = 2 * kStages + 2,
       BAR_Q = 2 * kStages + 4, BAR_DRAIN = 2 * kStages + 5, kNumBars = 2 * kStages + 6 };
constexpr int kOffBar = kOffW + kHeads * 4;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16 + 1024;   // + slack to align the base to 1 KB
constexpr uint32_t kTmemCols = 128;                 // two 64-column accumulators
static_assert(kCtasPerSm * kTmemCols <= 512, "TMEM of the resident CTAs");
static_assert(kOffStage % 1024 == 0 && kStageBytes % 1024 == 0, "swizzled tiles need 1 KB alignment");

struct ScoreArgs {
    const float *w;            // [T, 64]
    const int32_t *table;      // [T, table_stride]
    int64_t table_stride;
    int page_shift;            // log2 page size
    int box_shift;             // log2 rows per key copy = min(page_shift, 7)
    const int32_t *ctx_lens;   // [T]
    int max_ctx;
    int64_t num_slots;
    float *scores;             // [T, score_stride]
    int64_t score_stride;
    int32_t *dev_status;
};

__device__ __forceinline__ uint8_t *align1k(uint8_t *p) {
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ void flag(int32_t *st, int bit) {
    if (st) atomicOr(st, bit);
}

// First slot of the key copy that holds position p0 (p0 a multiple of the
// copy size), or -1 when the table entry is empty or the copy would leave
// the cache.
__device__ __forceinline__ int64_t copy_row(const ScoreArgs &a, int t, int p0) {
    const int32_t blk = __ldg(a.table + (int64_t)t * a.table_stride + (p0 >> a.page_shift));
    if (blk < 0) return -1;
    const int64_t y = ((int64_t)blk << a.page_shift) + (p0 & ((1 << a.page_shift) - 1));
    return (y + (1 << a.box_shift) <= a.num_slots) ? y : -1;
}

__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    indexer_score_kernel(const ScoreArgs a, const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = align1k(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int t = blockIdx.y;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + kOffMisc);
    float *w_s = reinterpret_cast<float *>(smem + kOffW);

    int ctx = __ldg(a.ctx_lens + t);
    if (ctx < 0 || ctx > a.max_ctx) {
        if (tid == 0 && blockIdx.x == 0) flag(a.dev_status, NVFP4MLA_DEV_BAD_INDEX);
        ctx = ctx < 0 ? 0 : a.max_ctx;
    }
    const int ntiles = (ctx + kTile - 1) / kTile;
    const int first = blockIdx.x;
    const int n = first < ntiles ? (ntiles - first + (int)gridDim.x - 1) / (int)gridDim.x : 0;
    if (n == 0) return;  // the whole CTA leaves before any barrier or TMEM use

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&bars[BAR_FULL + s], 1);
            mbar_init(&bars[BAR_EMPTY + s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars[BAR_TFULL + b], 1);
            mbar_init(&bars[BAR_TEMPTY + b], 4);  // one arrival per epilogue warp
        }
        mbar_init(&bars[BAR_Q], 1);
        mbar_init(&bars[BAR_DRAIN], 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&misc[0], kTmemCols);
        tmem_relinquish();
    }
    if (tid < kHeads) w_s[tid] = __ldg(a.w + (int64_t)t * kHeads + tid);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    bool ok = true;

    if (warp == 0) {
        // ------------------------------------------------------ key copies
        if (lane == 0) {
            mbar_arrive_expect_tx(&bars[BAR_Q], kHeads * kDimI);
            tma_load_2d(smem + kOffQ, &tm_q, 0, t * kHeads, &bars[BAR_Q]);
            const int box = 1 << a.box_shift;
            const int ncopies = kTile >> a.box_shift;  // 1..16
            bool bad = false;
            int i = 0;
            for (; i < n; ++i) {
                const int s = i % kStages;
                if (i >= kStages && !mbar_wait(&bars[BAR_EMPTY + s], ((i / kStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                const int tile = first + i * (int)gridDim.x;
                uint32_t bytes = 0;
                for (int j = 0; j < ncopies; ++j) {
                    const int p0 = tile * kTile + j * box;
                    if (p0 >= ctx) break;
                    const int64_t y = copy_row(a, t, p0);
                    if (y >= 0) bytes += (uint32_t)(box * kDimI);
                    else bad = true;
                }
                mbar_arrive_expect_tx(&bars[BAR_FULL + s], bytes);
                uint8_t *dst = smem + kOffStage + s * kStageBytes;
                for (int j = 0; j < ncopies; ++j) {
                    const int p0 = tile * kTile + j * box;
                    if (p0 >= ctx) break;
                    const int64_t y = copy_row(a, t, p0);
                    if (y >= 0) tma_load_2d(dst + j * box * kDimI, &tm_k, 0, (int32_t)y, &bars[BAR_FULL + s]);
                }
            }
            if (bad) flag(a.dev_status, NVFP4MLA_DEV_BAD_INDEX);
            // Leave no copy in flight: wait for the last stages' copies.
            for (int j = i > kStages ? i - kStages : 0; j < i; ++j)
                if (!mbar_wait(&bars[BAR_FULL + j % kStages], (j / kStages) & 1)) ok = false;
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA
        if (lane == 0) {
            const uint32_t idesc = idesc_e4m3_f32(kTile, kHeads);
            const uint64_t dq = smem_desc(smem_u32(smem + kOffQ), 16, 1024);
            ok = mbar_wait(&bars[BAR_Q], 0);
            for (int i = 0; i < n && ok; ++i) {
                const int s = i % kStages, b = i & 1;
                if (!mbar_wait(&bars[BAR_FULL + s], (i / kStages) & 1)) {
                    ok = false;
                    break;
                }
                if (i >= 2 && !mbar_wait(&bars[BAR_TEMPTY + b], ((i >> 1) - 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t dk = smem_desc(smem_u32(smem + kOffStage + s * kStageBytes), 16, 1024);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)  // 32 bytes of K per step: +2 in the >>4 address field
                    mma_ss_f8(tmem + b * 64, dk + 2 * kk, dq + 2 * kk, idesc, kk > 0 ? 1u : 0u);
                mma_commit(&bars[BAR_EMPTY + s]);
                mma_commit(&bars[BAR_TFULL + b]);
            }
            // Leave no MMA in flight before TMEM is released.
            mma_commit(&bars[BAR_DRAIN]);
            if (!mbar_wait(&bars[BAR_DRAIN], 0)) ok = false;
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int wq = warp & 3;  // TMEM lanes 32*wq .. 32*wq+31
        const int row = 32 * wq + lane;
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        const int box = 1 << a.box_shift;
        const int32_t *trow = a.table + (int64_t)t * a.table_stride;
        // block-table entry of this thread's position in tile i, read one
        // tile ahead so the load is off the per-tile critical path
        auto entry = [&](int i) -> int32_t {
            const int p = (first + i * (int)gridDim.x) * kTile + row;
            return (i < n && p < ctx) ? __ldg(trow + (p >> a.page_shift)) : -1;
        };
        int32_t blk = entry(0);
        for (int i = 0; i < n; ++i) {
            const int b = i & 1;
            const int32_t blk_next = entry(i + 1);
            const bool got = mbar_wait(&bars[BAR_TFULL + b], (i >> 1) & 1);
            if (!__all_sync(0xffffffffu, got)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t r0[32], r1[32];
            tmem_ld32(tmem + lane_base + b * 64, r0);
            tmem_ld32(tmem + lane_base + b * 64 + 32, r1);
            tmem_ld_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[BAR_TEMPTY + b]);
            // four independent accumulation chains over the heads
            float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int h = 0; h < 32; h += 4) {
                const float4 wv = *reinterpret_cast<const float4 *>(w_s + h);
                acc[0] = fmaf(wv.x, fmaxf(__uint_as_float(r0[h]), 0.0f), acc[0]);
                acc[1] = fmaf(wv.y, fmaxf(__uint_as_float(r0[h + 1]), 0.0f), acc[1]);
                acc[2] = fmaf(wv.z, fmaxf(__uint_as_float(r0[h + 2]), 0.0f), acc[2]);
                acc[3] = fmaf(wv.w, fmaxf(__uint_as_float(r0[h + 3]), 0.0f), acc[3]);
            }
#pragma unroll
            for (int h = 0; h < 32; h += 4) {
                const float4 wv = *reinterpret_cast<const float4 *>(w_s + 32 + h);
                acc[0] = fmaf(wv.x, fmaxf(__uint_as_float(r1[h]), 0.0f), acc[0]);
                acc[1] = fmaf(wv.y, fmaxf(__uint_as_float(r1[h + 1]), 0.0f), acc[1]);
                acc[2] = fmaf(wv.z, fmaxf(__uint_as_float(r1[h + 2]), 0.0f), acc[2]);
                acc[3] = fmaf(wv.w, fmaxf(__uint_as_float(r1[h + 3]), 0.0f), acc[3]);
            }
            const float score = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            const int p = (first + i * (int)gridDim.x) * kTile + row;
            if (p < ctx) {
                // a position whose key copy was refused (empty table entry or
                // a page outside the cache) scores -inf
                const int p0 = p & ~(box - 1);
                const int64_t y = ((int64_t)blk << a.page_shift) + (p0 & ((1 << a.page_shift) - 1));
                const bool valid = blk >= 0 && y + box <= a.num_slots;
                a.scores[(int64_t)t * a.score_stride + p] = valid ? score : -INFINITY;
            }
            blk = blk_next;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
    if (!ok) flag(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
}

// ------------------------------------------------------------------ top-k
// Each request's score row is shared by P CTAs of 1024 threads (P chosen so
// the grid fills the SMs, at most 8); CTA p owns a contiguous part of the
// row (P nearly equal parts, multiples of 128 positions).
//
// Usual path:
//   0. at launch, a part of at most kSliceCap positions is bulk-copied into
//      shared memory (nine 16 KB copies, one mbarrier counting the bytes);
//   1. a threshold tau: a median of group maxima over 8192 sampled keys
//      (group_median_key) chosen so that about 1.4 x topk positions or more
//      score at or above it -- sampled from the CTA's own part when it sits
//      in shared memory, else from whole 32-position lines of the row (the
//      same sample in every CTA; sample_threshold when no group size fits);
//   2. one pass marks the part's positions with score >= tau, each thread
//      owning a run of consecutive positions, and one block scan orders
//      them; the CTA publishes them, their count, its tau and its largest
//      candidate key in the workspace;
//   3. the last CTA of the request to arrive on its counter (an atomic add;
//      nobody waits) concatenates the P lists -- again in position order --
//      and, if topk <= m <= kCandCap candidates were found, finds the
//      topk-th largest key exactly (select_fast over the published key
//      range); if that key is at or above every part's tau, every position
//      at or above it was collected, and the CTA writes the list.
// Otherwise (too few or too many candidates, or a key below some part's
// tau) that last CTA runs the general path over the whole row alone,
// streaming it through a ring of three 32 KB buffers (the area of step 0):
//   A  min and max of the finite scores;
//   B  histogram of a linear binning of [min, max] into 2048 bins (monotone
//      in the score: bins above the one holding the topk-th largest score,
//      d*, are taken whole);
//   C  the scores of bin d* are collected and an exact radix select among
//      them gives the threshold key and the number of ties taken;
//   D  the ordered write: per 8192-position chunk warp w takes positions
//      256w .. 256w+255, two scans over the warps give its first tie rank
//      and first output slot, and ballots place the chosen positions;
// and when even that binning fails (all equal scores, fewer finite scores
// than topk, too many in bin d*), a three-digit radix select over the whole
// row replaces A-C.
constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;
static_assert(kTopkWarps == 32, "one warp reduces the per-warp minima and maxima");
constexpr int kBins = 2048;
constexpr int kChunk = 8192;  // floats per streamed chunk
constexpr int kRing = 3;
constexpr int kCandCap = 8192;    // 4 x the largest topk
constexpr int kMaxParts = 8;
// A CTA's part of the row, when it holds at most kSliceCap positions, is
// bulk-copied into shared memory at launch (the area the general path later
// uses as its ring), so the collect pass reads it there.
constexpr int kSliceCap = 36 * kTopkThreads;  // 36 positions per thread
constexpr int kAreaBytes = kSliceCap * 4 > kRing * kChunk * 4 ? kSliceCap * 4 : kRing * kChunk * 4;
constexpr int kSlicePiece = 4096;  // positions per bulk copy of the part
constexpr int kTopkDynSmem = kAreaBytes + kCandCap * 8;  // 216 KB
static_assert(kCandCap >= 8192, "the sampled keys (at most 8192) share the candidate area");
static_assert(kChunk == kTopkWarps * 256, "pass D gives each warp 256 positions of a chunk");

struct TopkArgs {
    const float *scores;
    int64_t score_stride;
    const int32_t *ctx_lens;
    int max_ctx;
    int topk;
    int32_t *out;
    int parts;           // P: CTAs per request
    uint32_t *arrivals;  // [T] arrival counters (zero between launches)
    uint4 *counts;       // [T][P] per CTA: candidates found, its threshold key, its largest candidate key
    uint2 *cand;         // [T][P][kCandCap] (key, position) in position order
    int32_t *dev_status;
};

// Order-preserving unsigned key of a score; -0 is first turned into +0 so
// the two zeros tie.
__device__ __forceinline__ uint32_t score_key(float f) {
    const uint32_t u = __float_as_uint(f + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive prefix sum over the 1024 threads of the block (scratch: 32 words).
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, uint32_t *scratch) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    if (lane == 31) scratch[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t x = scratch[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        scratch[lane] = x;
    }
    __syncthreads();
    const uint32_t before = warp > 0 ? scratch[warp - 1] : 0u;
    __syncthreads();  // scratch may be reused right after
    return v + before;
}

// Exclusive scan of one value per warp (lane 0's `v`); returns this warp's
// exclusive prefix and the block total.  Every thread calls it.
__device__ __forceinline__ uint32_t warp_excl_scan(uint32_t v, uint32_t *slots, uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) slots[warp] = v;
    __syncthreads();
    if (warp == 0) {
        const uint32_t x = slots[lane];
        uint32_t incl = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        slots[lane] = incl - x;
        if (lane == 31) *total = incl;
    }
    __syncthreads();
    return slots[warp];
}

// Given a 1024- or 2048-bin histogram and want >= 1 items to take from the
// top: out[0] = the bin holding the want-th largest item, out[1] = how many
// of its items are taken, out[2] = the total count.  Every thread calls it.
__device__ __forceinline__ void find_bin(const uint32_t *hist, int nb, uint32_t want, uint32_t *scratch,
                                         uint32_t *out) {
    const int tid = threadIdx.x;
    uint32_t c_hi = 0, c_lo = 0;
    if (2 * tid < nb) {
        c_hi = hist[nb - 1 - 2 * tid];
        c_lo = hist[nb - 2 - 2 * tid];
    }
    const uint32_t incl = block_incl_scan(c_hi + c_lo, scratch);
    const uint32_t before = incl - c_hi - c_lo;
    if (2 * tid < nb) {
        if (want > before && want <= before + c_hi) {
            out[0] = (uint32_t)(nb - 1 - 2 * tid);
            out[1] = want - before;
        } else if (want > before + c_hi && want <= incl) {
            out[0] = (uint32_t)(nb - 2 - 2 * tid);
            out[1] = want - before - c_hi;
        }
    }
    if (tid == kTopkThreads - 1) out[2] = incl;
    __syncthreads();
}

__device__ __forceinline__ void add_to_hist(uint32_t *hist, uint32_t d, int lane) {
    // d == 0xFFFFFFFF: nothing to add; equal digits in a warp add once
    const uint32_t peers = __match_any_sync(0xffffffffu, d);
    if (d != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (uint32_t)__popc(peers));
}

__device__ __forceinline__ uint32_t radix_digit(uint32_t k, int pass, uint32_t prefix) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int bits = pass == 2 ? 10 : 11;
    const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + bits));
    return (k & hi_mask) == prefix ? (k >> shift) & ((1u << bits) - 1u) : 0xFFFFFFFFu;
}

// The want-th largest of n keys in shared memory (want <= n): returns the
// key; *ties = how many keys equal to it are taken.  Every thread calls it.
__device__ uint32_t select_in_smem(const uint32_t *keys, uint32_t n, uint32_t want, uint32_t *hist,
                                   uint32_t *scratch, uint32_t *found, uint32_t *ties) {
    const int tid = threadIdx.x, lane = tid & 31;
    uint32_t prefix = 0, remaining = want;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        for (int i = tid; i < kBins; i += kTopkThreads) hist[i] = 0;
        __syncthreads();
        for (uint32_t base = 0; base < n; base += kTopkThreads) {
            const uint32_t i = base + tid;
            add_to_hist(hist, i < n ? radix_digit(keys[i], pass, prefix) : 0xFFFFFFFFu, lane);
        }
        __syncthreads();
        find_bin(hist, pass == 2 ? 1024 : 2048, remaining, scratch, found);
        prefix |= found[0] << (pass == 0 ? 21 : (pass == 1 ? 10 : 0));
        remaining = found[1];
        __syncthreads();
    }
    *ties = remaining;
    return prefix;
}

// mm[0], mm[1] = the smallest and largest of n keys in shared memory (n >= 1).
// Every thread calls it; `scratch` and `sub` are 32 words each.
__device__ void block_min_max(const uint32_t *keys, uint32_t n, uint32_t *scratch, uint32_t *sub, uint32_t *mm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    uint32_t lo = 0xFFFFFFFFu, hi = 0u;
    for (uint32_t i = tid; i < n; i += kTopkThreads) {
        const uint32_t k = keys[i];
        lo = min(lo, k);
        hi = max(hi, k);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (lane == 0) {  // per-warp minima and maxima (kTopkWarps == 32)
        scratch[warp] = lo;
        sub[warp] = hi;
    }
    __syncthreads();
    if (warp == 0) {
        lo = scratch[lane];
        hi = sub[lane];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        if (lane == 0) {
            mm[0] = lo;
            mm[1] = hi;
        }
    }
    __syncthreads();
}

// The want-th largest of n keys in shared memory (1 <= want <= n), exactly
// as select_in_smem gives it, usually in one histogram pass: keys are binned
// by (key - min) >> shift, a monotone map onto at most 2048 bins, so every
// bin above the one holding the want-th largest key, b*, is taken whole; the
// few keys of b* (at most 32) are then ranked by one warp.  When b* holds
// more than 32 keys, they are copied to `spill` (room for n keys) and binned
// once more over their own, narrower range; only if that fails too does the
// radix select run, on b*'s keys.  A range below 2048 gives one key per bin,
// so b* itself is the answer.  Keys equal to the result all fall in b*,
// so the ties counted there are the ties overall.  A caller that knows a
// range [lo0, hi0] (lo0 < hi0) holding every key skips the first min/max
// pass.  Every thread calls it; `sub` is 32 words of scratch, `mm` 2.
__device__ uint32_t select_fast(const uint32_t *keys, uint32_t n, uint32_t want, uint32_t *hist, uint32_t *scratch,
                                uint32_t *found, uint32_t *ties, uint32_t *sub, uint32_t *mm, uint32_t *spill,
                                uint32_t lo0 = 1u, uint32_t hi0 = 0u) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
#pragma unroll 1
    for (int level = 0; level < 2; ++level) {
        if (tid == 0) found[0] = 0;  // keys of b* collected so far (below)
        for (int i = tid; i < kBins; i += kTopkThreads) hist[i] = 0;
        if (level == 0 && lo0 < hi0) {  // a range holding every key is known: no min/max pass
            if (tid == 0) {
                mm[0] = lo0;
                mm[1] = hi0;
            }
            __syncthreads();
        } else {
            block_min_max(keys, n, scratch, sub, mm);
        }
        const uint32_t lo = mm[0], hi = mm[1];
        if (lo == hi) {  // all keys equal: the threshold is that key, want of them taken
            *ties = want;
            __syncthreads();  // mm may be reused right after
            return lo;
        }
        const uint32_t range = hi - lo;
        const int shift = max(0, 32 - __clz(range) - 11);  // range >> shift < 2048
        for (uint32_t i = tid; i < n; i += kTopkThreads) atomicAdd(&hist[(keys[i] - lo) >> shift], 1u);
        __syncthreads();
        find_bin(hist, kBins, want, scratch, found + 1);  // found[1] = b*, found[2] = taken from b*
        const uint32_t bstar = found[1], within = found[2], cnt = hist[bstar];
        if (shift == 0) {  // one key per bin: b* is the threshold, within of its keys taken
            *ties = within;
            __syncthreads();  // found and hist may be reused right after
            return lo + bstar;
        }
        if (cnt <= 32u) {
            for (uint32_t i = tid; i < n; i += kTopkThreads) {
                const uint32_t k = keys[i];
                if (((k - lo) >> shift) == bstar) sub[atomicAdd(&found[0], 1u)] = k;
            }
            __syncthreads();
            if (warp == 0) {
                // lane i holds key i of b* (if any); the want-th largest overall is
                // the within-th largest of b*: the key v with #(> v) < within <= #(>= v)
                const uint32_t v = lane < (int)cnt ? sub[lane] : 0u;
                uint32_t gt = 0, ge = 0;
                for (uint32_t j = 0; j < cnt; ++j) {
                    const uint32_t u = __shfl_sync(0xffffffffu, v, j);
                    gt += u > v;
                    ge += u >= v;
                }
                const bool hit = lane < (int)cnt && gt < within && within <= ge;
                const uint32_t who = __ballot_sync(0xffffffffu, hit);
                if (lane == __ffs(who) - 1) {
                    mm[0] = v;
                    mm[1] = within - gt;
                }
            }
            __syncthreads();
            *ties = mm[1];
            const uint32_t thr = mm[0];
            __syncthreads();  // mm, sub and found may be reused right after
            return thr;
        }
        if (level == 1) {  // the radix select below, over the keys spilled at level 0
            __syncthreads();  // every thread has read hist[b*]
            break;
        }
        // b*'s keys, on their own: the within-th largest of them
        for (uint32_t i = tid; i < n; i += kTopkThreads) {
            const uint32_t k = keys[i];
            if (((k - lo) >> shift) == bstar) spill[atomicAdd(&found[0], 1u)] = k;
        }
        __syncthreads();
        keys = spill;
        n = cnt;
        want = within;
    }
    return select_in_smem(keys, n, want, hist, scratch, found, ties);
}

// Score of a key (inverse of score_key).
__device__ __forceinline__ float key_score(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// A sampling threshold: a key tau with at least r of the n keys >= tau and
// few more (key 0 marks an empty sample and is never counted).  One pass
// over a linear binning of the scores' range into 2048 bins (monotone in the
// score), tau = the smallest key in the bin holding the r-th largest score,
// so every key of that bin and the bins above is >= tau.  Falls back to the
// exact radix select when the binning cannot be formed (fewer than r finite
// scores, all equal).  Every thread calls it; `sub` is 32 words, `mm` 2.
__device__ uint32_t sample_threshold(const uint32_t *keys, uint32_t n, uint32_t r, uint32_t *hist,
                                     uint32_t *scratch, uint32_t *found, uint32_t *sub, uint32_t *mm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    float lo = INFINITY, hi = -INFINITY;
    for (uint32_t i = tid; i < n; i += kTopkThreads) {
        const uint32_t k = keys[i];
        const float x = key_score(k);
        if (k != 0u && x > -INFINITY && x < INFINITY) {
            lo = fminf(lo, x);
            hi = fmaxf(hi, x);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (lane == 0) {
        scratch[warp] = __float_as_uint(lo);
        sub[warp] = __float_as_uint(hi);
    }
    for (int i = tid; i < kBins; i += kTopkThreads) hist[i] = 0;
    __syncthreads();
    if (warp == 0) {
        lo = __uint_as_float(scratch[lane]);
        hi = __uint_as_float(sub[lane]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
            hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        }
        if (lane == 0) {
            mm[0] = __float_as_uint(lo);
            mm[1] = __float_as_uint(hi);
        }
    }
    __syncthreads();
    lo = __uint_as_float(mm[0]);
    hi = __uint_as_float(mm[1]);
    const float scale = (float)kBins / (hi - lo);
    const bool binned = hi > lo && scale > 0.0f && scale < INFINITY;  // block-uniform
    auto bin = [&](uint32_t k) -> int {
        const float x = key_score(k);
        if (k == 0u || !(x > -INFINITY && x < INFINITY)) return -1;
        const int b = (int)((x - lo) * scale);
        return b < kBins - 1 ? b : kBins - 1;
    };
    if (binned) {
        for (uint32_t i = tid; i < n; i += kTopkThreads) {
            const int b = bin(keys[i]);
            if (b >= 0) atomicAdd(&hist[b], 1u);
        }
        __syncthreads();
        find_bin(hist, kBins, r, scratch, found);
    }
    if (!binned || found[2] < r) {  // block-uniform: the exact select
        __syncthreads();
        uint32_t unused;
        return select_in_smem(keys, n, r, hist, scratch, found, &unused);
    }
    const int bstar = (int)found[0];
    uint32_t kmin = 0xFFFFFFFFu;
    for (uint32_t i = tid; i < n; i += kTopkThreads) {
        const uint32_t k = keys[i];
        if (bin(k) == bstar) kmin = min(kmin, k);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
    __syncthreads();  // find_bin's readers of scratch are done
    if (lane == 0) scratch[warp] = kmin;
    __syncthreads();
    if (warp == 0) {
        kmin = scratch[lane];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
        if (lane == 0) mm[0] = kmin;
    }
    __syncthreads();
    const uint32_t tau = mm[0];
    __syncthreads();  // mm and scratch may be reused right after
    return tau;
}

// A median of group maxima over 8192 sampled keys (8 per thread, key 0 for
// no sample): groups of G = 8 * lg keys (a lane's 8, then lg lanes); each
// warp takes the lower median of its 256 / G group maxima and the result is
// the 16th smallest of the 32 warps' medians.  For keys drawn from one
// distribution, a share of about ln 2 / G of it lies at or above the median
// of the groups' maxima.  Every thread calls it; `sub` is 32 words, `mm` 1.
__device__ uint32_t group_median_key(const uint32_t (&sk)[8], int G, uint32_t *sub, uint32_t *mm) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int lg = G / 8, ng = 256 / G;  // lanes per group, groups per warp
    uint32_t mx = sk[0];
#pragma unroll
    for (int j = 1; j < 8; ++j) mx = max(mx, sk[j]);
    for (int off = 1; off < lg; off <<= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    // lower median of the warp's ng group maxima (group k led by lane k * lg)
    uint32_t below = 0;
    for (int k = 0; k < ng; ++k) {
        const uint32_t u = __shfl_sync(0xffffffffu, mx, k * lg);
        below += u < mx || (u == mx && k * lg < lane);
    }
    const uint32_t who = __ballot_sync(0xffffffffu, lane % lg == 0 && below == (uint32_t)(ng - 1) / 2);
    const uint32_t med = __shfl_sync(0xffffffffu, mx, __ffs(who) - 1);
    if (lane == 0) sub[warp] = med;
    __syncthreads();
    if (warp == 0) {  // the 16th smallest of the 32 warps' medians
        const uint32_t e = sub[lane];
        uint32_t rank = 0;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const uint32_t u = __shfl_sync(0xffffffffu, e, k);
            rank += u < e || (u == e && k < lane);
        }
        if (rank == 15u) mm[0] = e;
    }
    __syncthreads();
    const uint32_t tau = mm[0];
    __syncthreads();  // sub and mm may be reused right after
    return tau;
}

// Write the list from m candidates held in position order: keys above thr,
// and the first need_eq keys equal to it.
static_assert(kCandCap < 65536, "write_from_candidates packs two counts of at most kCandCap in one word");
__device__ void write_from_candidates(const uint32_t *ck, const int32_t *cp, uint32_t m, uint32_t thr,
                                      uint32_t need_eq, int32_t *o, uint32_t *scratch) {
    const uint32_t tid = threadIdx.x;
    const uint32_t per = (m + kTopkThreads - 1) / kTopkThreads;  // each thread owns a contiguous run
    const uint32_t i0 = min(m, tid * per), i1 = min(m, i0 + per);
    uint32_t above = 0, ties = 0;
    for (uint32_t i = i0; i < i1; ++i) {
        const uint32_t k = ck[i];
        above += k > thr;
        ties += k == thr;
    }
    // one scan of both counts, packed 16 bits each (m <= kCandCap < 65536):
    // the run's first slot is the keys above thr before it plus the ties
    // taken before it
    const uint32_t packed = above | ties << 16;
    const uint32_t ex = block_incl_scan(packed, scratch) - packed;
    uint32_t tie_rank = ex >> 16;
    uint32_t at = (ex & 0xFFFFu) + min(tie_rank, need_eq);
    for (uint32_t i = i0; i < i1; ++i) {
        const uint32_t k = ck[i];
        if (k > thr || (k == thr && tie_rank++ < need_eq)) o[at++] = cp[i];
    }
}

__global__ void __launch_bounds__(kTopkThreads, 1) indexer_topk_kernel(const TopkArgs a) {
    extern __shared__ __align__(128) uint8_t dyn[];
    float *ring = reinterpret_cast<float *>(dyn);
    const float *slice = ring;  // this CTA's part of the row, until the general path
    uint32_t *cand_key = reinterpret_cast<uint32_t *>(dyn + kAreaBytes);
    int32_t *cand_pos = reinterpret_cast<int32_t *>(cand_key + kCandCap);
    __shared__ uint64_t full[kRing + 1];  // the ring's buffers, then the part's copies
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t scratch[32], slots_a[32], slots_b[32];
    __shared__ uint32_t found[4], totals[2], sub32[32], mm2[2];
    __shared__ float red_lo[kTopkWarps], red_hi[kTopkWarps];
    __shared__ uint32_t ncand, cmax, seg_off[kMaxParts + 1];
    __shared__ int last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = blockIdx.y, part = blockIdx.x, P = a.parts;
    const int topk = a.topk;
    int ctx = __ldg(a.ctx_lens + t);
    if (ctx < 0 || ctx > a.max_ctx) {
        if (tid == 0 && part == 0) flag(a.dev_status, NVFP4MLA_DEV_BAD_INDEX);
        ctx = ctx < 0 ? 0 : a.max_ctx;
    }
    int32_t *o = a.out + (int64_t)t * topk;
    if (ctx <= topk) {  // every position, then -1 (no counter is touched)
        if (part == 0)
            for (int i = tid; i < topk; i += kTopkThreads) o[i] = i < ctx ? i : -1;
        return;
    }
    const float *s = a.scores + (int64_t)t * a.score_stride;
    // this CTA's part of the row: P nearly equal ranges, multiples of 128
    const int span = ((ctx + P - 1) / P + 127) / 128 * 128;
    const int r0 = min(ctx, part * span), r1 = min(ctx, r0 + span);
    const bool in_smem = r1 - r0 <= kSliceCap;  // block-uniform
    if (tid == 0) {
        for (int b = 0; b <= kRing; ++b) mbar_init(&full[b], 1);
        fence_mbar_init();
        ncand = 0;
        cmax = 0;
        if (in_smem && r1 > r0) mbar_arrive_expect_tx(&full[kRing], ((uint32_t)(r1 - r0) * 4u + 15u) & ~15u);
    }
    __syncthreads();
    if (in_smem && r1 > r0) {
        // the part's copy, one 16 KB piece per thread of the first warp;
        // whole 16-byte units: r0 is a multiple of 128 floats and the row
        // holds ctx rounded up to 4 floats
        const uint32_t total = ((uint32_t)(r1 - r0) * 4u + 15u) & ~15u;
        const uint32_t off = (uint32_t)tid * kSlicePiece * 4u;
        if (tid < kSliceCap / kSlicePiece && off < total)
            bulk_g2s(ring + off / 4, s + r0 + off / 4, min((uint32_t)kSlicePiece * 4u, total - off), &full[kRing]);
    }
    // false (block-uniform) once the part's copy is in shared memory; true
    // if it never landed within the bounded wait (reported: leave)
    auto slice_lost = [&]() -> bool {
        if (!in_smem || r1 <= r0) return false;
        if (__syncthreads_and(mbar_wait(&full[kRing], 0))) return false;
        if (tid == 0) {  // leave no copy in flight, report
            (void)mbar_wait(&full[kRing], 0);
            flag(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
        }
        return true;
    };

    // ------------------------------------------------------- streaming
    uint32_t seq = 0;     // chunks streamed through the ring so far
    uint32_t issued = 0;  // chunks whose copy has been issued (thread 0)
    bool ok = true;
    // chunk c of the range starting at r0 (r1 = its end)
    auto issue = [&](int r0, int r1, int c) {
        const uint32_t q = seq + (uint32_t)c;
        const int n = min(kChunk, r1 - r0 - c * kChunk);
        // whole 16-byte units; r0 is a multiple of kChunk and the row holds
        // ctx rounded up to 4 floats
        const uint32_t bytes = ((uint32_t)n * 4u + 15u) & ~15u;
        uint64_t *bar = &full[q % kRing];
        mbar_arrive_expect_tx(bar, bytes);
        bulk_g2s(ring + (q % kRing) * kChunk, s + r0 + (int64_t)c * kChunk, bytes, bar);
        issued = q + 1;
    };
    // One pass over [r0, r1): body(chunk data, chunk index, valid floats)
    // for every chunk in order.  Returns false (block-uniformly) if a copy
    // never landed within the bounded wait.
    auto stream = [&](int r0, int r1, auto &&body) -> bool {
        const int nchunks = r1 > r0 ? (r1 - r0 + kChunk - 1) / kChunk : 0;
        if (tid == 0)
            for (int c = 0; c < min(kRing, nchunks); ++c) issue(r0, r1, c);
        for (int c = 0; c < nchunks; ++c) {
            const uint32_t q = seq + (uint32_t)c;
            const bool got = mbar_wait(&full[q % kRing], (q / kRing) & 1);
            if (__syncthreads_or(!got)) {
                seq = q;
                return false;
            }
            body(ring + (q % kRing) * kChunk, c, min(kChunk, r1 - r0 - c * kChunk));
            __syncthreads();
            if (tid == 0 && c + kRing < nchunks) issue(r0, r1, c + kRing);
        }
        seq += (uint32_t)nchunks;
        return true;
    };
    auto fail = [&]() {  // leave no copy in flight, report, leave
        if (tid == 0) {
            for (uint32_t q = seq; q < issued; ++q) (void)mbar_wait(&full[q % kRing], (q / kRing) & 1);
            flag(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
        }
    };

    // ------------------------------------------- 1. sampled threshold tau
    // tau is estimated from 8192 sampled keys (at most), 8 per thread, as a
    // median of group maxima (group_median_key) where a group of G samples
    // fits: G = the largest power of two in [8, 256] with
    // ctx * ln 2 / G >= 1.4 * topk, so about 1.4 x topk or more of the
    // sampled stretch scores at or above tau.  A CTA whose part sits in
    // shared memory and holds at least 8192 positions samples its own part
    // (every (n / 8192)-th position) and keeps its own tau; otherwise every
    // CTA of the request draws the same sample of whole 32-position lines of
    // the row (line i of warp i % 32), and when no G fits or a warp holds
    // fewer than 7 lines, tau comes from a binning of that sample instead
    // (sample_threshold, aiming at 1.25 x topk).  The selecting CTA checks
    // that the exact threshold is at or above every part's tau, so every
    // position at or above it was collected; if not, or if the candidates
    // are fewer than topk or more than fit, the request takes the general
    // path.
    uint32_t tau;
    {
        int G = 0;
        for (int g = 8; g <= 256; g *= 2)
            if ((int64_t)ctx * 693 >= (int64_t)1400 * topk * g) G = g;
        const int n = r1 - r0;
        uint32_t sk[(8192 / 32 + kTopkWarps - 1) / kTopkWarps];
        if (in_smem && n >= 8192 && G > 0) {  // block-uniform
            if (slice_lost()) return;
            const int st = n / 8192;  // 8191 * st < n
#pragma unroll
            for (int j = 0; j < 8; ++j) sk[j] = score_key(slice[(warp * 256 + j * 32 + lane) * st]);
            tau = group_median_key(sk, G, sub32, mm2);
        } else {
            const int64_t lines = ((int64_t)ctx + 31) / 32;
            const int lstride = (int)max((int64_t)1, (lines * 32 + 8191) / 8192);
            const int nsl = (int)((lines + lstride - 1) / lstride);  // sampled lines, <= 256
            const int last_base = (nsl - 1) * lstride * 32;
            const uint32_t S = (uint32_t)((nsl - 1) * 32 + min(32, ctx - last_base));
#pragma unroll
            for (int j = 0; j < 8; ++j) {  // all of a warp's line loads in flight at once
                const int i = warp + kTopkWarps * j;
                const int p = i * lstride * 32 + lane;
                sk[j] = (i < nsl && p < ctx) ? score_key(__ldcg(s + p)) : 0u;  // 0 is below every score's key
            }
            if (G > 0 && nsl >= 7 * kTopkWarps) {  // block-uniform
                tau = group_median_key(sk, G, sub32, mm2);
            } else {
                uint32_t *samp = cand_key;  // free until step 2
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int i = warp + kTopkWarps * j;
                    if (i < nsl) samp[i * 32 + lane] = sk[j];
                }
                const uint32_t r = (uint32_t)min((int64_t)S, (int64_t)topk * S * 5 / (4 * (int64_t)ctx) + 9);
                __syncthreads();
                tau = sample_threshold(samp, (uint32_t)nsl * 32, r, hist, scratch, found, sub32, mm2);
            }
        }
    }

    // ------------------------------- 2. collect this CTA's candidates
    // With P > 1 each candidate also goes straight to this CTA's workspace
    // list as it is found, for the selecting CTA.
    uint2 *const pub_dst = P > 1 ? a.cand + ((int64_t)t * P + part) * kCandCap : nullptr;
    if (slice_lost()) return;
    uint32_t m = 0;  // candidates found in the range (block-uniform; may pass the cap)
    const float tau_f = key_score(tau);  // score >= tau_f  <=>  key >= tau (scores are never NaN)
    if (in_smem) {
        // From the part's copy in shared memory.  Thread i owns the run
        // [i * L, (i + 1) * L) of the part (L / 4 odd, at most 9 float4:
        // the eight lanes of a quarter warp then read 16-byte words in
        // distinct banks), so position order is thread order: one pass marks
        // the run's candidates in a 36-bit mask, one block scan of the
        // counts places the threads, and each thread writes its few
        // candidates.  Reads stay below 1024 * L <= kSliceCap; positions at
        // or past the part's end n are masked.
        const int n = r1 - r0;
        const int l4 = ((n + kTopkThreads - 1) / kTopkThreads + 3) / 4 | 1;  // float4 per thread
        const int base = tid * 4 * l4;
        const float4 *v4 = reinterpret_cast<const float4 *>(slice + base);
        uint64_t hits = 0;
        if (base + 4 * l4 <= n) {  // the whole run lies in the part
#pragma unroll
            for (int i = 0; i < kSliceCap / kTopkThreads / 4; ++i)
                if (i < l4) {
                    const float4 v = v4[i];
                    hits |= (uint64_t)((v.x >= tau_f) | (v.y >= tau_f) << 1 | (v.z >= tau_f) << 2 |
                                       (v.w >= tau_f) << 3)
                            << (4 * i);
                }
        } else {
#pragma unroll
            for (int i = 0; i < kSliceCap / kTopkThreads / 4; ++i)
                if (i < l4) {
                    const float4 v = v4[i];
                    const int q = base + 4 * i;
                    hits |= (uint64_t)((q < n && v.x >= tau_f) | (q + 1 < n && v.y >= tau_f) << 1 |
                                       (q + 2 < n && v.z >= tau_f) << 2 | (q + 3 < n && v.w >= tau_f) << 3)
                            << (4 * i);
                }
        }
        const uint32_t c = (uint32_t)__popcll(hits);
        uint32_t at = block_incl_scan(c, scratch) - c;
        m = scratch[kTopkWarps - 1];  // the block total: warp 0's scan of the warp sums
        uint32_t kmax = 0;
        while (hits) {
            const int b = __ffsll((long long)hits) - 1;
            hits &= hits - 1;
            const uint32_t k = score_key(slice[base + b]);
            if (at < (uint32_t)kCandCap) {
                cand_key[at] = k;
                cand_pos[at] = r0 + base + b;
                if (pub_dst) pub_dst[at] = make_uint2(k, (uint32_t)(r0 + base + b));
            }
            kmax = max(kmax, k);
            ++at;
        }
        kmax = __reduce_max_sync(0xffffffffu, kmax);
        if (lane == 0 && kmax) atomicMax(&cmax, kmax);
        __syncthreads();  // every thread's candidates are written before anyone reads them
    } else {
    // Straight from global memory (the row was just written and sits in
    // L2), in batches of 16K positions: warp w takes the 512 positions
    // [b0 + 512w, b0 + 512w + 512) as J = 4 float4 per lane, load j of lane
    // l covering positions 128j + 4l .. +3 (each load instruction reads 512
    // contiguous bytes; all of a lane's loads are in flight at once).
    // Position order inside a warp is (j, lane, element): the per-lane counts
    // of the four loads, packed 8 bits each into one word, take one warp
    // scan; one block scan of the warp totals places the warps.  A float4
    // that starts below r1 lies in the row, which holds ctx rounded up to 4
    // floats (r0 and span are multiples of 4).
    {
        constexpr int J = 4;
        uint32_t kmax = 0;  // the largest candidate key seen by this thread
        float4 nx[J];  // the next batch's loads, in flight while this one is scanned
        auto load_batch = [&](int b0, float4 (&d)[J]) {
            const int wb = b0 + warp * (32 * 4 * J);
#pragma unroll
            for (int j = 0; j < J; ++j) {
                const int p = wb + 128 * j + 4 * lane;
                d[j] = p < r1 ? __ldcg(reinterpret_cast<const float4 *>(s + p))
                              : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
            }
        };
        if (r0 < r1) load_batch(r0, nx);
#pragma unroll 1
        for (int b0 = r0; b0 < r1; b0 += kTopkThreads * 4 * J) {
            const int wb = b0 + warp * (32 * 4 * J);
            float4 v4[J];
#pragma unroll
            for (int j = 0; j < J; ++j) v4[j] = nx[j];
            if (b0 + kTopkThreads * 4 * J < r1) load_batch(b0 + kTopkThreads * 4 * J, nx);
            // bit 4j+e: position wb + 128j + 4*lane + e is a candidate (its
            // score >= tau's score, the same test as key >= tau for every
            // score but NaN); positions past r1 are tested only in the last,
            // partial batch
            uint32_t sel = 0;
            if (b0 + kTopkThreads * 4 * J <= r1) {  // block-uniform
#pragma unroll
                for (int j = 0; j < J; ++j) {
                    sel |= (v4[j].x >= tau_f ? 1u : 0u) << (4 * j + 0);
                    sel |= (v4[j].y >= tau_f ? 1u : 0u) << (4 * j + 1);
                    sel |= (v4[j].z >= tau_f ? 1u : 0u) << (4 * j + 2);
                    sel |= (v4[j].w >= tau_f ? 1u : 0u) << (4 * j + 3);
                }
            } else {
#pragma unroll
                for (int j = 0; j < J; ++j) {
                    const int p = wb + 128 * j + 4 * lane;
                    sel |= (p + 0 < r1 && v4[j].x >= tau_f ? 1u : 0u) << (4 * j + 0);
                    sel |= (p + 1 < r1 && v4[j].y >= tau_f ? 1u : 0u) << (4 * j + 1);
                    sel |= (p + 2 < r1 && v4[j].z >= tau_f ? 1u : 0u) << (4 * j + 2);
                    sel |= (p + 3 < r1 && v4[j].w >= tau_f ? 1u : 0u) << (4 * j + 3);
                }
            }
            uint32_t pc = 0;  // count of load j in byte j (<= 4 per lane, <= 128 per warp)
#pragma unroll
            for (int j = 0; j < J; ++j) pc |= (uint32_t)__popc((sel >> (4 * j)) & 0xFu) << (8 * j);
            uint32_t inc = pc;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, inc, off);
                if (lane >= off) inc += y;
            }
            const uint32_t tot = __shfl_sync(0xffffffffu, inc, 31);
            const uint32_t exc = inc - pc;
            const uint32_t wtot = (tot & 0xFFu) + ((tot >> 8) & 0xFFu) + ((tot >> 16) & 0xFFu) + (tot >> 24);
            uint32_t at_j = m + warp_excl_scan(wtot, slots_a, &totals[0]);  // first slot of load 0's candidates
#pragma unroll
            for (int j = 0; j < J; ++j) {
                uint32_t at = at_j + ((exc >> (8 * j)) & 0xFFu);
                const int p = wb + 128 * j + 4 * lane;
                uint32_t bits = (sel >> (4 * j)) & 0xFu;  // few lanes hold any: visit set bits only
                while (bits) {
                    const int e = __ffs(bits) - 1;
                    bits &= bits - 1u;
                    const float x = e == 0 ? v4[j].x : e == 1 ? v4[j].y : e == 2 ? v4[j].z : v4[j].w;
                    const uint32_t k = score_key(x);
                    if (at < (uint32_t)kCandCap) {
                        cand_key[at] = k;
                        cand_pos[at] = p + e;
                        if (pub_dst) pub_dst[at] = make_uint2(k, (uint32_t)(p + e));
                    }
                    kmax = max(kmax, k);
                    ++at;
                }
                at_j += (tot >> (8 * j)) & 0xFFu;
            }
            m += totals[0];
        }
        kmax = __reduce_max_sync(0xffffffffu, kmax);
        if (lane == 0 && kmax) atomicMax(&cmax, kmax);
        __syncthreads();  // every thread's candidates are written before anyone reads them
    }
    }

    // ----------------------------- 3. the last CTA of the request selects
    uint32_t mtot = m;
    uint32_t tau_max = tau;  // the highest threshold among the request's parts
    uint32_t key_lo = tau, key_hi = cmax;  // a range holding every candidate key
    if (P > 1) {
        const int64_t slot = (int64_t)t * P + part;  // its candidates are in the workspace already
        if (tid == 0) a.counts[slot] = make_uint4(m, tau, cmax, 0u);
        __threadfence();
        __syncthreads();
        if (tid == 0) last = atomicAdd(a.arrivals + t, 1u) == (uint32_t)(P - 1);
        __syncthreads();
        if (!last) return;
        __threadfence();
        if (tid == 0) {
            a.arrivals[t] = 0;  // ready for the next launch
            uint32_t acc = 0, tmax = 0, tmin = 0xFFFFFFFFu, kmax = 0;
            bool fits = true;
            uint4 cq[kMaxParts];
#pragma unroll
            for (int q = 0; q < kMaxParts; ++q)  // every part's load in flight at once
                if (q < P) cq[q] = __ldcg(a.counts + (int64_t)t * P + q);
#pragma unroll
            for (int q = 0; q < kMaxParts; ++q)
                if (q < P) {
                    seg_off[q] = acc;
                    acc += cq[q].x;
                    fits &= cq[q].x <= (uint32_t)kCandCap;
                    tmax = max(tmax, cq[q].y);
                    tmin = min(tmin, cq[q].y);
                    kmax = max(kmax, cq[q].z);
                }
            seg_off[P] = fits ? acc : 0xFFFFFFFFu;
            sub32[0] = tmax;
            sub32[1] = tmin;
            sub32[2] = kmax;
        }
        __syncthreads();
        mtot = seg_off[P];
        tau_max = sub32[0];
        key_lo = sub32[1];
        key_hi = sub32[2];
        if (mtot >= (uint32_t)topk && mtot <= (uint32_t)kCandCap) {
            // concatenate in part order = position order; slot i of the
            // joined list belongs to the part q with seg_off[q] <= i <
            // seg_off[q + 1], so every load is independent of the others
            constexpr int kPer = (kCandCap + kTopkThreads - 1) / kTopkThreads;
            uint2 kp[kPer];
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const uint32_t i = tid + (uint32_t)k * kTopkThreads;
                if (i < mtot) {
                    int q = 0;
                    while (q + 1 < P && seg_off[q + 1] <= i) ++q;
                    kp[k] = __ldcg(a.cand + ((int64_t)t * P + q) * kCandCap + (i - seg_off[q]));
                }
            }
#pragma unroll
            for (int k = 0; k < kPer; ++k) {
                const uint32_t i = tid + (uint32_t)k * kTopkThreads;
                if (i < mtot) {
                    cand_key[i] = kp[k].x;
                    cand_pos[i] = (int32_t)kp[k].y;
                }
            }
            __syncthreads();
        }
    }
    if (mtot >= (uint32_t)topk && mtot <= (uint32_t)kCandCap) {
        uint32_t need_eq;
        // the ring area is free in the last CTA: room for the second binning level
        // every candidate key lies in [key_lo, key_hi]: each is at or above
        // its part's tau and at most its part's largest
        const uint32_t thr = select_fast(cand_key, mtot, (uint32_t)topk, hist, scratch, found, &need_eq, sub32, mm2,
                                         reinterpret_cast<uint32_t *>(ring), key_lo, key_hi);
        // every position at or above thr was collected when thr is at or
        // above each part's tau (block-uniform)
        if (thr >= tau_max) {
            write_from_candidates(cand_key, cand_pos, mtot, thr, need_eq, o, scratch);
            return;
        }
    }

    // ---------------------- tau missed: the general path over the whole row
    for (int i = tid; i < kBins; i += kTopkThreads) hist[i] = 0;
    if (tid == 0) ncand = 0;
    __syncthreads();
    // A: finite range
    float lo = INFINITY, hi = -INFINITY;
    ok = stream(0, ctx, [&](const float *buf, int c, int n) {
        for (int i = tid; i < kChunk / 4; i += kTopkThreads) {
            const float4 v4 = reinterpret_cast<const float4 *>(buf)[i];
            const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (4 * i + e < n && v[e] > -INFINITY) {
                    lo = fminf(lo, v[e]);
                    hi = fmaxf(hi, v[e]);
                }
        }
    });
    if (!ok) return fail();
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    if (lane == 0) {
        red_lo[warp] = lo;
        red_hi[warp] = hi;
    }
    __syncthreads();
    lo = red_lo[lane];
    hi = red_hi[lane];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
    }
    const float scale = (float)kBins / (hi - lo);
    bool fast = hi > lo && scale > 0.0f && scale < INFINITY;  // block-uniform
    // Monotone binning: x <= y gives bin(x) <= bin(y); -inf scores get -1.
    auto bin = [&](float x) -> int {
        if (!(x > -INFINITY)) return -1;
        const int b = (int)((x - lo) * scale);
        return b < kBins - 1 ? b : kBins - 1;
    };
    uint32_t thr = 0, need_eq = 0;  // threshold key and ties taken at it
    int dstar = 0;                  // threshold bin
    if (fast) {
        // B: histogram of the bins
        ok = stream(0, ctx, [&](const float *buf, int c, int n) {
            for (int i = tid; i < kChunk / 4; i += kTopkThreads) {
                const float4 v4 = reinterpret_cast<const float4 *>(buf)[i];
                const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int b = 4 * i + e < n ? bin(v[e]) : -1;
                    if (b >= 0) atomicAdd(&hist[b], 1u);
                }
            }
        });
        if (!ok) return fail();
        find_bin(hist, kBins, (uint32_t)topk, scratch, found);
        fast = found[2] >= (uint32_t)topk;  // enough finite scores
    }
    if (fast) {
        dstar = (int)found[0];
        const uint32_t want = found[1];  // to take from bin d*
        // C: the scores of bin d*
        ok = stream(0, ctx, [&](const float *buf, int c, int n) {
            for (int i = tid; i < kChunk / 4; i += kTopkThreads) {
                const float4 v4 = reinterpret_cast<const float4 *>(buf)[i];
                const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const bool cnd = 4 * i + e < n && bin(v[e]) == dstar;
                    const uint32_t cb = __ballot_sync(0xffffffffu, cnd);
                    if (cb) {
                        uint32_t at = 0;
                        if (lane == 0) at = atomicAdd(&ncand, (uint32_t)__popc(cb));
                        at = __shfl_sync(0xffffffffu, at, 0) + __popc(cb & ((1u << lane) - 1u));
                        if (cnd && at < (uint32_t)kCandCap) cand_key[at] = score_key(v[e]);
                    }
                }
            }
        });
        if (!ok) return fail();
        const uint32_t mc = ncand;
        fast = mc <= (uint32_t)kCandCap;
        if (fast) thr = select_in_smem(cand_key, mc, want, hist, scratch, found, &need_eq);
    }
    if (!fast) {
        // radix select over the whole row
        dstar = 0;  // every position counts as "in the threshold bin"
        uint32_t prefix = 0, remaining = (uint32_t)topk;
#pragma unroll 1
        for (int pass = 0; pass < 3; ++pass) {
            for (int i = tid; i < kBins; i += kTopkThreads) hist[i] = 0;
            __syncthreads();
            ok = stream(0, ctx, [&](const float *buf, int c, int n) {
                for (int i = tid; i < kChunk / 4; i += kTopkThreads) {
                    const float4 v4 = reinterpret_cast<const float4 *>(buf)[i];
                    const float v[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        add_to_hist(hist, 4 * i + e < n ? radix_digit(score_key(v[e]), pass, prefix) : 0xFFFFFFFFu,
                                    lane);
                }
            });
            if (!ok) return fail();
            find_bin(hist, pass == 2 ? 1024 : 2048, remaining, scratch, found);
            prefix |= found[0] << (pass == 0 ? 21 : (pass == 1 ? 10 : 0));
            remaining = found[1];
            __syncthreads();
        }
        thr = prefix;
        need_eq = remaining;
    }
    // D: ordered write
    uint32_t run_sel = 0, run_ties = 0;  // over the chunks done
    const uint32_t lt_mask = (1u << lane) - 1u;
    ok = stream(0, ctx, [&](const float *buf, int c, int n) {
        const float4 fa = reinterpret_cast<const float4 *>(buf)[warp * 64 + lane];
        const float4 fb = reinterpret_cast<const float4 *>(buf)[warp * 64 + 32 + lane];
        uint32_t eq_b[8], def_b[8];
        uint32_t ties = 0;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            // round r: chunk positions 256w + 32r + lane, held by lane
            // 8(r%4) + lane/4 of fa (r < 4) or fb as element lane%4
            const int src = 8 * (r & 3) + (lane >> 2);
            const float4 h = r < 4 ? fa : fb;
            const float x0 = __shfl_sync(0xffffffffu, h.x, src);
            const float x1 = __shfl_sync(0xffffffffu, h.y, src);
            const float x2 = __shfl_sync(0xffffffffu, h.z, src);
            const float x3 = __shfl_sync(0xffffffffu, h.w, src);
            const int el = lane & 3;
            const float x = el == 0 ? x0 : (el == 1 ? x1 : (el == 2 ? x2 : x3));
            const bool in = warp * 256 + 32 * r + lane < n;
            const uint32_t k = score_key(x);
            const int bb = fast ? bin(x) : 0;
            const bool at_thr = in && bb == dstar;
            eq_b[r] = __ballot_sync(0xffffffffu, at_thr && k == thr);
            def_b[r] = __ballot_sync(0xffffffffu, in && (bb > dstar || (at_thr && k > thr)));
            ties += __popc(eq_b[r]);
        }
        const uint32_t tie0 = run_ties + warp_excl_scan(ties, slots_a, &totals[0]);
        uint32_t sel = 0, seen = 0;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const bool mine_eq = (eq_b[r] >> lane) & 1u;
            const bool take_tie = mine_eq && tie0 + seen + __popc(eq_b[r] & lt_mask) < need_eq;
            def_b[r] |= __ballot_sync(0xffffffffu, take_tie);
            seen += __popc(eq_b[r]);
            sel += __popc(def_b[r]);
        }
        uint32_t at = run_sel + warp_excl_scan(sel, slots_b, &totals[1]);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            if ((def_b[r] >> lane) & 1u) o[at + __popc(def_b[r] & lt_mask)] = c * kChunk + warp * 256 + 32 * r + lane;
            at += __popc(def_b[r]);
        }
        run_ties += totals[0];
        run_sel += totals[1];
    });
    if (!ok) return fail();
}

}  // namespace idx

// ---------------------------------------------------------------- launch
static PFN_cuTensorMapEncodeTiled_v12000 index_map_encoder() {
    static std::atomic<PFN_cuTensorMapEncodeTiled_v12000> fn{nullptr};  // looked up once, by any thread
    PFN_cuTensorMapEncodeTiled_v12000 f = fn.load();
    if (!f) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !p) {
            (void)cudaGetLastError();
            return nullptr;
        }
        f = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        fn.store(f);
    }
    return f;
}

// 2-D byte matrix [rows, 128] with a box of box_rows x 128 bytes, 128-byte swizzle.
static bool make_byte_map(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows) {
    auto enc = index_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)idx::kDimI, rows};
    const cuuint64_t strides[1] = {(cuuint64_t)idx::kDimI};
    const cuuint32_t box[2] = {(cuuint32_t)idx::kDimI, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int64_t indexer_score_stride(int32_t max_ctx) { return ((int64_t)max_ctx + 127) / 128 * 128; }

cudaError_t launch_indexer_scores(const uint8_t *q, const float *w, const uint8_t *keys, int64_t num_slots,
                                  const int32_t *table, int64_t table_stride, int page_shift,
                                  const int32_t *ctx_lens, int32_t max_ctx, int32_t T, float *scores,
                                  int64_t score_stride, int32_t *dev_status, cudaStream_t stream) {
    if (T == 0 || max_ctx == 0) return cudaSuccess;
    using namespace idx;
    auto kern = indexer_score_kernel;
    static std::atomic<bool> attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    ScoreArgs a;
    a.w = w;
    a.table = table;
    a.table_stride = table_stride;
    a.page_shift = page_shift;
    a.box_shift = page_shift < 7 ? page_shift : 7;
    a.ctx_lens = ctx_lens;
    a.max_ctx = max_ctx;
    a.num_slots = num_slots;
    a.scores = scores;
    a.score_stride = score_stride;
    a.dev_status = dev_status;
    CUtensorMap tm_q, tm_k;
    if (!make_byte_map(&tm_q, q, (uint64_t)T * kHeads, kHeads) ||
        !make_byte_map(&tm_k, keys, (uint64_t)num_slots, 1u << a.box_shift))
        return cudaErrorInvalidValue;
    // CTAs per token: fill the resident CTA slots of the device once.
    const int slots = current_device_sm_count() * kCtasPerSm;
    const int max_tiles = (max_ctx + kTile - 1) / kTile;
    int x = slots / T;
    if (x < 1) x = 1;
    if (x > max_tiles) x = max_tiles;
    indexer_score_kernel<<<dim3((unsigned)x, (unsigned)T), kThreads, kSmemBytes, stream>>>(a, tm_q, tm_k);
    return cudaGetLastError();
}

int indexer_topk_parts(int32_t T, int sm_count) {
    if (T <= 0) return 1;
    const int p = sm_count / T;
    return p < 1 ? 1 : (p > idx::kMaxParts ? idx::kMaxParts : p);
}

// Workspace of a split selection: [T] arrival counters, then [T][P] (count,
// threshold key, largest candidate key, unused), then [T][P][kCandCap]
// candidates (8 bytes each); sections 256-byte aligned.
size_t indexer_topk_workspace_bytes(int32_t T, int sm_count) {
    const int P = indexer_topk_parts(T, sm_count);
    if (P == 1 || T <= 0) return 0;
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    return up((size_t)T * 4) + up((size_t)T * P * 16) + (size_t)T * P * idx::kCandCap * 8;
}

cudaError_t launch_indexer_topk(const float *scores, int64_t score_stride, const int32_t *ctx_lens, int32_t max_ctx,
                                int32_t T, int32_t topk, int32_t *positions, void *workspace, int32_t *dev_status,
                                cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    static std::atomic<bool> attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(idx::indexer_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 idx::kTopkDynSmem);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    idx::TopkArgs a;
    a.scores = scores;
    a.score_stride = score_stride;
    a.ctx_lens = ctx_lens;
    a.max_ctx = max_ctx;
    a.topk = topk;
    a.out = positions;
    a.parts = indexer_topk_parts(T, current_device_sm_count());
    a.dev_status = dev_status;
    a.arrivals = nullptr;
    a.counts = nullptr;
    a.cand = nullptr;
    if (a.parts > 1) {
        if (!workspace) return cudaErrorInvalidValue;
        auto up = [](size_t x) { return (x + 255) / 256 * 256; };
        uint8_t *w = static_cast<uint8_t *>(workspace);
        a.arrivals = reinterpret_cast<uint32_t *>(w);
        a.counts = reinterpret_cast<uint4 *>(w + up((size_t)T * 4));
        a.cand = reinterpret_cast<uint2 *>(w + up((size_t)T * 4) + up((size_t)T * a.parts * 16));
    }
    idx::indexer_topk_kernel<<<dim3((unsigned)a.parts, (unsigned)T), idx::kTopkThreads, idx::kTopkDynSmem, stream>>>(
        a);
    return cudaGetLastError();
}

}  // namespace nvfp4mla
