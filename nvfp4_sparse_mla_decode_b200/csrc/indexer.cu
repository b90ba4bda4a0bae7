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
// swizzle) into a 4-stage ring; the epilogue reads one TMEM lane (one
// position) per thread and folds the 64 heads with ReLU and the weights.
// The work is HBM-bound (128 key bytes per position against 16K FLOP), so
// the design goal is to keep every SM streaming keys: several CTAs per SM,
// each with a copy warp, an MMA warp and four epilogue warps, double-buffered
// accumulators (2 x 64 TMEM columns).
//
// Selection (indexer_topk_kernel): one CTA per request, a three-digit radix
// select (11 + 11 + 10 bits of an order-preserving key) for the k-th largest
// score, then one ordered pass in which each warp owns a contiguous range of
// positions and writes its selected positions with ballots, so the list
// comes out in increasing position order.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

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
constexpr int kStages = 4;
constexpr int kThreads = 192;                  // warp 0 copies, warp 1 MMA + TMEM, warps 2-5 epilogue
constexpr int kCtasPerSm = 3;
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
        for (int i = 0; i < n; ++i) {
            const int b = i & 1;
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
            float acc = 0.0f;
#pragma unroll
            for (int h = 0; h < 32; h += 4) {
                const float4 wv = *reinterpret_cast<const float4 *>(w_s + h);
                acc = fmaf(wv.x, fmaxf(__uint_as_float(r0[h]), 0.0f), acc);
                acc = fmaf(wv.y, fmaxf(__uint_as_float(r0[h + 1]), 0.0f), acc);
                acc = fmaf(wv.z, fmaxf(__uint_as_float(r0[h + 2]), 0.0f), acc);
                acc = fmaf(wv.w, fmaxf(__uint_as_float(r0[h + 3]), 0.0f), acc);
            }
#pragma unroll
            for (int h = 0; h < 32; h += 4) {
                const float4 wv = *reinterpret_cast<const float4 *>(w_s + 32 + h);
                acc = fmaf(wv.x, fmaxf(__uint_as_float(r1[h]), 0.0f), acc);
                acc = fmaf(wv.y, fmaxf(__uint_as_float(r1[h + 1]), 0.0f), acc);
                acc = fmaf(wv.z, fmaxf(__uint_as_float(r1[h + 2]), 0.0f), acc);
                acc = fmaf(wv.w, fmaxf(__uint_as_float(r1[h + 3]), 0.0f), acc);
            }
            const int p = (first + i * (int)gridDim.x) * kTile + row;
            if (p < ctx) {
                // a position whose key copy was refused (empty table entry or
                // a page outside the cache) scores -inf
                const bool valid = copy_row(a, t, p & ~(box - 1)) >= 0;
                a.scores[(int64_t)t * a.score_stride + p] = valid ? acc : -INFINITY;
            }
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
constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;

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

__global__ void __launch_bounds__(kTopkThreads, 1)
    indexer_topk_kernel(const float *__restrict__ scores, int64_t score_stride, const int32_t *__restrict__ ctx_lens,
                        int max_ctx, int topk, int32_t *__restrict__ out, int32_t *dev_status) {
    __shared__ uint32_t hist[2048];
    __shared__ uint32_t scratch[32];
    __shared__ uint32_t found[2];
    __shared__ uint32_t wcnt[kTopkWarps][2];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = blockIdx.x;
    int ctx = __ldg(ctx_lens + t);
    if (ctx < 0 || ctx > max_ctx) {
        if (tid == 0) flag(dev_status, NVFP4MLA_DEV_BAD_INDEX);
        ctx = ctx < 0 ? 0 : max_ctx;
    }
    int32_t *o = out + (int64_t)t * topk;
    if (ctx <= topk) {  // every position, then -1
        for (int i = tid; i < topk; i += kTopkThreads) o[i] = i < ctx ? i : -1;
        return;
    }
    const float *s = scores + (int64_t)t * score_stride;

    // Radix select of the topk-th largest key, most significant digit first.
    uint32_t prefix = 0;        // digits found so far, in place
    uint32_t remaining = topk;  // how many keys still to take at or below the prefix
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        const uint32_t hi_mask = pass == 0 ? 0u : (0xFFFFFFFFu << (shift + (pass == 2 ? 10 : 11)));
        for (int i = tid; i < 2048; i += kTopkThreads) hist[i] = 0;
        __syncthreads();
        // every thread runs the same number of rounds, so the warp-wide
        // match below always sees full warps
        for (int base = 0; base < ctx; base += 4 * kTopkThreads) {
            const int p = base + 4 * tid;  // 4 consecutive positions per thread
            float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
            if (p < ctx) v = __ldcg(reinterpret_cast<const float4 *>(s + p));
            const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                uint32_t d = 0xFFFFFFFFu;
                if (p + e < ctx) {
                    const uint32_t k = score_key(vv[e]);
                    if ((k & hi_mask) == prefix) d = (k >> shift) & (uint32_t)(nb - 1);
                }
                const uint32_t peers = __match_any_sync(0xffffffffu, d);
                if (d != 0xFFFFFFFFu && lane == __ffs(peers) - 1) atomicAdd(&hist[d], (uint32_t)__popc(peers));
            }
        }
        __syncthreads();
        // Thread i looks at bins nb-1-2i and nb-2-2i (descending); the
        // running count from the top tells which bin holds the target.
        uint32_t c_hi = 0, c_lo = 0;
        if (2 * tid < nb) {
            c_hi = hist[nb - 1 - 2 * tid];
            c_lo = hist[nb - 2 - 2 * tid];
        }
        const uint32_t incl = block_incl_scan(c_hi + c_lo, scratch);
        const uint32_t before = incl - c_hi - c_lo;
        if (2 * tid < nb) {
            if (remaining > before && remaining <= before + c_hi) {
                found[0] = (uint32_t)(nb - 1 - 2 * tid);
                found[1] = remaining - before;
            } else if (remaining > before + c_hi && remaining <= incl) {
                found[0] = (uint32_t)(nb - 2 - 2 * tid);
                found[1] = remaining - before - c_hi;
            }
        }
        __syncthreads();
        prefix |= found[0] << shift;
        remaining = found[1];
        __syncthreads();
    }
    const uint32_t thr = prefix;     // the topk-th largest key
    const uint32_t need_eq = remaining;  // keys equal to thr to take, by position

    // Each warp owns a contiguous range of positions (a multiple of 128).
    const int seg = ((ctx + kTopkWarps * 128 - 1) / (kTopkWarps * 128)) * 128;
    const int w_lo = warp * seg;
    const int w_hi = min(ctx, w_lo + seg);
    uint32_t gt = 0, eq = 0;
    for (int base = w_lo; base < w_hi; base += 128) {
        const int p = base + 4 * lane;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p < w_hi) v = __ldcg(reinterpret_cast<const float4 *>(s + p));
        const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (p + e < w_hi) {
                const uint32_t k = score_key(vv[e]);
                gt += k > thr;
                eq += k == thr;
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        gt += __shfl_xor_sync(0xffffffffu, gt, off);
        eq += __shfl_xor_sync(0xffffffffu, eq, off);
    }
    if (lane == 0) {
        wcnt[warp][0] = gt;
        wcnt[warp][1] = eq;
    }
    __syncthreads();
    if (warp == 0) {
        // per warp: ties before its range, then how many it writes and where
        const uint32_t g = wcnt[lane][0], e = wcnt[lane][1];
        uint32_t e_incl = e;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, e_incl, off);
            if (lane >= off) e_incl += y;
        }
        const uint32_t e_before = e_incl - e;
        const uint32_t take = need_eq > e_before ? min(e, need_eq - e_before) : 0u;
        const uint32_t sel = g + take;
        uint32_t s_incl = sel;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, s_incl, off);
            if (lane >= off) s_incl += y;
        }
        __syncwarp();
        wcnt[lane][0] = s_incl - sel;  // first output slot of this warp
        wcnt[lane][1] = e_before;      // ties before this warp's range
    }
    __syncthreads();
    uint32_t at = wcnt[warp][0];
    uint32_t ties = wcnt[warp][1];
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int base = w_lo; base < w_hi; base += 128) {
        const int p = base + 4 * lane;
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p < w_hi) v = __ldcg(reinterpret_cast<const float4 *>(s + p));
        const float vv[4] = {v.x, v.y, v.z, v.w};
        // positions in order: element e of every lane, lanes in order, is
        // NOT increasing position order (lane l holds p..p+3), so walk the
        // 128 positions as 4 rounds of 32 consecutive ones via shuffles
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            // round r covers positions base + 32r .. base + 32r + 31; lane l
            // takes position base + 32r + l, held by lane (8r + l/4) as
            // element l%4
            const int src = 8 * r + (lane >> 2);
            const int el = lane & 3;
            const float x0 = __shfl_sync(0xffffffffu, vv[0], src);
            const float x1 = __shfl_sync(0xffffffffu, vv[1], src);
            const float x2 = __shfl_sync(0xffffffffu, vv[2], src);
            const float x3 = __shfl_sync(0xffffffffu, vv[3], src);
            const float x = el == 0 ? x0 : (el == 1 ? x1 : (el == 2 ? x2 : x3));
            const int q = base + 32 * r + lane;
            const bool in = q < w_hi;
            const uint32_t k = in ? score_key(x) : 0u;
            const bool is_eq = in && k == thr;
            const uint32_t eq_b = __ballot_sync(0xffffffffu, is_eq);
            const bool take = in && (k > thr || (is_eq && ties + __popc(eq_b & lt_mask) < need_eq));
            const uint32_t sel_b = __ballot_sync(0xffffffffu, take);
            if (take) o[at + __popc(sel_b & lt_mask)] = q;
            at += __popc(sel_b);
            ties += __popc(eq_b);
        }
    }
}

}  // namespace idx

// ---------------------------------------------------------------- launch
static PFN_cuTensorMapEncodeTiled_v12000 index_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || !p) {
            (void)cudaGetLastError();
            return nullptr;
        }
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
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
    static bool attr_set[64] = {};
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

cudaError_t launch_indexer_topk(const float *scores, int64_t score_stride, const int32_t *ctx_lens, int32_t max_ctx,
                                int32_t T, int32_t topk, int32_t *positions, int32_t *dev_status,
                                cudaStream_t stream) {
    if (T == 0) return cudaSuccess;
    idx::indexer_topk_kernel<<<(unsigned)T, idx::kTopkThreads, 0, stream>>>(scores, score_stride, ctx_lens, max_ctx,
                                                                           topk, positions, dev_status);
    return cudaGetLastError();
}

}  // namespace nvfp4mla
