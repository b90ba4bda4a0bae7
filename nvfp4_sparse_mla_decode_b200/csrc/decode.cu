// decode.cu -- sparse MLA decode over NVFP4 (or staged E4M3) cache rows on
// the fifth-generation tensor cores of B200 (sm_100a).
//
// What it computes (page "Prime Intellect Launches Prime Inference, Serving
// 600B Tokens Daily", section "Four-bit caches make room"): each query token
// attends only to the cache rows its sparse-indexer list names; rows are
// unpacked on chip from NVFP4 to FP16; the scores q.k and the output p.V use
// FP16 operands with FP32 accumulation; empty list entries take no part.
//
// Work decomposition.  One CTA owns (token t, head group g of HG <= 64 heads,
// split s of the token's valid entries).  The token's list is compacted once
// per CTA (empty entries dropped, order kept), so every tile of 128 rows is
// full except the last one, whose missing rows are zero-filled and masked.
//
// Orientation.  Cache rows are the M dimension (M = 128), heads the N
// dimension (N = HG):
//   S^T[row, h]  = K[row, 0:576] . Q[h, 0:576]          (tcgen05, K-major A/B)
//   O^T[dv, h]  += V^T[dv, row] . P^T[row, h]           (tcgen05, MN-major A/B)
// Both accumulators live in tensor memory; O^T (512 x HG FP32) takes 4*HG
// columns.  One FP16 tile of 128 rows x 576 dims sits in shared memory in the
// 128-byte-swizzled layout; it serves as the K-major A operand of the score
// MMA and (latent part) as the MN-major A operand of the output MMA, so each
// row is unpacked exactly once.  P^T overwrites the RoPE chunk of the tile
// once the score MMAs have consumed it.
//
// Warp roles (640 threads, five warpgroups):
//   warps 0-3   thread 0 issues the nine Q tensor copies and every MMA;
//               warp 1 initialises the mbarriers, warp 3 owns TMEM
//   warps 4-11  softmax, two warpgroups with half of the heads each (TMEM
//               lanes = tile rows), then the epilogue and the split merge
//   warps 12-19 gather + unpack: each thread owns 4 rows x one 8-dim slice
//               of every 64-dim chunk; chunks 2p and 2p+1 are written as a
//               pair once output block p of the previous tile is done, and
//               the same registers then start loading that pair of the next
//               tile, so the gather hides behind the current tile's work.
// Each role sets its own register budget with setmaxnreg (RegSplit).
//
// Online softmax in base 2 with a lazily updated reference max: a head's
// reference moves (and O^T and the partial sums are rescaled) only when a
// score exceeds it by more than 8, so P = 2^(s - m) <= 256 fits FP16.
//
// Splits: when the grid would not fill the SMs, S CTAs share a token's
// list.  Each writes its unnormalised FP32 partial O and (max, row sum) to
// the workspace (its own merge slice stays in shared memory), the S CTAs meet
// on a counter (cooperative launch, bounded wait) and each merges one
// 512/S-wide dv slice of every head; there is no second kernel.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <atomic>

#include <cmath>

#include "common.cuh"
#include "decode_common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace nvfp4mla {
using namespace ptx;
#ifdef NVFP4MLA_TRACE
void set_trace_buffer(unsigned long long *p) { set_trace_local(p); }
void set_trace_all_buffer(unsigned long long *p) { set_trace_all_local(p); }
#endif

namespace dec {
constexpr int kTileRows = 128;
constexpr int kChunks = 9;                           // 8 latent chunks of 64 dims + RoPE
constexpr int kChunkBytes = kTileRows * 128;         // 16384
constexpr int kTileBytes = kChunks * kChunkBytes;    // 147456
constexpr int kMaxHG = 64;
constexpr int kOffQ = kTileBytes;                    // Q: 9 chunks x HG rows x 128 B
constexpr int kOffIdx = kOffQ + kMaxHG * kDim * 2;   // compacted list share (int32)
constexpr int kOffM = kOffIdx + kMaxTopk * 4;        // reference max per head (log2 units)
constexpr int kOffAux = kOffM + kMaxHG * 4;          // rescale factors / 1/l per head
constexpr int kOffRed = kOffAux + kMaxHG * 4;        // 4 warps x 64 floats
constexpr int kOffBar = kOffRed + 4 * kMaxHG * 4;
constexpr int kNumBars = 17;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kMaxHG * kLatent * 4 <= kTileBytes, "FP32 output staging must fit in the tile region");
constexpr int kThreads = 640;
// warps 0-3: MMA issue (warp 0) + TMEM allocation (warp 3); warps 4-11: two
// softmax warpgroups (half of the heads each); warps 12-19: gather + unpack.
constexpr int kSoftmaxWarp0 = 4;
constexpr int kUnpackWarp0 = 12;
// Per-thread register budgets per role (setmaxnreg).  At launch every thread
// holds kRegsLaunch registers (65536 / 640 rounded down to a multiple of 8);
// a role may only decrease below it with .dec and increase above it with .inc,
// and the new total must fit in what the block was launched with.  The split
// depends on the instantiation: with 64 heads per CTA a softmax thread keeps
// 32 per-head values and two 32-column output blocks at once, while the
// unpack warps hold a tile's raw words plus the next tile's row slots
// (chosen by measurement among the splits with the fewest spills).
constexpr int kRegsLaunch = 96;
template <int HG, bool kStaged>
struct RegSplit {
    static constexpr int mma = 40;                                         // warpgroup 0 (.dec)
    static constexpr int softmax = HG == 64 ? 136 : 128;  // warpgroups 1-2 (.inc)
    static constexpr int unpack = HG == 64 ? 80 : 88;      // warpgroups 3-4 (.dec)
    static_assert(mma < kRegsLaunch && unpack < kRegsLaunch && softmax > kRegsLaunch, "setmaxnreg direction");
    static_assert(mma % 8 == 0 && softmax % 8 == 0 && unpack % 8 == 0, "setmaxnreg granularity");
    static_assert(128 * mma + 256 * softmax + 256 * unpack <= 640 * kRegsLaunch, "register budget");
};

constexpr int BAR_CHUNK_FULL = 0;  // [9] unpack -> MMA, count 8 warps
constexpr int BAR_CHUNK_FREE = 9;  // [4] output MMAs of a 128-dv block done
constexpr int BAR_S_FULL = 13;     // score MMAs of a tile done
constexpr int BAR_P_FULL = 14;     // P^T written (4 softmax warps)
constexpr int BAR_DRAIN = 15;      // every MMA issued so far done
constexpr int BAR_Q_FULL = 16;     // Q tensor copies landed (one arrive with the byte count)

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;      // O^T: 4 blocks of HG columns
constexpr uint32_t kColS = 256;    // S^T: HG columns
constexpr float kRescaleThreshold = 8.0f;
constexpr int kMaxSplits = 16;
// Merge scratch in the (by then free) tile region: split weights at 0, and
// at kOffOwn the CTA's own partial dv slice (S <= 4: [HG][512/S] FP32).
constexpr int kOffOwn = 16384;
static_assert((kMaxSplits + 1) * kMaxHG * 4 <= kOffOwn, "merge weights must fit below the own slice");
static_assert(kOffOwn + kMaxHG * (kLatent / 2) * 4 <= kTileBytes, "own slice must fit in the tile region");
}  // namespace dec

// Merge of the S split partials of one (token, head group), run by the 256
// softmax threads of each of the S CTAs of the group once their partial is
// written: one thread announces this CTA's partial on the group's arrival
// counter (release; the softmax-group barrier before it orders every
// thread's partial stores ahead of it), waits (bounded) until all S have,
// and then the group combines the dv slice [split*512/S, (split+1)*512/S)
// of every head:
//   out = sum_s w_s O_s / sum_s w_s l_s,  w_s = 2^(m_s - max m)
// over the splits with rows (l_s > 0); split 0 also writes
// lse = (max m + log2 of the denominator) ln 2.  With S <= 4 the CTA's own
// slice is already in shared memory; the others are read with 16-byte
// loads, up to 16 in flight per thread.  The launch is cooperative, so all S
// CTAs are resident together and the wait ends.  The last CTA to leave
// resets both counters, which lets the next call start from zero.
template <int HG, int S>
__device__ __forceinline__ void merge_splits(const DecodeArgs &a, int t, int g, int split, uint8_t *smem, int mt,
                                             [[maybe_unused]] unsigned long long t_start) {
    TRACE_SETUP();
    using namespace dec;
    constexpr int kMergeThreads = 256;
    constexpr int D = kLatent / S;           // dv per CTA
    constexpr int NQ = D / 4;                // float4 per head
    constexpr int ITEMS = HG * NQ;
    constexpr bool kOwnInSmem = S <= 4;
    // items per batch: up to 24 global vectors in flight per thread (the own
    // slice is read from shared memory when it is combined)
    constexpr int kGlobal = kOwnInSmem ? S - 1 : S;
    constexpr int kPerThread = (ITEMS + kMergeThreads - 1) / kMergeThreads;
    constexpr int B = (24 / kGlobal) < 1 ? 1 : ((24 / kGlobal) > kPerThread ? kPerThread : (24 / kGlobal));
    uint32_t *arrive = a.counters + 2 * ((int64_t)t * a.G + g);
    uint32_t *depart = arrive + 1;
    uint32_t *flag = reinterpret_cast<uint32_t *>(smem + kOffMisc) + 1;
    float *w_s = reinterpret_cast<float *>(smem);  // [S][HG] weights
    float *inv_den = w_s + kMaxSplits * HG;         // [HG]
    const float *own = reinterpret_cast<const float *>(smem + kOffOwn);  // [HG][D]
    named_bar(3, kMergeThreads);  // every partial store of the group precedes the release
    if (mt == 0) {
        TRACE(280);
        __threadfence();
        red_release_gpu_add(arrive, 1u);
        const bool ok = spin_until_geq(arrive, (uint32_t)S);
        if (!ok && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
        *flag = ok ? 1u : 0u;
        TRACE(281);
    }
    named_bar(3, kMergeThreads);
    if (!*flag) return;  // counters stay raised: the caller must clear them after a timeout
    const int dv0 = split * D;
    const int64_t part = (int64_t)a.H * kLatent;  // next split of the same (t, head)
    const float *src = a.ws_o + ((int64_t)t * S * a.H + (int64_t)g * HG) * kLatent + dv0;
    __half *dst = a.out + ((int64_t)t * a.H + (int64_t)g * HG) * kLatent + dv0;
    float4 o[B][kGlobal];  // the foreign partials (all S when the own slice is not in shared memory)
    auto load_batch = [&](int base) {
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const int item = base + b * kMergeThreads;
            const int h = item / NQ, q = item - h * NQ;
#pragma unroll
            for (int j = 0; j < kGlobal; ++j) {
                const int s = kOwnInSmem && j >= split ? j + 1 : j;
                o[b][j] = item < ITEMS
                              ? __ldcg(reinterpret_cast<const float4 *>(src + (int64_t)h * kLatent + 4 * q + s * part))
                              : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            }
        }
    };
    auto combine_batch = [&](int base) {
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const int item = base + b * kMergeThreads;
            if (item < ITEMS) {
                const int h = item / NQ, q = item - h * NQ;
                float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                if (kOwnInSmem) {
                    const float w = w_s[split * HG + h];
                    const float4 v = *reinterpret_cast<const float4 *>(own + h * D + 4 * q);
                    acc.x = w * v.x;
                    acc.y = w * v.y;
                    acc.z = w * v.z;
                    acc.w = w * v.w;
                }
#pragma unroll
                for (int j = 0; j < kGlobal; ++j) {  // an empty split's partial is zero and its weight 0
                    const int s = kOwnInSmem && j >= split ? j + 1 : j;
                    const float w = w_s[s * HG + h];
                    acc.x += w * o[b][j].x;
                    acc.y += w * o[b][j].y;
                    acc.z += w * o[b][j].z;
                    acc.w += w * o[b][j].w;
                }
                const float r = inv_den[h];
                __half2 *d2 = reinterpret_cast<__half2 *>(dst + (int64_t)h * kLatent + 4 * q);
                d2[0] = __floats2half2_rn(acc.x * r, acc.y * r);
                d2[1] = __floats2half2_rn(acc.z * r, acc.w * r);
            }
        }
    };
    // The first batch of partial loads is in flight while the weights are
    // computed from the statistics.
    load_batch(mt);
    if (mt < HG) {
        const float *ml = a.ws_ml + 2 * ((int64_t)t * S * a.H + (int64_t)g * HG + mt);
        float2 v[S];
#pragma unroll
        for (int s = 0; s < S; ++s) v[s] = __ldcg(reinterpret_cast<const float2 *>(ml + 2 * (int64_t)s * a.H));
        float mmax = -INFINITY;
#pragma unroll
        for (int s = 0; s < S; ++s)
            if (v[s].y > 0.0f) mmax = fmaxf(mmax, v[s].x);
        float den = 0.0f;
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const float w = v[s].y > 0.0f ? ex2(v[s].x - mmax) : 0.0f;
            w_s[s * HG + mt] = w;
            den += w * v[s].y;
        }
        inv_den[mt] = den > 0.0f ? 1.0f / den : 0.0f;
        if (split == 0)
            a.lse[(int64_t)t * a.H + (int64_t)g * HG + mt] =
                den > 0.0f ? (mmax + lg2(den)) * 0.69314718055994531f : -INFINITY;
    }
    named_bar(3, kMergeThreads);
    if (mt == 0) TRACE(282);
    combine_batch(mt);
    for (int base = mt + kMergeThreads * B; base < ITEMS; base += kMergeThreads * B) {
        load_batch(base);
        combine_batch(base);
    }
    named_bar(3, kMergeThreads);
    if (mt == 0) {
        TRACE(283);
        const uint32_t old = atomicAdd(depart, 1u);
        if (old == (uint32_t)S - 1u) {  // every CTA of the group is past its wait
            atomicExch(arrive, 0u);
            atomicExch(depart, 0u);
        }
    }
}

template <int HG, bool kStaged>
__global__ void __launch_bounds__(dec::kThreads, 1)
    sparse_mla_decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_qn,
                             const __grid_constant__ CUtensorMap tm_qr) {
    using namespace dec;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
#ifdef NVFP4MLA_TRACE
    const unsigned long long t_start = clock64();
    if (tid == 0 && g_trace_all) {
        g_trace_all[3 * blockIdx.x] = global_ns();
        g_trace_all[3 * blockIdx.x + 2] = sm_id();
    }
#else
    const unsigned long long t_start = 0;  // timestamps exist only in trace builds
#endif
    TRACE_SETUP();
    const int split = blockIdx.x % a.S;
    const int rest = blockIdx.x / a.S;
    const int g = rest % a.G;
    const int t = rest / a.G;

    if (smem_u32(smem) & 1023u) {  // the swizzled operand layout needs a 1 KB aligned base
        if (tid == 0 && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_LAYOUT);
        return;
    }
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kOffBar);
    uint32_t *misc = reinterpret_cast<uint32_t *>(smem + kOffMisc);
    int32_t *idx_s = reinterpret_cast<int32_t *>(smem + kOffIdx);
    float *m_s = reinterpret_cast<float *>(smem + kOffM);
    float *aux_s = reinterpret_cast<float *>(smem + kOffAux);
    float *red_s = reinterpret_cast<float *>(smem + kOffRed);
    uint32_t *cnt_s = reinterpret_cast<uint32_t *>(smem + kOffRed);  // reused before the softmax starts

    // ---------------------------------------------------------------- setup
    if (warp == 1) {  // one barrier per lane
        uint32_t count = 0;
        if (lane < BAR_CHUNK_FREE) count = 8;           // chunk written by the 8 unpack warps
        else if (lane < BAR_P_FULL) count = 1;          // MMA commits
        else if (lane == BAR_P_FULL) count = 8;         // 8 softmax warps
        else if (lane == BAR_DRAIN) count = 1;
        else if (lane == BAR_Q_FULL) count = 1;         // thread 0, with the Q byte count
        if (count) mbar_init(&bars[lane], count);
        fence_mbar_init();
    }
    if (warp == 3) {  // a warp with no setup work: the allocation can take a while
        tmem_alloc(&misc[0], kTmemCols);
        tmem_relinquish();
        if (lane == 0) TRACE(260);
    }
    if (tid < HG) m_s[tid] = -INFINITY;

    // Compact the token's list: keep valid entries in list order; this CTA
    // keeps entries [lo, hi) of the compacted order.
    const int32_t *lst = a.indices + (int64_t)t * a.topk;
    int32_t vals[4];
    uint32_t bal[4];
    bool bad = false;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int p = tid + 512 * k;  // warps 16.. have no list entries (p >= 2048)
        int32_t v = (p < a.topk && tid < 512) ? __ldg(lst + p) : -1;
        bool entry_bad = false;
        if (a.block_table && v >= 0) {  // request-local position -> slot through the block table
            int64_t slot = -1;
            if ((int64_t)v < a.max_pos) {
                const int32_t blk = __ldg(a.block_table + (int64_t)t * a.table_stride + (v >> a.page_shift));
                if (blk >= 0) slot = ((int64_t)blk << a.page_shift) + (v & ((1 << a.page_shift) - 1));
            }
            entry_bad = slot < 0 || slot >= a.num_slots;
            v = entry_bad ? -1 : (int32_t)slot;
        }
        const bool ok = v >= 0 && (int64_t)v < a.num_slots;
        bad |= (p < a.topk) && (entry_bad || v < -1 || (int64_t)v >= a.num_slots);
        vals[k] = v;
        bal[k] = __ballot_sync(0xffffffffu, ok);
        if (lane == 0 && warp < 16) cnt_s[k * 16 + warp] = __popc(bal[k]);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0 && split == 0 && g == 0 && a.dev_status)
        atomicOr(a.dev_status, NVFP4MLA_DEV_BAD_INDEX);
    if (tid == 0) TRACE(261);
    __syncthreads();
    if (tid == 0) TRACE(262);
    // Exclusive prefix of the 64 per-(round, warp) counts.  Every warp scans
    // them itself (two per lane) and reads its own offsets from the lane that
    // holds them, so no second block barrier is needed.
    int before[4];
    int n_valid;
    {
        const uint32_t c0 = cnt_s[2 * lane], c1 = cnt_s[2 * lane + 1];
        uint32_t incl = c0 + c1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - c0 - c1;
        n_valid = (int)__shfl_sync(0xffffffffu, incl, 31);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int j = k * 16 + (warp & 15);  // count index of (round k, this warp)
            const uint32_t mine = (j & 1) ? excl + c0 : excl;
            const uint32_t b = __shfl_sync(0xffffffffu, mine, j >> 1);
            before[k] = warp < 16 ? (int)b : 0;
        }
    }
    const int per = (n_valid + a.S - 1) / a.S;
    const int lo = split * per;
    const int hi = min(n_valid, lo + per);
    const int n_mine = max(0, hi - lo);
    const int ntiles = (n_mine + kTileRows - 1) / kTileRows;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if (warp < 16 && ((bal[k] >> lane) & 1u)) {
            const int pos = before[k] + __popc(bal[k] & ((1u << lane) - 1u));
            if (pos >= lo && pos < hi) idx_s[pos - lo] = (kStaged && !a.rows_by_slot) ? (tid + 512 * k) : vals[k];
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    if (tid == 0) TRACE(0);

    // Register budget (launched with 96 x 640 = 61440): the MMA/idle
    // warpgroup and the unpack warps give registers to the softmax warps
    // (see RegSplit).  Each role changes its budget inside its own branch so
    // the compiler sizes each role's code separately.
    if (warp < 4) {
        regs_dec<RegSplit<HG, kStaged>::mma>();
        // Q of (t, heads g*HG ..) -> shared memory, K-major, 128-byte swizzle:
        // chunk c holds dims 64c..64c+63 of every head (chunk 8 = RoPE).  Nine
        // tensor copies (box: 64 dims x HG heads, swizzled by the copy engine
        // into exactly the MMA operand layout), so Q takes no load/store-unit
        // slots from the row gather.
        if (tid == 0) {
            const int32_t row = t * a.H + g * HG;
            mbar_arrive_expect_tx(&bars[BAR_Q_FULL], (uint32_t)(HG * kDim * 2));
#pragma unroll 1
            for (int c = 0; c < 8; ++c) tma_load_2d(smem + kOffQ + c * (HG * 128), &tm_qn, 64 * c, row, &bars[BAR_Q_FULL]);
            tma_load_2d(smem + kOffQ + 8 * (HG * 128), &tm_qr, 0, row, &bars[BAR_Q_FULL]);
        }
        // ------------------------------------------------------------- MMA
        if (warp == 0 && lane == 0) {
            const uint32_t idesc_qk = idesc_f16_f32(128, HG, false, false);
            const uint32_t idesc_pv = idesc_f16_f32(128, HG, true, true);
            const uint64_t dK0 = smem_desc(smem_u32(smem), 16, 1024);
            const uint64_t dQ0 = smem_desc(smem_u32(smem + kOffQ), 16, 1024);
            const uint64_t dV0 = smem_desc(smem_u32(smem), kChunkBytes, 1024);
            const uint64_t dP0 = smem_desc(smem_u32(smem + 8 * kChunkBytes), kChunkBytes, 1024);
            bool ok = mbar_wait(&bars[BAR_Q_FULL], 0);  // always: the Q copies must land before the CTA exits
            // Descriptors advance by adding (byte offset >> 4) to the start
            // address field; the chunk and block loops stay rolled so the
            // compiler keeps a handful of descriptors live, not one per MMA.
            for (int i = 0; i < ntiles && ok; ++i) {
                const uint32_t par = i & 1;
                uint64_t dk = dK0, dq = dQ0;
#pragma unroll 1
                for (int c = 0; c < kChunks; ++c) {
                    if (!mbar_wait(&bars[BAR_CHUNK_FULL + c], par)) {
                        ok = false;
                        break;
                    }
                    if (i == 1) TRACE(64 + c);
                    tc_fence_after();
                    mma_ss(tmem + kColS, dk, dq, idesc_qk, c != 0);
                    mma_ss(tmem + kColS, dk + 2, dq + 2, idesc_qk, 1u);
                    mma_ss(tmem + kColS, dk + 4, dq + 4, idesc_qk, 1u);
                    mma_ss(tmem + kColS, dk + 6, dq + 6, idesc_qk, 1u);
                    dk += (uint64_t)(kChunkBytes >> 4);
                    dq += (uint64_t)((HG * 128) >> 4);
                }
                if (!ok) break;
                mma_commit(&bars[BAR_S_FULL]);
                if (i < 8) TRACE(1 + 6 * i);
                if (!mbar_wait(&bars[BAR_P_FULL], par)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (i < 8) TRACE(2 + 6 * i);
                uint64_t dv = dV0;
#pragma unroll 1
                for (int dc = 0; dc < 4; ++dc) {
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_ss(tmem + kColO + dc * HG, dv + (uint64_t)(kk * 128), dP0 + (uint64_t)(kk * 128),
                               idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(&bars[BAR_CHUNK_FREE + dc]);
                    if (i == 0) TRACE(112 + dc);
                    dv += (uint64_t)((2 * kChunkBytes) >> 4);
                }
                if (i < 8) TRACE(3 + 6 * i);
            }
            if (!ok && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
            mma_commit(&bars[BAR_DRAIN]);  // nothing may still write TMEM at teardown
            mbar_wait(&bars[BAR_DRAIN], 0);
            TRACE(60);
        }
        __syncwarp();
    } else if (warp < kUnpackWarp0) {
        // --------------------------------------------------------- softmax
        regs_inc<RegSplit<HG, kStaged>::softmax>();
        // Two warpgroups; warpgroup sw owns heads [h0, h0 + HWG).  A head's
        // reference max, rescale and row sum never depend on other heads, so
        // the groups only meet at the P^T barrier and the epilogue.  With
        // HG = 16 the second group has no heads and only keeps the barrier
        // count.
        constexpr int NSW = HG >= 32 ? 2 : 1;
        constexpr int HWG = HG / NSW;
        const int sw = (warp - kSoftmaxWarp0) >> 2;
        const int st = tid - 32 * kSoftmaxWarp0 - 128 * sw;  // tile row == TMEM lane
        const int wq = st >> 5;
        const uint32_t bar_id = 1 + sw;
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        uint8_t *p_tile = smem + 8 * kChunkBytes;  // P^T overwrites the RoPE chunk
        const int h0 = sw * HWG;
        const bool active = sw < NSW;
        float lp[HWG];  // this thread's (row slot's) running sum per head
#pragma unroll
        for (int j = 0; j < HWG; ++j) lp[j] = 0.0f;
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            // S_FULL(i) also covers PV(i-1): the MMA thread issued it earlier,
            // so O^T is quiescent and may be rescaled here.
            // the wait's outcome is agreed by the whole warpgroup, so its four
            // warps always meet at the same named barriers
            if (named_bar_or(bar_id, 128, !mbar_wait(&bars[BAR_S_FULL], i & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (st == 0 && sw == 0 && i < 8) TRACE(4 + 6 * i);
            if (active) {
                float sv[HWG];
                {
                    uint32_t rs[HWG];
                    tmem_ld_cols<HWG>(tmem + lane_base + kColS + h0, rs);
                    tmem_ld_wait();
#pragma unroll
                    for (int h = 0; h < HWG; ++h) sv[h] = __uint_as_float(rs[h]) * a.scale_log2;
                }
                const int nrows = min(kTileRows, n_mine - kTileRows * i);
                const bool valid = st < nrows;
                bool need = false;
                if (valid) {
#pragma unroll
                    for (int h = 0; h < HWG; ++h) need |= sv[h] > m_s[h0 + h] + kRescaleThreshold;
                }
                if (named_bar_or(bar_id, 128, need)) {
#pragma unroll
                    for (int c0 = 0; c0 < HWG; c0 += 16) {  // column max, 16 heads at a time
                        float mx[16];
#pragma unroll
                        for (int h = 0; h < 16; ++h) mx[h] = valid ? sv[c0 + h] : -INFINITY;
                        warp_transpose_reduce<16, true>(mx, lane);
                        if (!(lane & 1)) red_s[wq * 64 + h0 + c0 + transposed_col<16>(lane, 0)] = mx[0];
                    }
                    named_bar(bar_id, 128);
                    if (st < HWG) {
                        const int h = h0 + st;
                        const float old = m_s[h];
                        float nm = old;
#pragma unroll
                        for (int w = 0; w < 4; ++w) nm = fmaxf(nm, red_s[w * 64 + h]);
                        aux_s[h] = (old == -INFINITY) ? 0.0f : ex2(old - nm);
                        m_s[h] = nm;
                    }
                    named_bar(bar_id, 128);
#pragma unroll
                    for (int h = 0; h < HWG; ++h) lp[h] *= aux_s[h0 + h];
                    if (i > 0) {
#pragma unroll 1
                        for (int dc = 0; dc < 4; ++dc) {
#pragma unroll
                            for (int cb = 0; cb < HWG; cb += 16) {  // 16 columns per round trip
                                uint32_t r[16];
                                const uint32_t addr = tmem + lane_base + kColO + dc * HG + h0 + cb;
                                tmem_ld16(addr, r);
                                tmem_ld_wait();
#pragma unroll
                                for (int h = 0; h < 16; ++h)
                                    r[h] = __float_as_uint(__uint_as_float(r[h]) * aux_s[h0 + cb + h]);
                                tmem_st16(addr, r);
                            }
                        }
                        tmem_st_wait();
                    }
                }
#pragma unroll
                for (int h = 0; h < HWG; ++h) {
                    sv[h] = valid ? ex2(sv[h] - m_s[h0 + h]) : 0.0f;
                    lp[h] += sv[h];
                }
#pragma unroll
                for (int j = 0; j < HWG / 8; ++j) {
                    uint4 pk;
                    pk.x = pack_half2(sv[8 * j + 0], sv[8 * j + 1]);
                    pk.y = pack_half2(sv[8 * j + 2], sv[8 * j + 3]);
                    pk.z = pack_half2(sv[8 * j + 4], sv[8 * j + 5]);
                    pk.w = pack_half2(sv[8 * j + 6], sv[8 * j + 7]);
                    *reinterpret_cast<uint4 *>(p_tile + sw128_offset(st, h0 / 8 + j)) = pk;
                }
                fence_proxy_async_smem();
                tc_fence_before();
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[BAR_P_FULL]);
            if (st == 0 && sw == 0 && i < 8) TRACE(5 + 6 * i);
        }
        if (!ok && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
        // ---------------------------------------------------------- epilogue
        // Row sums and the per-head statistics need no TMEM, so they are
        // done while the last tile's output MMAs still run.
        const bool have = ok && ntiles > 0;
        if (active) {
            // row sums: reduce each head's 128 per-row partials (16 heads at a time)
#pragma unroll
            for (int c0 = 0; c0 < HWG; c0 += 16) {
                float v[16];
#pragma unroll
                for (int h = 0; h < 16; ++h) v[h] = lp[c0 + h];
                warp_transpose_reduce<16, false>(v, lane);
                if (!(lane & 1)) red_s[wq * 64 + h0 + c0 + transposed_col<16>(lane, 0)] = v[0];
            }
            named_bar(bar_id, 128);
            if (st < HWG) {
                const int h = h0 + st;
                const float l = have ? red_s[h] + red_s[64 + h] + red_s[128 + h] + red_s[192 + h] : 0.0f;
                const float m = m_s[h];
                aux_s[h] = l > 0.0f ? 1.0f / l : 0.0f;
                const int64_t hrow = (int64_t)t * a.H + (int64_t)g * HG + h;
                if (a.S == 1) {
                    a.lse[hrow] = l > 0.0f ? (m + lg2(l)) * 0.69314718055994531f : -INFINITY;
                } else {
                    const int64_t prow = ((int64_t)t * a.S + split) * a.H + (int64_t)g * HG + h;
                    a.ws_ml[2 * prow] = l > 0.0f ? m : -INFINITY;
                    a.ws_ml[2 * prow + 1] = l;
                }
            }
            named_bar(bar_id, 128);
        }
        // Output block b is final once the last tile's block-b MMAs are done.
        auto wait_block = [&](int b) {
            if (ok && ntiles > 0) {
                if (!mbar_wait(&bars[BAR_CHUNK_FREE + b], (ntiles - 1) & 1)) {
                    ok = false;
                    if (a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
                }
                tc_fence_after();
            }
        };
        if (st == 0 && sw == 0) TRACE(270);
        if (st == 0 && sw == 0) TRACE(271);
        const bool leader = (warp == kSoftmaxWarp0 && lane == 0);
        if (a.S == 1) {
            // O^T (TMEM, lanes = dv) -> normalised FP16 rows staged in the
            // (now free) tile region, then one bulk copy of HG x 1 KB to
            // out[t, g*HG .., :].
            wait_block(3);
            float inv_l[HWG];
#pragma unroll
            for (int h = 0; h < HWG; ++h) inv_l[h] = active ? aux_s[h0 + h] : 0.0f;
            uint8_t *stage = smem;
            if (active) {
#pragma unroll 1
                for (int dc = 0; dc < 4; ++dc) {
                    const int dv = 128 * dc + st;
                    uint32_t r[HWG];
                    if (have) {
                        tmem_ld_cols<HWG>(tmem + lane_base + kColO + dc * HG + h0, r);
                        tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int h = 0; h < HWG; ++h) r[h] = 0u;
                    }
#pragma unroll
                    for (int h = 0; h < HWG; ++h)
                        reinterpret_cast<__half *>(stage)[(h0 + h) * kLatent + dv] =
                            __float2half_rn(__uint_as_float(r[h]) * inv_l[h]);
                }
                fence_proxy_async_smem();
            }
            named_bar(3, 256);
            if (leader) {
                bulk_s2g(a.out + ((int64_t)t * a.H + (int64_t)g * HG) * kLatent, stage, HG * kLatent * 2);
                bulk_commit_wait_read();
            }
        } else {
            // Unnormalised partial O (this split's rows, scaled to its own
            // reference max), up to two 128-dv blocks per TMEM round trip.
            // Blocks 0-1 that go to the workspace leave as soon as they are
            // final, while blocks 2-3 are still being accumulated; the rest
            // follow once everything is done.  Blocks inside this CTA's own
            // merge slice (S <= 4) go to shared memory at kOffOwn (the tile
            // is no longer read by then); the others go to the workspace
            // straight from registers (for each head a warp writes 32
            // consecutive dv, one 128-byte segment).  The softmax-group
            // barrier and the release in the merge order these stores ahead
            // of the arrival.
            float *dst = a.ws_o + (((int64_t)t * a.S + split) * a.H + (int64_t)g * HG + h0) * kLatent + st;
            const int own_n = a.S <= 4 ? 4 / a.S : 0;  // 128-dv blocks in the own slice
            const int own_dc0 = split * own_n;
            const int own_d = kLatent / a.S;
            float *own = reinterpret_cast<float *>(smem + kOffOwn) + (int64_t)h0 * own_d + st;
            auto is_own = [&](int b) { return b >= own_dc0 && b < own_dc0 + own_n; };
            auto drain = [&](int b0, int b1) {  // b1 < 0: one block
                uint32_t r[2][HWG];
                if (have) {
                    tmem_ld_cols<HWG>(tmem + lane_base + kColO + b0 * HG + h0, r[0]);
                    if (b1 >= 0) tmem_ld_cols<HWG>(tmem + lane_base + kColO + b1 * HG + h0, r[1]);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int h = 0; h < HWG; ++h) r[0][h] = r[1][h] = 0u;
                }
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const int b = j == 0 ? b0 : b1;
                    if (b < 0) continue;
                    if (is_own(b)) {
#pragma unroll
                        for (int h = 0; h < HWG; ++h) own[h * own_d + 128 * (b - own_dc0)] = __uint_as_float(r[j][h]);
                    } else {
#pragma unroll
                        for (int h = 0; h < HWG; ++h)
                            __stcg(dst + (int64_t)h * kLatent + 128 * b, __uint_as_float(r[j][h]));
                    }
                }
            };
            wait_block(1);
            if (active) {
                const bool g0 = !is_own(0), g1 = !is_own(1);
                if (g0 && g1) drain(0, 1);
                else if (g0) drain(0, -1);
                else if (g1) drain(1, -1);
            }
            wait_block(3);
            if (active) {  // blocks 2-3 and any own block among 0-1
                const bool o0 = is_own(0), o1 = is_own(1);
                if (o0 && o1) {
                    drain(0, 1);
                    drain(2, 3);
                } else if (o0 || o1) {
                    drain(o0 ? 0 : 1, 2);
                    drain(3, -1);
                } else {
                    drain(2, 3);
                }
            }
        }
        if (st == 0 && sw == 0) TRACE(279);
        if (a.S > 1) {
            const int mt = tid - 32 * kSoftmaxWarp0;
            switch (a.S) {
                case 2: merge_splits<HG, 2>(a, t, g, split, smem, mt, t_start); break;
                case 4: merge_splits<HG, 4>(a, t, g, split, smem, mt, t_start); break;
                case 8: merge_splits<HG, 8>(a, t, g, split, smem, mt, t_start); break;
                default: merge_splits<HG, 16>(a, t, g, split, smem, mt, t_start); break;
            }
        }
        if (leader) TRACE(61);
    } else {
        // ---------------------------------------------------- gather + unpack
        regs_dec<RegSplit<HG, kStaged>::unpack>();
        const int ut = tid - 32 * kUnpackWarp0;
        const int sub = ut & 7;   // 8-dim slice of every 64-dim chunk
        const int rg = ut >> 3;   // rows rg, rg+32, rg+64, rg+96 of each tile
        constexpr int kWords = kStaged ? 18 : 11;  // raw 32-bit words per row held per tile
        uint32_t raw[4][kWords];
        int32_t slot[4];  // rows of the tile whose words are being loaded
        bool rvalid[4];
        // Row loads come in groups, in the order the pairs consume them:
        // group p < 4 = chunks 2p and 2p+1, group 4 = RoPE, and for NVFP4
        // rows group 5 = the 32 scales.  Rows past the end are not read and
        // stay zero.
        auto set_rows = [&](int i) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int e = kTileRows * i + rg + 32 * k;
                rvalid[k] = e < n_mine;
                slot[k] = rvalid[k] ? idx_s[e] : 0;
            }
        };
        // FP8 rows: row `slot` of the cache, or row (t, list position) of
        // the staging buffer.
        const int64_t row0 = (kStaged && !a.rows_by_slot) ? (int64_t)t * a.topk : 0;
        auto row_base = [&](int k) -> const uint8_t * {
            return kStaged ? a.src + (row0 + slot[k]) * kStagedRowBytes
                           : a.src + (int64_t)slot[k] * kRowBytes;
        };
        auto load_group = [&](int grp) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint8_t *rp = row_base(k);
                if (kStaged) {
                    if (grp < 4) {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int c = 2 * grp + j;
                            const uint2 w2 = rvalid[k] ? ldg64(rp + 64 * c + 8 * sub) : make_uint2(0u, 0u);
                            raw[k][2 * c] = w2.x;
                            raw[k][2 * c + 1] = w2.y;
                        }
                    } else if (grp == 4) {
                        const uint2 w2 = rvalid[k] ? ldg64(rp + 64 * 8 + 8 * sub) : make_uint2(0u, 0u);
                        raw[k][16] = w2.x;
                        raw[k][17] = w2.y;
                    }
                } else {
                    if (grp < 4) {
#pragma unroll
                        for (int j = 0; j < 2; ++j) {
                            const int c = 2 * grp + j;
                            raw[k][c] = rvalid[k] ? ldg32(rp + 32 * c + 4 * sub) : 0u;
                        }
                    } else if (grp == 4) {
                        const uint2 w2 = rvalid[k] ? ldg64(rp + kRopeOff + 8 * sub) : make_uint2(0u, 0u);
                        raw[k][9] = w2.x;
                        raw[k][10] = w2.y;
                    } else {
                        raw[k][8] = rvalid[k] ? ldg32(rp + kScaleOff + 4 * sub) : 0u;
                    }
                }
            }
        };
        bool ok = true;
        if (ntiles > 0) {
            set_rows(0);
            load_group(5);
#pragma unroll
            for (int grp = 0; grp < 5; ++grp) load_group(grp);
        }
        if (ut == 0) TRACE(277);
        // Decode chunk c of this thread's 4 rows into the swizzled tile.
        auto unpack_chunk = [&](int c) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                uint32_t o[4];
                if (kStaged) {
                    e4m3x8_to_f16x8(raw[k][2 * c], raw[k][2 * c + 1], o);
                } else if (c < 8) {
                    const uint32_t sw = __shfl_sync(0xffffffffu, raw[k][8], (lane & ~7) | c);
                    const uint32_t sb = (sw >> (8 * (sub >> 1))) & 0xFFu;
                    const uint32_t s2 = e4m3x2_to_f16x2(sb | (sb << 8));
                    e2m1x8_to_f16x8(raw[k][c], o);
#pragma unroll
                    for (int j = 0; j < 4; ++j) o[j] = hmul2_u32(o[j], s2);
                } else {
                    e4m3x8_to_f16x8(raw[k][9], raw[k][10], o);
                }
                *reinterpret_cast<uint4 *>(smem + c * kChunkBytes + sw128_offset(rg + 32 * k, sub)) =
                    make_uint4(o[0], o[1], o[2], o[3]);
            }
        };
        for (int i = 0; i < ntiles && ok; ++i) {
            const bool more = i + 1 < ntiles;
            // Chunks 2p and 2p+1 are released together by output block p, so
            // they are written as a pair behind one wait and one fence; the
            // RoPE chunk (8, where P^T lives) was released by block 3.  As
            // soon as a pair's words are decoded, the same registers start
            // loading that pair of the next tile, so the gather of tile i+1
            // is spread over the unpack of tile i.
#pragma unroll
            for (int p = 0; p < 5; ++p) {
                if (p < 4 && i > 0 && !mbar_wait(&bars[BAR_CHUNK_FREE + p], (i - 1) & 1)) {
                    ok = false;
                    break;
                }
                if (ut == 0 && i == 1) TRACE(80 + p);
                if (p < 4) {
                    unpack_chunk(2 * p);
                    unpack_chunk(2 * p + 1);
                } else {
                    unpack_chunk(8);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&bars[BAR_CHUNK_FULL + (p < 4 ? 2 * p : 8)]);
                    if (p < 4) mbar_arrive(&bars[BAR_CHUNK_FULL + 2 * p + 1]);
                }
                if (ut == 0 && i == 1) TRACE(96 + p);
                if (lane == 0 && i == 1) TRACE(128 + 16 * (ut >> 5) + p);
                if (more) {
                    if (p == 0) set_rows(i + 1);
                    load_group(p);
                    if (p == 3 && !kStaged) load_group(5);  // scales: last used by pair 3
                }
            }
            if (ut == 0 && i < 8) TRACE(6 + 6 * i);
        }
        if (ut == 0) TRACE(62);
        if (!ok && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
    }

    // ---------------------------------------------------------------- teardown
    tc_fence_before();
    __syncthreads();
    if (warp == 3) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
#ifdef NVFP4MLA_TRACE
    if (tid == 0 && g_trace_all) g_trace_all[3 * blockIdx.x + 1] = global_ns();
#endif
}

int current_device_sm_count() {
    static std::atomic<int> cached[64] = {};  // 0: not asked yet
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
        (void)cudaGetLastError();  // no device: leave no error behind for later launches
        return 148;
    }
    int n = cached[dev].load();
    if (!n) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
            (void)cudaGetLastError();
            return 148;
        }
        cached[dev].store(n);
    }
    return n;
}

bool make_decode_plan(int32_t T, int32_t H, int32_t topk, int sm_count, DecodePlan *plan, int splits,
                      int heads_per_cta) {
    DecodePlan p{};
    if (H != 16 && H != 32 && H != 64 && H != 128) return false;
    if (topk < 1 || topk > kMaxTopk || T < 0 || sm_count < 1) return false;
    const int max_s = std::min(dec::kMaxSplits, (topk + dec::kTileRows - 1) / dec::kTileRows);
    if (heads_per_cta == 0) {
        // 64 heads per CTA, or 32 when twice the head groups still fit in one
        // wave at the most splits the list takes: twice the CTAs on the same
        // work (on a B200, T = 1..4 with H = 64 or 128: 8-17 % less time; when
        // halving the head group would cost splits it is no faster)
        p.heads_per_cta = H < 64 ? H : 64;
        if (p.heads_per_cta == 64 && (int64_t)T * (H / 32) * max_s <= sm_count) p.heads_per_cta = 32;
    } else if ((heads_per_cta == 16 || heads_per_cta == 32 || heads_per_cta == 64) && heads_per_cta <= H) {
        p.heads_per_cta = heads_per_cta;  // H is a power of two: it divides H
    } else {
        return false;
    }
    p.head_groups = H / p.heads_per_cta;
    const int64_t units = (int64_t)T * p.head_groups;
    int S = 1;
    if (splits == 0) {
        // Split a token's list over S CTAs only while the whole grid still
        // fits in one wave of one CTA per SM (the merge needs every CTA
        // resident).
        while (S * 2 <= max_s && units * S * 2 <= sm_count) S *= 2;
        if (S > 1 && units > (int64_t)(kSplitCounterBytes / 8)) S = 1;
    } else {
        // a caller's split count: a power of two the list has tiles for,
        // with every CTA of a split grid resident and its counters in place
        if (splits < 1 || splits > max_s || (splits & (splits - 1))) return false;
        if (splits > 1 && (units * splits > sm_count || units > (int64_t)(kSplitCounterBytes / 8))) return false;
        S = splits;
    }
    p.splits = S;
    p.workspace_bytes = S > 1 ? kSplitCounterBytes + (size_t)T * S * H * (kLatent + 2) * sizeof(float) : 0;
    *plan = p;
    return true;
}

// Tensor maps for Q: a 2-D FP16 view [rows = T*H, cols] of q_nope (cols 512)
// or q_rope (cols 64), box 64 cols x HG rows, 128-byte swizzle.
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// Encoded maps are kept in a small per-thread cache keyed by (address, rows,
// cols, box rows), so a caller that reuses its query buffers pays for the
// encoding once.
bool make_q_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    struct Entry {
        const void *base;
        uint64_t rows, cols;
        uint32_t box_rows;
        CUtensorMap map;
    };
    constexpr int kEntries = 16;
    thread_local Entry cache[kEntries] = {};
    thread_local int next = 0;
    for (int i = 0; i < kEntries; ++i) {
        const Entry &e = cache[i];
        if (e.base == base && e.rows == rows && e.cols == cols && e.box_rows == box_rows) {
            *m = e.map;
            return true;
        }
    }
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    cache[next] = Entry{base, rows, cols, box_rows, *m};
    next = (next + 1) % kEntries;
    return true;
}

// Tensor map for the NVFP4 kernel's split exchange area: a 2-D FP32 view
// [rows, 2048] of ws_o (row = one 4-head piece of one split's partial, 512 dv
// x 4 heads), box box_x floats x box_rows rows, no swizzle; cached per host
// thread like the Q maps.
bool make_xch_map(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_x, uint32_t box_rows) {
    struct Entry {
        const void *base;
        uint64_t rows;
        uint32_t box_x, box_rows;
        CUtensorMap map;
    };
    constexpr int kEntries = 8;
    thread_local Entry cache[kEntries] = {};
    thread_local int next = 0;
    for (int i = 0; i < kEntries; ++i) {
        const Entry &e = cache[i];
        if (e.base == base && e.rows == rows && e.box_x == box_x && e.box_rows == box_rows) {
            *m = e.map;
            return true;
        }
    }
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)kLatent * 4, rows};
    const cuuint64_t strides[1] = {(cuuint64_t)kLatent * 16};
    const cuuint32_t box[2] = {box_x, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    cache[next] = Entry{base, rows, box_x, box_rows, *m};
    next = (next + 1) % kEntries;
    return true;
}

template <int HG, bool kStaged>
static cudaError_t launch_hg(const DecodeArgs &a, int64_t nblocks, cudaStream_t stream) {
    auto kern = sparse_mla_decode_kernel<HG, kStaged>;
    static std::atomic<bool> attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
        // The per-role register split (setmaxnreg) assumes the block starts
        // with kRegsLaunch registers per thread; with fewer, a role's
        // increase could never be granted, so refuse to launch.
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != dec::kRegsLaunch || fa.maxThreadsPerBlock < dec::kThreads) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
    }
    // Split launches are cooperative: the runtime refuses the launch unless
    // every CTA can be resident at once, which the merge's wait relies on.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)nblocks);
    cfg.blockDim = dim3(dec::kThreads);
    cfg.dynamicSmemBytes = dec::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.S > 1 ? 1 : 0;
    CUtensorMap tm_qn, tm_qr;
    const uint64_t rows = (uint64_t)a.T * (uint64_t)a.H;
    if (!make_q_map(&tm_qn, a.q_nope, rows, kLatent, HG) || !make_q_map(&tm_qr, a.q_rope, rows, kRope, HG))
        return cudaErrorInvalidValue;
    return cudaLaunchKernelEx(&cfg, kern, a, tm_qn, tm_qr);
}

cudaError_t launch_sparse_mla_decode(RowSource rows, const void *q_nope, const void *q_rope, const uint8_t *src,
                                     int64_t num_slots, const int32_t *indices, int32_t topk, int32_t T,
                                     int32_t H, float sm_scale, void *out, float *lse, void *workspace,
                                     const DecodePlan &plan, int32_t *dev_status, cudaStream_t stream,
                                     const int32_t *block_table, int64_t table_stride, int page_shift,
                                     const DecodeTestHooks *hooks) {
    if (T == 0) return cudaSuccess;
    DecodeArgs a;
    a.q_nope = static_cast<const __half *>(q_nope);
    a.q_rope = static_cast<const __half *>(q_rope);
    a.src = src;
    a.num_slots = num_slots;
    a.indices = indices;
    a.topk = topk;
    a.T = T;
    a.H = H;
    a.G = plan.head_groups;
    a.S = plan.splits;
    a.scale_log2 = (float)((double)sm_scale * 1.4426950408889634);
    a.out = static_cast<__half *>(out);
    a.lse = lse;
    // workspace: [split counters, kSplitCounterBytes][ws_ml][ws_o]
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    a.counters = plan.splits > 1 ? reinterpret_cast<uint32_t *>(ws) : nullptr;
    a.ws_ml = plan.splits > 1 ? reinterpret_cast<float *>(ws + kSplitCounterBytes) : nullptr;
    a.ws_o = plan.splits > 1 ? a.ws_ml + (size_t)T * plan.splits * H * 2 : nullptr;
    a.dev_status = dev_status;
    a.block_table = block_table;
    a.table_stride = table_stride;
    a.page_shift = page_shift;
    a.max_pos = block_table ? (table_stride << page_shift) : 0;
    a.rows_by_slot = rows == RowSource::kFp8Cache;
    a.wait_cycles = hooks ? hooks->wait_cycles : ptx::kWaitCycles;
    a.test_withhold = hooks ? hooks->withhold : 0;
    const bool staged = rows != RowSource::kNvfp4Cache;
    const int64_t nblocks = (int64_t)T * plan.head_groups * plan.splits;
    if (!staged) return launch_nvfp4_decode(a, plan.heads_per_cta, nblocks, stream);
    cudaError_t e;
    switch (plan.heads_per_cta * 2 + (staged ? 1 : 0)) {
        case 32: e = launch_hg<16, false>(a, nblocks, stream); break;
        case 33: e = launch_hg<16, true>(a, nblocks, stream); break;
        case 64: e = launch_hg<32, false>(a, nblocks, stream); break;
        case 65: e = launch_hg<32, true>(a, nblocks, stream); break;
        case 128: e = launch_hg<64, false>(a, nblocks, stream); break;
        case 129: e = launch_hg<64, true>(a, nblocks, stream); break;
        default: return cudaErrorInvalidValue;
    }
    return e;
}

}  // namespace nvfp4mla
