// decode_nvfp4.cu -- sparse MLA decode over 352-byte NVFP4 cache rows on the
// fifth-generation tensor cores of B200 (sm_100a), pipelined so that row
// gather, on-chip unpack, the score MMAs, the softmax and the output MMAs of
// neighbouring tiles overlap.
//
// What it computes (page "Prime Intellect Launches Prime Inference, Serving
// 600B Tokens Daily", section "Four-bit caches make room"): each query token
// attends only to the cache rows its sparse-indexer list names; the rows are
// unpacked on chip from NVFP4 to FP16; q.k and p.V run with FP16 operands and
// FP32 accumulation; list entries that name no row take no part.  The same
// section credits a multi-stage pipeline in which one group of warps unpacks
// rows while others score and accumulate; this kernel is that idea laid out
// for sm_100a: every stage has its own warps and its own ring.
//
// Work decomposition: one CTA per (token t, head group g of HG <= 64 heads,
// split s of the token's valid list entries).  The list is compacted once per
// CTA (empty entries dropped, order kept), so every 128-row tile is full
// except the last one.
//
// Per tile j (rows = the M dimension, heads = N):
//   S^T[row, h]  = K[row, 0:576] . Q[h, 0:576]      A = K from tensor memory
//   O^T[dv, h]  += V^T[dv, row] . P^T[row, h]       A = V^T, B = P^T in shared
// The score MMA reads its K operand from tensor memory (a ring of four
// 64-dim chunks written by the unpack warps with tcgen05.st), so only Q
// streams from shared memory.  Score and output MMAs are issued by two
// different warps, so the barrier waits of one stream overlap the MMAs of
// the other.  V is the latent part of the same rows; it is
// decoded a second time, 16 rows at a time, into a two-slot shared-memory
// ring in the MN-major layout the output MMA reads.  The score MMAs of tile
// j+1 need only the K ring and a free S buffer (S is double-buffered), so
// they run while the softmax of tile j is still working.
//
// Warp roles (768 threads, six warpgroups):
//   warp 0      score MMA issue (whole warp, one elected lane issues)
//   warps 1, 3  gather: the CTA's Q by tensor copies (warp 1), then the
//               valid rows in 16-byte cp.async pieces into a two-tile raw
//               ring (rows padded to 368 bytes so the unpack warps read
//               them without bank conflicts)
//   warp 2      tensor-memory allocation and release; output MMA issue
//   warps 4-11  K unpack: thread = tile row = TMEM lane; warps 4-7 take the
//               even 64-dim chunks, warps 8-11 the odd ones (and RoPE)
//   warps 12-15 softmax (thread = tile row), then the epilogue and the split
//               merge
//   warps 16-23 V unpack, two sets of four alternating the 16-row groups
//               of a tile (16 rows x 8 dv groups per ring slot), rows read
//               again from L2 (they arrived one tile earlier)
//
// Tensor memory (512 columns): O^T at 0 (four 128-dv blocks of HG columns),
// S^T double-buffered at 256 and 320, the K ring at 384 (4 x 32 columns).
//
// Online softmax in base 2 with a lazily updated reference max: a head's
// reference moves (and O^T and the row sums are rescaled) only when a score
// exceeds it by more than 8, so p = 2^(s - m) <= 256 fits FP16.
//
// Splits: when T * G alone would leave SMs idle, S CTAs share a token's list;
// each writes its unnormalised FP32 partial and (max, row sum), the S CTAs
// meet on a counter (cooperative launch, bounded wait) and each merges one
// 512/S-wide dv slice of every head.  A CTA whose wait runs out marks the
// counter poisoned, so later launches on the same workspace report the
// timeout instead of merging stale partials.
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
void set_trace_buffer_nv4(unsigned long long *p) { set_trace_local(p); }
#endif

namespace nv4 {
constexpr int kTileRows = 128;
constexpr int kMaxHG = 64;
constexpr int kRawStride = 368;                            // 352-byte row + 16 bytes of padding
constexpr int kRawSlotBytes = kTileRows * kRawStride;      // 47104
constexpr int kVRows = 16;                                 // rows per V ring slot (one MMA K step)
constexpr int kVSlotBytes = kVRows * kLatent * 2;          // 16384
constexpr int kVSlots = 2;                                 // V ring depth
constexpr int kRawSlots = 2;                               // raw tiles in shared memory
constexpr int kVGroups = kTileRows / kVRows;               // 8
constexpr int kKChunks = 9;                                // 8 latent chunks of 64 dims + RoPE
constexpr int kKSlots = 4;
constexpr int kOffQ = 0;                                   // 9 chunks x HG rows x 128 B
constexpr int kOffP = kOffQ + kKChunks * kMaxHG * 128;     // 73728: P^T, 128 rows x 128 B
constexpr int kOffV = kOffP + kTileRows * 128;             // 90112: V ring
constexpr int kOffRaw = kOffV + kVSlots * kVSlotBytes;     // 155648: raw ring
constexpr int kOffIdx = kOffRaw + kRawSlots * kRawSlotBytes;  // compacted list share
constexpr int kOffM = kOffIdx + kMaxTopk * 4;              // reference max per head (log2 units)
constexpr int kOffAux = kOffM + kMaxHG * 4;                // rescale factors, then 1/l
constexpr int kOffRed = kOffAux + kMaxHG * 4;              // 4 warps x 64 floats
constexpr int kOffBar = kOffRed + 4 * kMaxHG * 4;
constexpr int kNumBars = 28;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kOffP % 1024 == 0 && kOffV % 1024 == 0, "swizzled operands need 1 KB alignment");
// the epilogue stages its output (or its own merge slice) over the V and raw
// rings, which are free by then; the merge weights go to the P^T region
constexpr int kOffStage = kOffV;
// split merge: S boxes of D dv x HG heads FP32 (HG x 2 KB in all) over P^T
// and the rings, then the merge weights
constexpr int kOffPartial = kOffP;
constexpr int kOffMergeW = kOffPartial + kMaxHG * kLatent * 4;
static_assert(kOffMergeW + (16 * kMaxHG + kMaxHG) * 4 <= kOffIdx, "merge areas must fit before the list");
static_assert(kOffPartial % 128 == 0 && kOffMergeW % 16 == 0, "merge areas take tensor copies and 16-byte accesses");
static_assert(kMaxHG * kLatent * 2 <= kOffIdx - kOffStage, "output staging must fit over the rings");
constexpr int kThreads = 768;
// the first tile's rows are copied by the gather warps and the eight V-unpack
// warps together (the V warps have nothing to do until those rows land)
constexpr int kTile0Threads = 64 + 256;
// the split merge's combine runs on the softmax and V-unpack threads, which
// meet at named barrier kMergeBar (barrier 1 is the softmax warps' own)
constexpr int kCombineThreads = 128 + 256;
constexpr int kMergeBar = 2;
constexpr int kKWarp0 = 4;
constexpr int kSoftWarp0 = 12;
constexpr int kVWarp0 = 16;
// Register budgets per warpgroup (setmaxnreg): launched with 80 per thread
// (65536 / 768 rounded down to a multiple of 8); the control and K-unpack
// warpgroups give registers to the softmax warps, whose threads hold a row of
// scores and of P.
constexpr int kRegsLaunch = 80;
constexpr int kRegsCtl = 48;
constexpr int kRegsK = 64;
constexpr int kRegsV = 80;
constexpr int kRegsSoft = 144;
static_assert(128 * kRegsCtl + 256 * kRegsK + 128 * kRegsSoft + 256 * kRegsV <= kThreads * kRegsLaunch,
              "register split exceeds the launch budget");

// mbarriers
constexpr int BAR_Q = 0;                           // Q tensor copies (expect_tx)
constexpr int BAR_RAW_FULL = 1;                    // [kRawSlots] raw tile landed (cp.async arrivals of 64 threads)
constexpr int BAR_RAW_FREE = BAR_RAW_FULL + kRawSlots;  // [kRawSlots] raw tile read by the 8 K-unpack warps
constexpr int BAR_K_FULL = BAR_RAW_FREE + kRawSlots;    // [4] K chunk in TMEM (4 warps)
constexpr int BAR_K_FREE = BAR_K_FULL + kKSlots;        // [4] score MMAs of the chunk done (commit)
constexpr int BAR_V_FULL = BAR_K_FREE + kKSlots;        // [kVSlots] V slot written (the 4 warps of a V set)
constexpr int BAR_V_FREE = BAR_V_FULL + kVSlots;        // [kVSlots] output MMAs of the slot done (commit)
constexpr int BAR_S_FULL = BAR_V_FREE + kVSlots;        // [2] score MMAs of a tile done (commit)
constexpr int BAR_P_FULL = BAR_S_FULL + 2;              // P^T written, O^T rescaled (4 softmax warps)
constexpr int BAR_PV_DONE = BAR_P_FULL + 1;             // output MMAs of a tile done (commit)
constexpr int BAR_DRAIN = BAR_PV_DONE + 1;              // every score MMA issued so far done
constexpr int BAR_S_FREE = BAR_DRAIN + 1;               // [2] softmax done reading an S buffer (4 softmax warps)
constexpr int BAR_DRAIN_PV = BAR_S_FREE + 2;            // every output MMA issued so far done
constexpr int BAR_ROWS0 = BAR_DRAIN_PV + 1;             // the first tile's rows landed (cp.async arrivals of kTile0Threads)
constexpr int BAR_K0DONE = BAR_ROWS0 + 1;              // the first tile's K unpacked (8 K-unpack warps)
constexpr int kBarsUsed = BAR_K0DONE + 1;
static_assert(kBarsUsed <= kNumBars, "barrier slots");

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;
constexpr uint32_t kColS = 256;
constexpr uint32_t kColK = 384;
constexpr float kRescaleThreshold = 8.0f;
constexpr int kMaxSplits = 16;
static_assert(kMaxSplits == 16, "merge weight area sized for 16 splits");
constexpr uint32_t kPoison = 0x80000000u;
}  // namespace nv4

// Whole-warp bounded wait: every lane polls, the result is agreed by vote
// so the warp stays converged for the elected-lane instructions after it.
// Whole-warp bounded wait (the warp agrees on the outcome); `lim` is the
// launch's wait bound in SM clock cycles.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, unsigned long long lim) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, lim));
}

__device__ __forceinline__ uint4 lds128(const uint8_t *p) { return *reinterpret_cast<const uint4 *>(p); }
__device__ __forceinline__ uint32_t lds32(const uint8_t *p) { return *reinterpret_cast<const uint32_t *>(p); }

// 64 latent dims of one row: 32 nibble bytes (two 16-byte words) and the
// four E4M3 scales of its 16-dim groups -> 32 f16x2 words, dims 2i, 2i+1 in
// word i (low half = even dim).  Exact: e2m1 x e4m3 has at most 6
// significant bits and lies inside FP16's range.
__device__ __forceinline__ void unpack_latent64(uint4 w0, uint4 w1, uint32_t scales, uint32_t (&o)[32]) {
    const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    // the four scales as two f16x2 pairs, then each broadcast to both halves
    const uint32_t s01 = e4m3x2_to_f16x2(scales & 0xFFFFu), s23 = e4m3x2_to_f16x2(scales >> 16);
    const uint32_t sc2[4] = {__byte_perm(s01, 0u, 0x1010), __byte_perm(s01, 0u, 0x3232), __byte_perm(s23, 0u, 0x1010),
                             __byte_perm(s23, 0u, 0x3232)};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t s2 = sc2[k];
        uint32_t lo[4], hi[4];
        e2m1x8_to_f16x8(w[2 * k], lo);
        e2m1x8_to_f16x8(w[2 * k + 1], hi);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            o[8 * k + i] = hmul2_u32(lo[i], s2);
            o[8 * k + 4 + i] = hmul2_u32(hi[i], s2);
        }
    }
}

// The combine of the split merge, run by kCombineThreads threads (the 128
// softmax threads and the 256 V-unpack threads, which are idle by then);
// ct = 0 .. kCombineThreads-1.  The rows of every split's partial for this
// CTA's dv slice are in the shared boxes, the weights in w_s and inv_den.
template <int HG, int S>
__device__ __forceinline__ void merge_combine(const DecodeArgs &a, int t, int g, int split, const uint8_t *smem,
                                              int ct) {
    using namespace nv4;
    constexpr int NQ = HG / 4;
    constexpr int D = kLatent / S;
    constexpr int C = D < 64 ? D : 64;
    constexpr int box_bytes = D * HG * 4;
    const float *w_s = reinterpret_cast<const float *>(smem + kOffMergeW);
    const float *inv_den = w_s + kMaxSplits * HG;
    __half *dst = a.out + ((int64_t)t * a.H + (int64_t)g * HG) * kLatent + split * D;
    // item = (piece q, dv d): neighbouring threads take neighbouring dv, so
    // the box reads are conflict-free; neighbouring lanes then swap halves
    // so that each stores two adjacent dv of one head (4 bytes; a warp store
    // covers 32 consecutive dv of two heads)
    const float *boxes = reinterpret_cast<const float *>(smem + kOffPartial);
    const bool odd = ct & 1;
    constexpr int kAll = D * NQ;  // even, so the two lanes of a pair are both in range or both out
    constexpr int kRounds = (kAll + kCombineThreads - 1) / kCombineThreads;
#pragma unroll 2
    for (int k = 0; k < kRounds; ++k) {
        const int item0 = ct + kCombineThreads * k;
        const bool in = item0 < kAll;
        const int item = in ? item0 : kAll - 1;  // out-of-range lanes still take part in the swap
        const int q = item / D, d = item - q * D;
        const int c = d / C, dd = d - c * C;
        const int off = c * (NQ * C * 4) + (q * C + dd) * 4;  // floats, within a box
        float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
        for (int s = 0; s < S; ++s) {
            const float4 v = *reinterpret_cast<const float4 *>(boxes + s * (box_bytes / 4) + off);
            const float4 w = *reinterpret_cast<const float4 *>(w_s + s * HG + 4 * q);
            acc.x += w.x * v.x;
            acc.y += w.y * v.y;
            acc.z += w.z * v.z;
            acc.w += w.w * v.w;
        }
        const float4 r = *reinterpret_cast<const float4 *>(inv_den + 4 * q);
        acc.x *= r.x;
        acc.y *= r.y;
        acc.z *= r.z;
        acc.w *= r.w;
        // even lane keeps heads 4q, 4q+1 and takes its neighbour's; odd lane
        // keeps heads 4q+2, 4q+3 and takes its neighbour's
        const float s0 = odd ? acc.x : acc.z, s1 = odd ? acc.y : acc.w;
        const float r0 = __shfl_xor_sync(0xffffffffu, s0, 1), r1 = __shfl_xor_sync(0xffffffffu, s1, 1);
        const float k0 = odd ? acc.z : acc.x, k1 = odd ? acc.w : acc.y;
        const int h = 4 * q + (odd ? 2 : 0);
        const int de = d & ~1;  // the pair's even dv
        // (own value, neighbour's value) in dv order
        const __half2 p0 = odd ? __floats2half2_rn(r0, k0) : __floats2half2_rn(k0, r0);
        const __half2 p1 = odd ? __floats2half2_rn(r1, k1) : __floats2half2_rn(k1, r1);
        if (in) {
            *reinterpret_cast<__half2 *>(dst + (int64_t)h * kLatent + de) = p0;
            *reinterpret_cast<__half2 *>(dst + (int64_t)(h + 1) * kLatent + de) = p1;
        }
    }
}

// The V-unpack threads' part in the split merge (vt = 0..255): they meet the
// softmax threads at the merge's named barriers and take items 128 + vt, ...
// of the combine.
template <int HG, int S>
__device__ __forceinline__ void merge_join_v(const DecodeArgs &a, int t, int g, int split, const uint8_t *smem,
                                             int vt) {
    using namespace nv4;
    const uint32_t *flag = reinterpret_cast<const uint32_t *>(smem + kOffMisc) + 1;
    named_bar(kMergeBar, kCombineThreads);  // the arrival wait is over and *flag set
    if (!*flag) return;                     // poisoned: the softmax threads write NaN
    named_bar(kMergeBar, kCombineThreads);  // weights computed, the other splits' rows landed
    merge_combine<HG, S>(a, t, g, split, smem, 128 + vt);
    named_bar(kMergeBar, kCombineThreads);
}

// Split merge, run by the 128 softmax threads of each of the S CTAs of a
// (token t, head group g).  Exchange area for the group (FP32): S partials,
// each [HG/4 pieces][512 dv][4 heads] (piece q = heads 4q .. 4q+3); split s
// owns dims [s*D, s*D + D), D = 512/S.  Before the merge every thread has
// written its dv rows of the partial straight from tensor memory (a warp
// store covers 32 consecutive dv of one piece, 512 contiguous bytes): rows
// owned by other splits to this split's partial in the exchange area, its
// own rows to shared memory box `split`.  Box layout (D dv x HG heads):
// chunks of C = min(D, 64) dv, each [HG/4][C][4] -- the shape of a tensor
// copy of C*4 floats x HG/4 rows of the exchange area.  Thread 0 announces
// the rows on the group's arrival counter (release, cumulative over the 128
// threads through the barrier before it), waits, bounded, until all S have
// arrived, then fetches the other splits' rows of this slice into boxes s !=
// split with tensor copies.  The threads combine dims [split*D, split*D + D)
// of every head:
//   out = sum_s w_s O_s / sum_s w_s l_s,  w_s = 2^(m_s - max m)
// over the splits with rows (l_s > 0); split 0 also writes
// lse = (max m + log2 of the denominator) ln 2.  The last CTA to leave resets
// the counters.  A wait that runs out sets the counter's poison bit: that CTA
// and every later one on the same counter report NVFP4MLA_DEV_TIMEOUT and
// write NaN to their slice instead of merging partials that were never
// written.
template <int HG, int S>
__device__ __forceinline__ void merge_splits_nv4(const DecodeArgs &a, const CUtensorMap *tm_xch, int t, int g,
                                                 int split, uint8_t *smem, uint64_t *bar, int mt,
                                                 [[maybe_unused]] unsigned long long t_start) {
    TRACE_SETUP();
    using namespace nv4;
    constexpr int kMergeThreads = 128;
    constexpr int NQ = HG / 4;
    constexpr int D = kLatent / S;
    constexpr int C = D < 64 ? D : 64;  // dv per tensor copy
    constexpr int box_bytes = D * HG * 4;
    uint32_t *arrive = a.counters + 2 * ((int64_t)t * a.G + g);
    uint32_t *depart = arrive + 1;
    uint32_t *flag = reinterpret_cast<uint32_t *>(smem + kOffMisc) + 1;
    float *w_s = reinterpret_cast<float *>(smem + kOffMergeW);  // [S][HG]
    float *inv_den = w_s + kMaxSplits * HG;                      // [HG]
    const int dv0 = split * D;
    named_bar(1, kMergeThreads);  // every thread's partial rows and statistics are written
    if (mt == 0) {
        TRACE(190);
        __threadfence();
        TRACE(191);
        const uint32_t old = (a.test_withhold == 2 && split == 0) ? 0u : atomicAdd(arrive, 1u);
        bool ok = (old & kPoison) == 0;
        if (ok) {
            const unsigned long long t0 = clock64();
            while (true) {
                const uint32_t v = ld_acquire_gpu(arrive);
                if (v & kPoison) {
                    ok = false;
                    break;
                }
                if (v >= (uint32_t)S) break;
                if (clock64() - t0 > a.wait_cycles) {
                    ok = false;
                    break;
                }
                __nanosleep(32);
            }
        }
        if (!ok) {
            atomicOr(arrive, kPoison);
            if (a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
        } else {
            fence_proxy_async_global();  // the other splits' rows, seen through the counter, to the copy engine
            // this barrier's first phase tracked the Q copies; they have
            // landed before its second phase is armed
            if (!mbar_wait(bar, 0, a.wait_cycles) && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
            mbar_arrive_expect_tx(bar, (uint32_t)((S - 1) * box_bytes));
            const int32_t row_g = ((t * a.G + g) * S) * NQ;  // first exchange row of the group
#pragma unroll 1
            for (int s = 0; s < S; ++s) {
                if (s == split) continue;
#pragma unroll
                for (int c = 0; c < D / C; ++c)
                    tma_load_2d(smem + kOffPartial + s * box_bytes + c * (NQ * C * 16), tm_xch, (dv0 + c * C) * 4,
                                row_g + s * NQ, bar);
            }
        }
        *flag = ok ? 1u : 0u;
        TRACE(192);
    }
    named_bar(kMergeBar, kCombineThreads);  // with the V-unpack threads (merge_join_v)
    __half *dst = a.out + ((int64_t)t * a.H + (int64_t)g * HG) * kLatent + dv0;
    if (!*flag) {  // poisoned: make the failure visible in the output
        for (int item = mt; item < HG * D; item += kMergeThreads) {
            const int h = item / D, d = item - h * D;
            dst[(int64_t)h * kLatent + d] = __float2half_rn(NAN);
        }
        if (split == 0 && mt < HG) a.lse[(int64_t)t * a.H + (int64_t)g * HG + mt] = NAN;
        return;
    }
    if (mt < HG) {  // split weights from the statistics while the rows travel
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
    const bool landed = mbar_wait(bar, 1, a.wait_cycles);  // the tensor copies (phase 1 of the Q barrier)
    if (!landed && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
    named_bar(kMergeBar, kCombineThreads);
    if (mt == 0) TRACE(193);
    merge_combine<HG, S>(a, t, g, split, smem, mt);
    named_bar(kMergeBar, kCombineThreads);
    if (mt == 0) {
        TRACE(194);
        const uint32_t old = atomicAdd(depart, 1u);
        if (old == (uint32_t)S - 1u) {  // every CTA of the group is past its wait
            atomicExch(arrive, 0u);
            atomicExch(depart, 0u);
        }
    }
}

template <int HG>
__global__ void __launch_bounds__(nv4::kThreads, 1)
    nvfp4_decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tm_qn,
                        const __grid_constant__ CUtensorMap tm_qr, const __grid_constant__ CUtensorMap tm_xch) {
    using namespace nv4;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int split = blockIdx.x % a.S;
    const int rest = blockIdx.x / a.S;
    const int g = rest % a.G;
    const int t = rest / a.G;
#ifdef NVFP4MLA_TRACE
    const unsigned long long t_start = clock64();
#else
    const unsigned long long t_start = 0;  // timestamps exist only in trace builds
#endif
    TRACE_SETUP();

    if (smem_u32(smem) & 1023u) {  // the swizzled operand layouts need a 1 KB aligned base
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
    if (warp == 1 && lane == 0) {
        for (int b = 0; b < kBarsUsed; ++b) {
            uint32_t count = 1;
            if (b >= BAR_RAW_FULL && b < BAR_RAW_FULL + kRawSlots) count = 64;  // cp.async arrivals
            else if (b == BAR_ROWS0) count = kTile0Threads;
            else if (b == BAR_K0DONE) count = 8;
            else if (b >= BAR_RAW_FREE && b < BAR_RAW_FREE + kRawSlots) count = 8;
            else if (b >= BAR_K_FULL && b < BAR_K_FULL + kKSlots) count = 4;
            else if (b >= BAR_V_FULL && b < BAR_V_FULL + kVSlots) count = 4;
            else if (b == BAR_P_FULL || b == BAR_S_FREE || b == BAR_S_FREE + 1) count = 4;
            mbar_init(&bars[b], count);
        }
        fence_mbar_init();
        // Q of (t, heads g*HG ..): nine tensor copies (box 64 dims x HG heads,
        // 128-byte swizzle) straight into the K-major operand layout.
        const int32_t row = t * a.H + g * HG;
        mbar_arrive_expect_tx(&bars[BAR_Q], (uint32_t)(HG * kDim * 2));
#pragma unroll 1
        for (int c = 0; c < 8; ++c) tma_load_2d(smem + kOffQ + c * (HG * 128), &tm_qn, 64 * c, row, &bars[BAR_Q]);
        tma_load_2d(smem + kOffQ + 8 * (HG * 128), &tm_qr, 0, row, &bars[BAR_Q]);
    }
    if (warp == 2) {
        tmem_alloc(&misc[0], kTmemCols);
        tmem_relinquish();
    }
    if (tid < HG) m_s[tid] = -INFINITY;

    // Compact the token's list: keep valid entries in list order; this CTA
    // keeps entries [lo, hi) of the compacted order.
    const int32_t *lst = a.indices + (int64_t)t * a.topk;
    int32_t vals[4];
    uint32_t bal[4];
    bool bad = false;
    // all of a thread's list loads (and then its block-table loads) are in
    // flight together; entries 512k + tid, warps 16.. hold none (p >= 2048)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int p = tid + 512 * k;
        vals[k] = (p < a.topk && tid < 512) ? __ldg(lst + p) : -1;
    }
    bool entry_bad[4] = {false, false, false, false};
    if (a.block_table) {  // request-local position -> slot through the block table
        int32_t blk[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
            blk[k] = (vals[k] >= 0 && (int64_t)vals[k] < a.max_pos)
                         ? __ldg(a.block_table + (int64_t)t * a.table_stride + (vals[k] >> a.page_shift))
                         : -1;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (vals[k] < 0) continue;
            const int64_t slot = blk[k] >= 0 ? ((int64_t)blk[k] << a.page_shift) + (vals[k] & ((1 << a.page_shift) - 1))
                                             : -1;
            entry_bad[k] = slot < 0 || slot >= a.num_slots;
            vals[k] = entry_bad[k] ? -1 : (int32_t)slot;
        }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int p = tid + 512 * k;
        const int32_t v = vals[k];
        const bool ok = v >= 0 && (int64_t)v < a.num_slots;
        bad |= (p < a.topk) && (entry_bad[k] || v < -1 || (int64_t)v >= a.num_slots);
        bal[k] = __ballot_sync(0xffffffffu, ok);
        if (lane == 0 && warp < 16) cnt_s[k * 16 + warp] = __popc(bal[k]);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0 && split == 0 && g == 0 && a.dev_status)
        atomicOr(a.dev_status, NVFP4MLA_DEV_BAD_INDEX);
    __syncthreads();
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
            const int j = k * 16 + (warp & 15);
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
            if (pos >= lo && pos < hi) idx_s[pos - lo] = vals[k];
        }
    }
    tc_fence_before();
    __syncthreads();  // also orders cnt_s reads before the softmax reuses the region
    tc_fence_after();
    const uint32_t tmem = misc[0];
    auto tile_rows = [&](int j) { return min(kTileRows, n_mine - kTileRows * j); };
    if (tid == 0) TRACE(0);

    if (warp < 4) {
        regs_dec<kRegsCtl>();
        if (warp == 0) {
            // ------------------------------------------------- score MMAs
            // S^T(j) = K(j) Q^T into S buffer j & 1, chunk by chunk as the K
            // ring fills; buffer j & 1 is reused once the softmax of tile
            // j - 2 has read it.
            const uint32_t id_qk = idesc_f16_f32(128, HG, false, false);
            const uint64_t dQ0 = smem_desc(smem_u32(smem + kOffQ), 16, 1024);
            bool ok = warp_wait(&bars[BAR_Q], 0, a.wait_cycles);  // always: the copies must land before the CTA may exit
            if (lane == 0) TRACE(1);
            uint32_t kn = 0;
            for (int j = 0; j < ntiles && ok; ++j) {
                if (j >= 2 && !warp_wait(&bars[BAR_S_FREE + (j & 1)], ((j >> 1) - 1) & 1, a.wait_cycles)) {
                    ok = false;
                    break;
                }
                const uint32_t dS = tmem + kColS + 64u * (uint32_t)(j & 1);
                if (lane == 0 && j < 8) TRACE(10 + 8 * j);
                uint64_t dq = dQ0;
#pragma unroll 1
                for (int c = 0; c < kKChunks; ++c) {
                    const uint32_t slot = kn & 3u;
                    if (!warp_wait(&bars[BAR_K_FULL + slot], (kn >> 2) & 1u, a.wait_cycles)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ak = tmem + kColK + 32u * slot;
                    mma_ts_warp(dS, ak, dq, id_qk, c != 0);
                    mma_ts_warp(dS, ak + 8, dq + 2, id_qk, 1u);
                    mma_ts_warp(dS, ak + 16, dq + 4, id_qk, 1u);
                    mma_ts_warp(dS, ak + 24, dq + 6, id_qk, 1u);
                    mma_commit_warp(&bars[BAR_K_FREE + slot]);
                    if (lane == 0 && j == 1) TRACE(240 + c);
                    dq += (uint64_t)((HG * 128) >> 4);
                    ++kn;
                }
                if (!ok) break;
                mma_commit_warp(&bars[BAR_S_FULL + (j & 1)]);
                if (lane == 0 && j < 8) TRACE(11 + 8 * j);
            }
            if (!ok && lane == 0 && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
            mma_commit_warp(&bars[BAR_DRAIN]);  // nothing may still read or write TMEM at teardown
            warp_wait(&bars[BAR_DRAIN], 0, a.wait_cycles);
        } else if (warp == 2) {
            // ------------------------------------------------ output MMAs
            // O^T += V^T(j) P^T(j), one 16-row V ring slot at a time, once the
            // softmax has written P^T(j) (and rescaled O^T if it had to).
            const uint32_t id_pv = idesc_f16_f32(128, HG, true, true);
            const uint64_t dV0 = smem_desc(smem_u32(smem + kOffV), 2048, 1024);
            const uint64_t dP0 = smem_desc(smem_u32(smem + kOffP), 2048, 1024);
            bool ok = true;
            uint32_t vn = 0;
            for (int j = 0; j < ntiles && ok; ++j) {
                if (!warp_wait(&bars[BAR_P_FULL], j & 1, a.wait_cycles)) {
                    ok = false;
                    break;
                }
                if (lane == 0 && j < 8) TRACE(12 + 8 * j);
                tc_fence_after();
                uint64_t dp = dP0;
#pragma unroll 1
                for (int gi = 0; gi < kVGroups; ++gi) {
                    const uint32_t slot = vn % kVSlots;
                    if (!warp_wait(&bars[BAR_V_FULL + slot], (vn / kVSlots) & 1u, a.wait_cycles)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0 && j == 1) TRACE(340 + gi);
                    tc_fence_after();
                    const uint64_t dv = dV0 + (uint64_t)(slot * (kVSlotBytes >> 4));
                    const uint32_t acc = (j > 0 || gi > 0) ? 1u : 0u;
                    if (lane == 0 && j == 1) TRACE(350 + gi);
                    mma_ss_warp(tmem + kColO, dv, dp, id_pv, acc);
                    if (lane == 0 && j == 1) TRACE(360 + gi);
                    mma_ss_warp(tmem + kColO + HG, dv + (uint64_t)(4096 >> 4), dp, id_pv, acc);
                    mma_ss_warp(tmem + kColO + 2 * HG, dv + (uint64_t)(2 * (4096 >> 4)), dp, id_pv, acc);
                    mma_ss_warp(tmem + kColO + 3 * HG, dv + (uint64_t)(3 * (4096 >> 4)), dp, id_pv, acc);
                    if (lane == 0 && j == 1) TRACE(370 + gi);
                    mma_commit_warp(&bars[BAR_V_FREE + slot]);
                    if (lane == 0 && j == 1) TRACE(260 + gi);
                    dp += (uint64_t)(2048 >> 4);
                    ++vn;
                }
                if (!ok) break;
                mma_commit_warp(&bars[BAR_PV_DONE]);
                if (lane == 0 && j < 8) TRACE(13 + 8 * j);
            }
            if (!ok && lane == 0 && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
            mma_commit_warp(&bars[BAR_DRAIN_PV]);  // nothing may still read or write TMEM at teardown
            warp_wait(&bars[BAR_DRAIN_PV], 0, a.wait_cycles);
        } else if (warp == 1 || warp == 3) {
            // ---------------------------------------------------- gather
            // 64 threads copy the tile's rows in 16-byte pieces (22 per row)
            // with cp.async; each thread's arrival on RAW_FULL fires when its
            // own copies have landed.
            const int gt = (warp == 1 ? 0 : 32) + lane;
            bool ok = true;
            for (int j = 0; j < ntiles; ++j) {
                const int slot = j % kRawSlots;
                if (j >= kRawSlots && !warp_wait(&bars[BAR_RAW_FREE + slot], ((j / kRawSlots) - 1) & 1, a.wait_cycles)) {
                    ok = false;
                    break;
                }
                const int nrows = tile_rows(j);
                uint8_t *dst = smem + kOffRaw + slot * kRawSlotBytes;
                const int32_t *ids = idx_s + kTileRows * j;
                const int items = nrows * (kRowBytes / 16);
                // the first tile is shared with the V warps (items gt, gt + 320, ...)
                const int step = j == 0 ? kTile0Threads : 64;
#pragma unroll 4
                for (int it = gt; it < items; it += step) {
                    const int r = it / (kRowBytes / 16), k = it - r * (kRowBytes / 16);
                    cp_async16(dst + r * kRawStride + 16 * k, a.src + (int64_t)ids[r] * kRowBytes + 16 * k);
                }
                cp_async_mbar_arrive(&bars[BAR_RAW_FULL + slot]);
                if (j == 0) cp_async_mbar_arrive(&bars[BAR_ROWS0]);
                if (gt == 0 && j < 8) TRACE(80 + j);
            }
            // copies still in flight land before the CTA may exit
            asm volatile("cp.async.wait_all;" ::: "memory");
            if (!ok && lane == 0 && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
        }
        __syncwarp();
    } else if (warp < kSoftWarp0) {
        // ------------------------------------------------------- K unpack
        regs_dec<kRegsK>();
        const int kw = warp - kKWarp0;  // 0..7
        const int quarter = warp & 3;   // TMEM lanes this warp may reach
        const int half = kw >> 2;       // even or odd chunks
        const int r = 32 * quarter + lane;
        const uint32_t lane_base = (uint32_t)(32 * quarter) << 16;
        bool ok = true;
        for (int j = 0; j < ntiles && ok; ++j) {
            const int rslot = j % kRawSlots;
            // the first tile's rows are complete once all kTile0Threads
            // copiers' copies have landed (ROWS0); RAW_FULL's first phase
            // tracks only the gather warps' share and nobody waits on it
            const bool landed = j == 0 ? warp_wait(&bars[BAR_ROWS0], 0, a.wait_cycles)
                                       : warp_wait(&bars[BAR_RAW_FULL + rslot], (j / kRawSlots) & 1, a.wait_cycles);
            if (!landed) {
                ok = false;
                break;
            }
            if (kw == 0 && lane == 0 && j < 8) TRACE(100 + j);
            const bool valid = r < tile_rows(j);
            const uint8_t *row = smem + kOffRaw + rslot * kRawSlotBytes + r * kRawStride;
#pragma unroll 1
            for (int c = half; c < kKChunks; c += 2) {
                const uint32_t n = (uint32_t)(kKChunks * j + c);
                const uint32_t slot = n & 3u;
                uint32_t o[32];
                if (valid) {
                    if (c < 8) {
                        unpack_latent64(lds128(row + 32 * c), lds128(row + 32 * c + 16), lds32(row + kScaleOff + 4 * c), o);
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const uint4 w = lds128(row + kRopeOff + 16 * q);
                            uint32_t e[4];
                            e4m3x8_to_f16x8(w.x, w.y, e);
                            o[8 * q + 0] = e[0];
                            o[8 * q + 1] = e[1];
                            o[8 * q + 2] = e[2];
                            o[8 * q + 3] = e[3];
                            e4m3x8_to_f16x8(w.z, w.w, e);
                            o[8 * q + 4] = e[0];
                            o[8 * q + 5] = e[1];
                            o[8 * q + 6] = e[2];
                            o[8 * q + 7] = e[3];
                        }
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0u;
                }
                if (n >= 4 && !warp_wait(&bars[BAR_K_FREE + slot], ((n >> 2) - 1) & 1u, a.wait_cycles)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                tmem_st32(tmem + lane_base + kColK + 32u * slot, o);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[BAR_K_FULL + slot]);
                if ((kw & 3) == 0 && lane == 0 && j == 1) TRACE(200 + c);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[BAR_RAW_FREE + rslot]);
            if (j == 0 && lane == 0) mbar_arrive(&bars[BAR_K0DONE]);
            if (kw == 0 && lane == 0 && j < 8) TRACE(110 + j);
        }
        if (!ok && lane == 0 && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
    } else if (warp < kVWarp0) {
        // -------------------------------------------------------- softmax
        regs_inc<kRegsSoft>();
        const int st = tid - 32 * kSoftWarp0;  // tile row == TMEM lane
        const int wq = st >> 5;
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        uint8_t *p_tile = smem + kOffP;
        // Scores are read from tensor memory twice, HC columns at a time:
        // once to decide whether any head's reference max must move, once to
        // form P.  The reference max is read from shared memory with 16-byte
        // broadcast loads.  Row sums: each HC-column block of P is folded
        // over the warp's 32 rows (transpose reduction) once P^T is
        // published, so a lane keeps only the sums of NL heads, lp_head(k).
        constexpr int HC = HG > 32 ? 32 : HG;
        constexpr int NB = HG / HC;            // column blocks
        constexpr int NL = NB * (HC >= 32 ? 1 : 1);
        auto lp_head = [&](int k) { return HC >= 32 ? HC * k + lane : (lane >> 1); };
        float lp[NL];
#pragma unroll
        for (int k = 0; k < NL; ++k) lp[k] = 0.0f;
        bool ok = true;
        // Every wait's outcome is agreed by all 128 threads (bar.red.or), so
        // the four warps always meet at the same named barriers.
        for (int j = 0; j < ntiles; ++j) {
            if (named_bar_or(1, 128, !warp_wait(&bars[BAR_S_FULL + (j & 1)], (j >> 1) & 1, a.wait_cycles))) {
                ok = false;
                break;
            }
            if (st == 0 && j < 8) TRACE(120 + j);
            tc_fence_after();
            const uint32_t s_addr = tmem + lane_base + kColS + 64u * (uint32_t)(j & 1);
            const bool valid = st < tile_rows(j);
            // the first tile always moves every reference max (they start at
            // -inf), so only later tiles read the scores for the check
            bool need = j == 0;
            if (j > 0) {
                uint32_t rs[HG];  // every score of the row: all loads in flight, one wait
#pragma unroll
                for (int c0 = 0; c0 < HG; c0 += HC) tmem_ld_cols<HC>(s_addr + c0, *reinterpret_cast<uint32_t(*)[HC]>(rs + c0));
                tmem_ld_wait();
#pragma unroll
                for (int h = 0; h < HG; h += 4) {
                    const float4 m4 = *reinterpret_cast<const float4 *>(m_s + h);
                    need |= __uint_as_float(rs[h + 0]) * a.scale_log2 > m4.x + kRescaleThreshold;
                    need |= __uint_as_float(rs[h + 1]) * a.scale_log2 > m4.y + kRescaleThreshold;
                    need |= __uint_as_float(rs[h + 2]) * a.scale_log2 > m4.z + kRescaleThreshold;
                    need |= __uint_as_float(rs[h + 3]) * a.scale_log2 > m4.w + kRescaleThreshold;
                }
            }
            const bool rescale = named_bar_or(1, 128, valid && need);
            if (rescale) {
                uint32_t rsa[HG];  // every score of the row: all loads in flight, one wait
#pragma unroll
                for (int c0 = 0; c0 < HG; c0 += 16) tmem_ld16(s_addr + c0, *reinterpret_cast<uint32_t(*)[16]>(rsa + c0));
                tmem_ld_wait();
#pragma unroll
                for (int c0 = 0; c0 < HG; c0 += 16) {  // column max, 16 heads at a time
                    float mx[16];
#pragma unroll
                    for (int h = 0; h < 16; ++h) mx[h] = valid ? __uint_as_float(rsa[c0 + h]) * a.scale_log2 : -INFINITY;
                    warp_transpose_reduce<16, true>(mx, lane);
                    if (!(lane & 1)) red_s[wq * 64 + c0 + transposed_col<16>(lane, 0)] = mx[0];
                }
                named_bar(1, 128);
                if (st < HG) {
                    const float old = m_s[st];
                    float nm = old;
#pragma unroll
                    for (int w = 0; w < 4; ++w) nm = fmaxf(nm, red_s[w * 64 + st]);
                    aux_s[st] = (old == -INFINITY) ? 0.0f : ex2(old - nm);
                    m_s[st] = nm;
                }
                named_bar(1, 128);
#pragma unroll
                for (int k = 0; k < NL; ++k) lp[k] *= aux_s[lp_head(k)];
            }
            // P (FP16, packed in registers) and this tile's row sums need
            // neither O^T nor the P^T buffer, so they are formed while the
            // output MMAs of the previous tile may still run; only the P^T
            // stores (and a rare O^T rescale) wait for those to finish.
            uint32_t pk[HG / 2];
            uint32_t rsp[HG];  // every score of the row: all loads in flight, one wait
#pragma unroll
            for (int c0 = 0; c0 < HG; c0 += HC) tmem_ld_cols<HC>(s_addr + c0, *reinterpret_cast<uint32_t(*)[HC]>(rsp + c0));
            tmem_ld_wait();
#pragma unroll
            for (int c0 = 0; c0 < HG; c0 += HC) {
                float pv[HC];
                {
                    const uint32_t *rs = rsp + c0;
#pragma unroll
                    for (int h = 0; h < HC; h += 4) {
                        const float4 m4 = *reinterpret_cast<const float4 *>(m_s + c0 + h);
                        pv[h + 0] = valid ? ex2(__uint_as_float(rs[h + 0]) * a.scale_log2 - m4.x) : 0.0f;
                        pv[h + 1] = valid ? ex2(__uint_as_float(rs[h + 1]) * a.scale_log2 - m4.y) : 0.0f;
                        pv[h + 2] = valid ? ex2(__uint_as_float(rs[h + 2]) * a.scale_log2 - m4.z) : 0.0f;
                        pv[h + 3] = valid ? ex2(__uint_as_float(rs[h + 3]) * a.scale_log2 - m4.w) : 0.0f;
                    }
                }
#pragma unroll
                for (int h = 0; h < HC; h += 2) pk[(c0 + h) / 2] = pack_half2(pv[h], pv[h + 1]);
                warp_transpose_reduce<HC, false>(pv, lane);
                lp[c0 / HC] += pv[0];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[BAR_S_FREE + (j & 1)]);  // this warp's reads of S(j) are done
            // O^T and P^T belong to the output MMAs of the previous tile
            // until they are done.
            if (j > 0) {
                if (named_bar_or(1, 128, !warp_wait(&bars[BAR_PV_DONE], (j - 1) & 1, a.wait_cycles))) {
                    ok = false;
                    break;
                }
                if (st == 0 && j < 8) TRACE(130 + j);
                tc_fence_after();
                if (rescale) {
#pragma unroll 1
                    for (int b = 0; b < 4; ++b) {
#pragma unroll
                        for (int cb = 0; cb < HG; cb += 16) {
                            uint32_t rr[16];
                            const uint32_t addr = tmem + lane_base + kColO + b * HG + cb;
                            tmem_ld16(addr, rr);
                            tmem_ld_wait();
#pragma unroll
                            for (int h = 0; h < 16; ++h) rr[h] = __float_as_uint(__uint_as_float(rr[h]) * aux_s[cb + h]);
                            tmem_st16(addr, rr);
                        }
                    }
                    tmem_st_wait();
                }
            }
#pragma unroll
            for (int jj = 0; jj < HG / 8; ++jj)
                *reinterpret_cast<uint4 *>(p_tile + sw128_offset(st, jj)) =
                    make_uint4(pk[4 * jj], pk[4 * jj + 1], pk[4 * jj + 2], pk[4 * jj + 3]);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0 && a.test_withhold != 1) mbar_arrive(&bars[BAR_P_FULL]);
            if (st == 0 && j < 8) TRACE(140 + j);
        }
        if (!ok && a.dev_status && lane == 0) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
        // ---------------------------------------------------------- epilogue
        if (st == 0) TRACE(170);
        const bool have = ok && ntiles > 0;
        if (HC >= 32 || !(lane & 1)) {  // row sums: one partial per warp and head
#pragma unroll
            for (int k = 0; k < NL; ++k) red_s[wq * 64 + lp_head(k)] = lp[k];
        }
        named_bar(1, 128);
        if (st < HG) {
            const float l = have ? red_s[st] + red_s[64 + st] + red_s[128 + st] + red_s[192 + st] : 0.0f;
            const float m = m_s[st];
            aux_s[st] = l > 0.0f ? 1.0f / l : 0.0f;
            const int64_t hrow = (int64_t)t * a.H + (int64_t)g * HG + st;
            if (a.S == 1) {
                a.lse[hrow] = l > 0.0f ? (m + lg2(l)) * 0.69314718055994531f : -INFINITY;
            } else {
                const int64_t prow = ((int64_t)t * a.S + split) * a.H + (int64_t)g * HG + st;
                a.ws_ml[2 * prow] = l > 0.0f ? m : -INFINITY;
                a.ws_ml[2 * prow + 1] = l;
            }
        }
        named_bar(1, 128);
        bool fin = have;
        if (have) {  // O^T is final once the last tile's output MMAs are done
            fin = !named_bar_or(1, 128, !warp_wait(&bars[BAR_PV_DONE], (ntiles - 1) & 1, a.wait_cycles));
            if (!fin && st == 0 && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
            tc_fence_after();
        }
        if (st == 0) TRACE(171);
        // Every K-unpack warp is past its last raw tile once the last output
        // MMAs are done (they needed every chunk), so the raw ring is free.
        uint8_t *stage = smem + kOffStage;
        if (a.S == 1) {
            // O^T (TMEM lanes = dv) -> normalised FP16 rows [HG][512] staged
            // in the raw ring, then one bulk copy of HG x 1 KB.
            constexpr int HC = HG > 32 ? 32 : HG;  // columns per TMEM load
#pragma unroll 1
            for (int b = 0; b < 4; ++b) {
                const int dv = 128 * b + st;
#pragma unroll
                for (int h0 = 0; h0 < HG; h0 += HC) {
                    uint32_t rr[HC];
                    if (fin) {
                        tmem_ld_cols<HC>(tmem + lane_base + kColO + b * HG + h0, rr);
                        tmem_ld_wait();
                    } else {
#pragma unroll
                        for (int h = 0; h < HC; ++h) rr[h] = 0u;
                    }
#pragma unroll
                    for (int h = 0; h < HC; ++h)
                        reinterpret_cast<__half *>(stage)[(h0 + h) * kLatent + dv] =
                            __float2half_rn(__uint_as_float(rr[h]) * aux_s[h0 + h]);
                }
            }
            fence_proxy_async_smem();
            named_bar(1, 128);
            if (st == 0) {
                bulk_s2g(a.out + ((int64_t)t * a.H + (int64_t)g * HG) * kLatent, stage, HG * kLatent * 2);
                bulk_commit_wait_read();
            }
        } else {
            // Unnormalised partial O of this split, row dv = this thread's
            // TMEM lane in each 128-dv block, as 4-head pieces: rows owned by
            // another split go straight to this split's partial in the
            // exchange area ([HG/4][512][4]; a warp store covers 32
            // consecutive dv of a piece), this split's own rows to shared
            // box `split` (chunks of C dv, [HG/4][C][4] each), over the P^T
            // and ring regions, which no MMA or copy uses any more.  A warp's
            // 32 rows never straddle two owners (D = 512/S is a multiple of
            // 32).
            const int D = kLatent / a.S;
            const int C = D < 64 ? D : 64;
            constexpr int NQ = HG / 4;
            float *own = reinterpret_cast<float *>(smem + kOffPartial + split * (D * HG * 4));
            float *xch = a.ws_o + (((int64_t)t * a.G + g) * a.S + split) * (int64_t)NQ * kLatent * 4;
            constexpr int HC = HG > 32 ? 32 : HG;
#pragma unroll 1
            for (int b = 0; b < 4; ++b) {
                const int dv = 128 * b + st;
                const bool mine = dv / D == split;
                const int d = dv - split * D, c = d / C, dd = d - (d / C) * C;
                uint32_t rr[HG];  // every head of row dv: all loads issued, one wait
                if (fin) {
#pragma unroll
                    for (int h0 = 0; h0 < HG; h0 += HC)
                        tmem_ld_cols<HC>(tmem + lane_base + kColO + b * HG + h0, *reinterpret_cast<uint32_t(*)[HC]>(rr + h0));
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int h = 0; h < HG; ++h) rr[h] = 0u;
                }
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                    const float4 v = make_float4(__uint_as_float(rr[4 * q]), __uint_as_float(rr[4 * q + 1]),
                                                 __uint_as_float(rr[4 * q + 2]), __uint_as_float(rr[4 * q + 3]));
                    if (mine)
                        *reinterpret_cast<float4 *>(own + c * (NQ * C * 4) + (q * C + dd) * 4) = v;
                    else
                        __stcg(reinterpret_cast<float4 *>(xch + ((int64_t)q * kLatent + dv) * 4), v);
                }
            }
            if (st == 0) TRACE(172);
            switch (a.S) {
                case 2: merge_splits_nv4<HG, 2>(a, &tm_xch, t, g, split, smem, &bars[BAR_Q], st, t_start); break;
                case 4: merge_splits_nv4<HG, 4>(a, &tm_xch, t, g, split, smem, &bars[BAR_Q], st, t_start); break;
                case 8: merge_splits_nv4<HG, 8>(a, &tm_xch, t, g, split, smem, &bars[BAR_Q], st, t_start); break;
                default: merge_splits_nv4<HG, 16>(a, &tm_xch, t, g, split, smem, &bars[BAR_Q], st, t_start); break;
            }
            if (st == 0) TRACE(174);
        }
    } else {
        // -------------------------------------------------------- V unpack
        // Two sets of four warps alternate the 16-row groups of a tile: set
        // vs converts groups vs, vs + 2, ... into ring slot vs, so each set
        // has two group periods for its own convert-and-store work.  Slot
        // layout (MN-major A operand of the output MMA): dv group dg (64
        // dims) at dg * 2048, row r of the 16 at r * 128, 16-byte chunk jj
        // swizzled by the row.  Thread = (row r, dv group dg); the rows are
        // read from L2 (the gather brought them in a tile earlier).
        if (kRegsV < kRegsLaunch) regs_dec<kRegsV < kRegsLaunch ? kRegsV : kRegsLaunch - 8>();
        if (ntiles > 0) {  // this thread's share of the first tile's row copies (items 64 + v, 64 + v + 320, ...)
            const int items = tile_rows(0) * (kRowBytes / 16);
            uint8_t *dst = smem + kOffRaw;
#pragma unroll 4
            for (int it = 64 + (tid - 32 * kVWarp0); it < items; it += kTile0Threads) {
                const int r = it / (kRowBytes / 16), k = it - r * (kRowBytes / 16);
                cp_async16(dst + r * kRawStride + 16 * k, a.src + (int64_t)idx_s[r] * kRowBytes + 16 * k);
            }
            cp_async_mbar_arrive(&bars[BAR_ROWS0]);
        }
        const int vs = (warp - kVWarp0) >> 2;  // V set: 0 or 1
        const int vw = (warp - kVWarp0) & 3;
        const int r = lane & 15;
        const int dg = 2 * vw + (lane >> 4);
        bool ok = true;
        uint32_t vn = (uint32_t)vs;  // ring position of this set's next group (groups alternate sets)
        for (int j = 0; j < ntiles && ok; ++j) {
            // Rows are read once they are in L2, which also keeps these loads
            // from racing the gather to HBM: the first tile's once its K has
            // been unpacked (a barrier that completes only once; V is needed
            // only after the tile's scores, and starting earlier would take
            // issue slots from that unpack), later tiles' once the softmax has
            // read their scores.  (S_FREE, unlike S_FULL or the raw ring,
            // cannot complete this buffer's next phase, tile j + 2, before
            // these warps finish tile j: the softmax reaches tile j + 2 only
            // after the output MMAs of tile j, which need every V group of it.)
            const bool rows_in = j == 0 ? warp_wait(&bars[BAR_K0DONE], 0, a.wait_cycles)
                                        : warp_wait(&bars[BAR_S_FREE + (j & 1)], (j >> 1) & 1, a.wait_cycles);
            if (!rows_in) {
                ok = false;
                break;
            }
            if (vs == 0 && vw == 0 && lane == 0 && j < 8) TRACE(150 + j);
            const int nrows = tile_rows(j);
            const int32_t *ids = idx_s + kTileRows * j;
            auto load = [&](int gi, uint4 &w0, uint4 &w1, uint32_t &sc) {
                const int e = kVRows * gi + r;
                if (e < nrows) {
                    const uint8_t *rp = a.src + (int64_t)ids[e] * kRowBytes;
                    w0 = __ldg(reinterpret_cast<const uint4 *>(rp + 32 * dg));
                    w1 = __ldg(reinterpret_cast<const uint4 *>(rp + 32 * dg + 16));
                    sc = __ldg(reinterpret_cast<const uint32_t *>(rp + kScaleOff + 4 * dg));
                } else {
                    w0 = w1 = make_uint4(0u, 0u, 0u, 0u);
                    sc = 0u;
                }
            };
            // this set's next two groups are in flight ahead of the one
            // being converted
            // (a rolled loop: this role's code stays small)
            constexpr int kMine = kVGroups / 2;
            uint4 a0, a1, b0, b1;  // rows of this set's current and next group
            uint32_t as, bs;
            load(vs, a0, a1, as);
            load(vs + 2, b0, b1, bs);
#pragma unroll 1
            for (int m = 0; m < kMine; ++m) {
                const uint32_t slot = vn % kVSlots;
                uint8_t *base = smem + kOffV + slot * kVSlotBytes + dg * 2048;
                uint32_t o[32];
                unpack_latent64(a0, a1, as, o);
                a0 = b0;
                a1 = b1;
                as = bs;
                if (m + 2 < kMine) load(vs + 2 * (m + 2), b0, b1, bs);
                if (vw == 0 && lane == 0 && j == 1) TRACE(300 + 20 * vs + 4 * m);
                if (vn >= kVSlots && !warp_wait(&bars[BAR_V_FREE + slot], ((vn / kVSlots) - 1) & 1u, a.wait_cycles)) {
                    ok = false;
                    break;
                }
                if (vw == 0 && lane == 0 && j == 1) TRACE(301 + 20 * vs + 4 * m);
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    *reinterpret_cast<uint4 *>(base + sw128_offset(r, jj)) =
                        make_uint4(o[4 * jj], o[4 * jj + 1], o[4 * jj + 2], o[4 * jj + 3]);
                fence_proxy_async_smem();
                if (vw == 0 && lane == 0 && j == 1) TRACE(302 + 20 * vs + 4 * m);
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[BAR_V_FULL + slot]);
                if (vw == 0 && lane == 0 && j == 1) TRACE(220 + vs + 2 * m);
                vn += 2;
            }
            if (vs == 0 && vw == 0 && lane == 0 && j < 8) TRACE(160 + j);
        }
        asm volatile("cp.async.wait_all;" ::: "memory");  // its first-tile copies land before the CTA may exit
        if (!ok && lane == 0 && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
        const int vt = tid - 32 * kVWarp0;
        switch (a.S) {  // the split merge's combine (the softmax warps run the rest of it)
            case 1: break;
            case 2: merge_join_v<HG, 2>(a, t, g, split, smem, vt); break;
            case 4: merge_join_v<HG, 4>(a, t, g, split, smem, vt); break;
            case 8: merge_join_v<HG, 8>(a, t, g, split, smem, vt); break;
            default: merge_join_v<HG, 16>(a, t, g, split, smem, vt); break;
        }
    }

    // ---------------------------------------------------------------- teardown
    if (tid == 32 * kSoftWarp0) TRACE(180);
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int HG>
static cudaError_t launch_nv4(const DecodeArgs &a, int64_t nblocks, cudaStream_t stream) {
    auto kern = nvfp4_decode_kernel<HG>;
    static std::atomic<bool> attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev].load(std::memory_order_acquire)) {
        // The per-role register split (setmaxnreg) assumes the block starts
        // with kRegsLaunch registers per thread; with fewer, an increase
        // could never be granted, so refuse to launch.
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        if (fa.numRegs != nv4::kRegsLaunch || fa.maxThreadsPerBlock < nv4::kThreads) return cudaErrorInvalidConfiguration;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, nv4::kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev].store(true, std::memory_order_release);
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)nblocks);
    cfg.blockDim = dim3(nv4::kThreads);
    cfg.dynamicSmemBytes = nv4::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.S > 1 ? 1 : 0;  // split launches need every CTA resident at once
    CUtensorMap tm_qn, tm_qr, tm_xch;
    const uint64_t rows = (uint64_t)a.T * (uint64_t)a.H;
    if (!make_q_map(&tm_qn, a.q_nope, rows, kLatent, HG) || !make_q_map(&tm_qr, a.q_rope, rows, kRope, HG))
        return cudaErrorInvalidValue;
    if (a.S > 1) {  // exchange rows: T * H * S / 4 pieces of 2048 floats; one copy = C dv x HG/4 pieces
        const int D = kLatent / a.S, C = D < 64 ? D : 64;
        if (!make_xch_map(&tm_xch, a.ws_o, rows * (uint64_t)a.S / 4, (uint32_t)(C * 4), HG / 4))
            return cudaErrorInvalidValue;
    } else {
        tm_xch = tm_qn;  // unused without splits
    }
    return cudaLaunchKernelEx(&cfg, kern, a, tm_qn, tm_qr, tm_xch);
}

cudaError_t launch_nvfp4_decode(const DecodeArgs &a, int heads_per_cta, int64_t nblocks, cudaStream_t stream) {
    switch (heads_per_cta) {
        case 16: return launch_nv4<16>(a, nblocks, stream);
        case 32: return launch_nv4<32>(a, nblocks, stream);
        case 64: return launch_nv4<64>(a, nblocks, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace nvfp4mla
