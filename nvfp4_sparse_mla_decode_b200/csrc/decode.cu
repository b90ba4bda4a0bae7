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
// Warp roles (512 threads):
//   warp 0      TMEM allocation; lane 0 issues every MMA
//   warps 4-7   softmax (TMEM lanes = tile rows) and epilogue
//   warps 8-15  gather + unpack: each thread owns 4 rows x one 8-dim slice
//               per 64-dim chunk; a whole tile's raw bytes are requested
//               before the tile's shared-memory chunks are released, so the
//               gather latency hides behind the previous tile's MMAs.
// Chunk-granular mbarriers let the unpack of tile i+1 overwrite a 64-dim
// chunk as soon as the output MMAs of tile i no longer need it.
//
// Online softmax in base 2 with a lazily updated reference max: a head's
// reference moves (and O^T and the partial sums are rescaled) only when a
// score exceeds it by more than 8, so P = 2^(s - m) <= 256 fits FP16.
//
// Splits (several CTAs per token) write normalized FP32 partials plus
// (m, l) to the workspace and a small combine kernel merges them.
#include <cuda_runtime.h>

#include <cmath>

#include "common.cuh"
#include "decode_common.cuh"
#include "kernels.h"
#include "ptx.cuh"

namespace nvfp4mla {
using namespace ptx;
#ifdef NVFP4MLA_TRACE
void set_trace_buffer(unsigned long long *p) { set_trace_local(p); }
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
constexpr int kNumBars = 16;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 64;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kMaxHG * kLatent * 4 <= kTileBytes, "FP32 output staging must fit in the tile region");
constexpr int kThreads = 512;

constexpr int BAR_CHUNK_FULL = 0;  // [9] unpack -> MMA, count 8 warps
constexpr int BAR_CHUNK_FREE = 9;  // [4] output MMAs of a 128-dv block done
constexpr int BAR_S_FULL = 13;     // score MMAs of a tile done
constexpr int BAR_P_FULL = 14;     // P^T written (4 softmax warps)
constexpr int BAR_DRAIN = 15;      // every MMA issued so far done

constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;      // O^T: 4 blocks of HG columns
constexpr uint32_t kColS = 256;    // S^T: HG columns
constexpr float kRescaleThreshold = 8.0f;
}  // namespace dec

template <int HG, bool kStaged>
__global__ void __launch_bounds__(dec::kThreads, 1) sparse_mla_decode_kernel(const DecodeArgs a) {
    using namespace dec;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
#ifdef NVFP4MLA_TRACE
    const unsigned long long t_start = clock64();
#endif
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
        else if (lane == BAR_P_FULL) count = 4;         // 4 softmax warps
        else if (lane == BAR_DRAIN) count = 1;
        if (count) mbar_init(&bars[lane], count);
        fence_mbar_init();
    }
    if (warp == 3) {  // a warp with no setup work: the allocation can take a while
        tmem_alloc(&misc[0], kTmemCols);
        tmem_relinquish();
    }
    if (tid < HG) m_s[tid] = -INFINITY;

    // Q of (t, heads g*HG ..) -> shared memory, K-major, 128-byte swizzle:
    // chunk c holds dims 64c..64c+63 of every head (chunk 8 = RoPE).
    // Issued as 16-byte async copies so every load of the CTA is in flight
    // at once; they complete before the setup barrier below.
    if (warp >= 8) {
        const int ut = tid - 256;
        const int64_t head0 = (int64_t)t * a.H + (int64_t)g * HG;
        for (int u = ut; u < HG * 72; u += 256) {
            const int h = u / 72, v = u % 72;
            const void *src = v < 64 ? static_cast<const void *>(a.q_nope + (head0 + h) * kLatent + 8 * v)
                                     : static_cast<const void *>(a.q_rope + (head0 + h) * kRope + 8 * (v - 64));
            cp_async16(smem + kOffQ + (v >> 3) * (HG * 128) + sw128_offset(h, v & 7), src);
        }
    }

    // Compact the token's list: keep valid entries in list order; this CTA
    // keeps entries [lo, hi) of the compacted order.
    const int32_t *lst = a.indices + (int64_t)t * a.topk;
    int32_t vals[4];
    uint32_t bal[4];
    bool bad = false;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int p = tid + 512 * k;
        const int32_t v = p < a.topk ? __ldg(lst + p) : -1;
        const bool ok = v >= 0 && (int64_t)v < a.num_slots;
        bad |= (p < a.topk) && (v < -1 || (int64_t)v >= a.num_slots);
        vals[k] = v;
        bal[k] = __ballot_sync(0xffffffffu, ok);
        if (lane == 0) cnt_s[k * 16 + warp] = __popc(bal[k]);
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0 && split == 0 && g == 0 && a.dev_status)
        atomicOr(a.dev_status, NVFP4MLA_DEV_BAD_INDEX);
    __syncthreads();
    // exclusive prefix of the 64 per-(round, warp) counts: warp 0 scans them
    // (2 per lane), everyone reads its 4 offsets and the total back
    uint32_t *pre_s = cnt_s + 64;
    if (warp == 0) {
        const uint32_t c0 = cnt_s[2 * lane], c1 = cnt_s[2 * lane + 1];
        uint32_t incl = c0 + c1;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const uint32_t excl = incl - c0 - c1;
        pre_s[2 * lane] = excl;
        pre_s[2 * lane + 1] = excl + c0;
        if (lane == 31) pre_s[64] = incl;
    }
    __syncthreads();
    int before[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) before[k] = (int)pre_s[k * 16 + warp];
    const int n_valid = (int)pre_s[64];
    const int per = (n_valid + a.S - 1) / a.S;
    const int lo = split * per;
    const int hi = min(n_valid, lo + per);
    const int n_mine = max(0, hi - lo);
    const int ntiles = (n_mine + kTileRows - 1) / kTileRows;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if ((bal[k] >> lane) & 1u) {
            const int pos = before[k] + __popc(bal[k] & ((1u << lane) - 1u));
            if (pos >= lo && pos < hi) idx_s[pos - lo] = kStaged ? (tid + 512 * k) : vals[k];
        }
    }
    if (warp >= 8) {
        cp_async_wait_all();
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = misc[0];
    if (tid == 0) TRACE(0);

    // Register budget (launched with 128 x 512): the MMA/idle warpgroup gives
    // registers to the softmax and unpack warps, 128 x 48 + 128 x 144 +
    // 256 x 160 = 65536.  Each role changes its budget inside its own branch
    // so the compiler sizes each role's code separately.
    if (warp < 4) {
        regs_dec<48>();
        // ------------------------------------------------------------- MMA
        if (warp == 0 && lane == 0) {
            const uint32_t idesc_qk = idesc_f16_f32(128, HG, false, false);
            const uint32_t idesc_pv = idesc_f16_f32(128, HG, true, true);
            const uint64_t dK0 = smem_desc(smem_u32(smem), 16, 1024);
            const uint64_t dQ0 = smem_desc(smem_u32(smem + kOffQ), 16, 1024);
            const uint64_t dV0 = smem_desc(smem_u32(smem), kChunkBytes, 1024);
            const uint64_t dP0 = smem_desc(smem_u32(smem + 8 * kChunkBytes), kChunkBytes, 1024);
            bool ok = true;
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
    } else if (warp < 8) {
        // --------------------------------------------------------- softmax
        regs_inc<144>();
        // Heads are processed in halves of HW = min(HG, 32): the reference
        // max, rescale and row sums of a head never depend on other heads.
        constexpr int HW = HG < 32 ? HG : 32;
        constexpr int NH = HG / HW;
        const int st = tid - 128;  // tile row == TMEM lane
        const int wq = st >> 5;
        const uint32_t lane_base = (uint32_t)(32 * wq) << 16;
        uint8_t *p_tile = smem + 8 * kChunkBytes;  // P^T overwrites the RoPE chunk
        float lp[NH];  // warp-partial row sums, column h0 + transposed_col<HW>(lane)
#pragma unroll
        for (int j = 0; j < NH; ++j) lp[j] = 0.0f;
        bool ok = true;
        for (int i = 0; i < ntiles; ++i) {
            // S_FULL(i) also covers PV(i-1): the MMA thread issued it earlier,
            // so O^T is quiescent and may be rescaled here.
            if (!mbar_wait(&bars[BAR_S_FULL], i & 1)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (st == 0 && i < 8) TRACE(4 + 6 * i);
            uint32_t rs[HG];
            tmem_ld_cols<HG>(tmem + lane_base + kColS, rs);
            tmem_ld_wait();
            const int nrows = min(kTileRows, n_mine - kTileRows * i);
            const bool valid = st < nrows;
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) {
                const int h0 = hh * HW;
                float sv[HW];
#pragma unroll
                for (int h = 0; h < HW; ++h) sv[h] = __uint_as_float(rs[h0 + h]) * a.scale_log2;
                bool need = false;
                if (valid) {
#pragma unroll
                    for (int h = 0; h < HW; ++h) need |= sv[h] > m_s[h0 + h] + kRescaleThreshold;
                }
                if (sm_bar_or(need)) {
                    {
                        float mx[HW];
#pragma unroll
                        for (int h = 0; h < HW; ++h) mx[h] = valid ? sv[h] : -INFINITY;
                        warp_transpose_reduce<HW, true>(mx, lane);
                        red_s[wq * 64 + h0 + transposed_col<HW>(lane, 0)] = mx[0];
                    }
                    sm_bar();
                    if (st < HW) {
                        const int h = h0 + st;
                        const float old = m_s[h];
                        float nm = old;
#pragma unroll
                        for (int w = 0; w < 4; ++w) nm = fmaxf(nm, red_s[w * 64 + h]);
                        aux_s[h] = (old == -INFINITY) ? 0.0f : ex2(old - nm);
                        m_s[h] = nm;
                    }
                    sm_bar();
                    lp[hh] *= aux_s[h0 + transposed_col<HW>(lane, 0)];
                    if (i > 0) {
#pragma unroll 1
                        for (int dc = 0; dc < 4; ++dc) {
                            uint32_t r[HW];
                            const uint32_t addr = tmem + lane_base + kColO + dc * HG + h0;
                            tmem_ld_cols<HW>(addr, r);
                            tmem_ld_wait();
#pragma unroll
                            for (int h = 0; h < HW; ++h) r[h] = __float_as_uint(__uint_as_float(r[h]) * aux_s[h0 + h]);
#pragma unroll
                            for (int cb = 0; cb < HW; cb += 16) {
                                uint32_t q[16];
#pragma unroll
                                for (int j = 0; j < 16; ++j) q[j] = r[cb + j];
                                tmem_st16(addr + cb, q);
                            }
                        }
                        tmem_st_wait();
                    }
                }
#pragma unroll
                for (int h = 0; h < HW; ++h) sv[h] = valid ? ex2(sv[h] - m_s[h0 + h]) : 0.0f;
#pragma unroll
                for (int j = 0; j < HW / 8; ++j) {
                    uint4 pk;
                    pk.x = pack_half2(sv[8 * j + 0], sv[8 * j + 1]);
                    pk.y = pack_half2(sv[8 * j + 2], sv[8 * j + 3]);
                    pk.z = pack_half2(sv[8 * j + 4], sv[8 * j + 5]);
                    pk.w = pack_half2(sv[8 * j + 6], sv[8 * j + 7]);
                    *reinterpret_cast<uint4 *>(p_tile + sw128_offset(st, h0 / 8 + j)) = pk;
                }
                warp_transpose_reduce<HW, false>(sv, lane);
                lp[hh] += sv[0];
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[BAR_P_FULL]);
            if (st == 0 && i < 8) TRACE(5 + 6 * i);
        }
        if (!ok && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
        // ---------------------------------------------------------- epilogue
        if (ok && ntiles > 0) {
            if (!mbar_wait(&bars[BAR_CHUNK_FREE + 3], (ntiles - 1) & 1)) {
                ok = false;
                if (a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_TIMEOUT);
            }
            tc_fence_after();
        }
        const bool have = ok && ntiles > 0;
        if (!(HW < 32 && (lane & 1))) {
#pragma unroll
            for (int hh = 0; hh < NH; ++hh) red_s[wq * 64 + hh * HW + transposed_col<HW>(lane, 0)] = lp[hh];
        }
        sm_bar();
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
        sm_bar();
        // O^T (TMEM, lanes = dv) -> normalized rows staged in the (now free)
        // tile region, then bulk copies to global memory.
        //  one split:   out[t, g*HG + h, :] (FP16), one copy of HG x 1 KB;
        //  split parts: ws_o[t, split, dc, g*HG + h, 0:128] (FP32, dv block
        //               major), one 32 KB copy per 128-dv block, issued as soon
        //               as the block is staged.
        float inv_l[HG];
#pragma unroll
        for (int h = 0; h < HG; ++h) inv_l[h] = aux_s[h];
        uint8_t *stage = smem;
        if (a.S == 1) {
#pragma unroll 1
            for (int dc = 0; dc < 4; ++dc) {
                const int dv = 128 * dc + st;
                uint32_t r[HG];
                if (have) {
                    tmem_ld_cols<HG>(tmem + lane_base + kColO + dc * HG, r);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int h = 0; h < HG; ++h) r[h] = 0u;
                }
#pragma unroll
                for (int h = 0; h < HG; ++h)
                    reinterpret_cast<__half *>(stage)[h * kLatent + dv] = __float2half_rn(__uint_as_float(r[h]) * inv_l[h]);
            }
            fence_proxy_async_smem();
            sm_bar();
            if (st == 0) {
                bulk_s2g(a.out + ((int64_t)t * a.H + (int64_t)g * HG) * kLatent, stage, HG * kLatent * 2);
                bulk_commit_wait_read();
            }
        } else {
#pragma unroll 1
            for (int dc = 0; dc < 4; ++dc) {
                float *blk = reinterpret_cast<float *>(stage + dc * (HG * 128 * 4));
                uint32_t r[HG];
                if (have) {
                    tmem_ld_cols<HG>(tmem + lane_base + kColO + dc * HG, r);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int h = 0; h < HG; ++h) r[h] = 0u;
                }
#pragma unroll
                for (int h = 0; h < HG; ++h) blk[h * 128 + st] = __uint_as_float(r[h]) * inv_l[h];
                fence_proxy_async_smem();
                sm_bar();
                if (st == 0)
                    bulk_s2g(a.ws_o + ((((int64_t)t * a.S + split) * 4 + dc) * a.H + (int64_t)g * HG) * 128, blk,
                             HG * 128 * 4);
            }
            if (st == 0) bulk_commit_wait_read();
        }
        if (st == 0) TRACE(61);
    } else {
        // ---------------------------------------------------- gather + unpack
        regs_inc<160>();
        const int ut = tid - 256;
        const int sub = ut & 7;   // 8-dim slice of every 64-dim chunk
        const int rg = ut >> 3;   // rows rg, rg+32, rg+64, rg+96 of each tile
        const uint8_t *row_ptr[4];
        bool rvalid[4];
        constexpr int kWords = kStaged ? 18 : 11;  // raw 32-bit words per row held per tile
        uint32_t raw[4][kWords];
        auto load_tile = [&](int i) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int e = kTileRows * i + rg + 32 * k;
                rvalid[k] = e < n_mine;
                const int32_t v = rvalid[k] ? idx_s[e] : 0;
                if (kStaged)
                    row_ptr[k] = a.src + ((int64_t)t * a.topk + v) * kStagedRowBytes;
                else
                    row_ptr[k] = a.src + (int64_t)v * kRowBytes;
                if (rvalid[k]) {
                    if (kStaged) {
#pragma unroll
                        for (int c = 0; c < kChunks; ++c) {
                            const uint2 w2 = ldg64(row_ptr[k] + 64 * c + 8 * sub);
                            raw[k][2 * c] = w2.x;
                            raw[k][2 * c + 1] = w2.y;
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < 8; ++c) raw[k][c] = ldg32(row_ptr[k] + 32 * c + 4 * sub);
                        raw[k][8] = ldg32(row_ptr[k] + kScaleOff + 4 * sub);
                        const uint2 rp = ldg64(row_ptr[k] + kRopeOff + 8 * sub);
                        raw[k][9] = rp.x;
                        raw[k][10] = rp.y;
                    }
                } else {
#pragma unroll
                    for (int w = 0; w < kWords; ++w) raw[k][w] = 0u;
                }
            }
        };
        bool ok = true;
        if (ntiles > 0) load_tile(0);
        for (int i = 0; i < ntiles && ok; ++i) {
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                if (i > 0 && !mbar_wait(&bars[BAR_CHUNK_FREE + (c < 8 ? (c >> 1) : 3)], (i - 1) & 1)) {
                    ok = false;
                    break;
                }
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
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[BAR_CHUNK_FULL + c]);
            }
            if (ut == 0 && i < 8) TRACE(6 + 6 * i);
            if (ok && i + 1 < ntiles) load_tile(i + 1);
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
}

// Merge split partials: out = sum_s w_s o_s / sum_s w_s with
// w_s = l_s 2^(m_s - max m), lse = (max m + log2 sum w) ln 2.  One block per
// (token, head); every load is issued before any of them is used.
template <int S>
__global__ void __launch_bounds__(128) combine_splits_kernel(const float *__restrict__ ws_o,
                                                             const float *__restrict__ ws_ml, int H,
                                                             __half *__restrict__ out, float *__restrict__ lse) {
    const int th = blockIdx.x;  // t*H + h
    const int t = th / H, h = th % H;
    float m[S], l[S];
    float4 o[S];
#pragma unroll
    for (int s = 0; s < S; ++s) {
        const int64_t prow = ((int64_t)t * S + s) * H + h;
        const float2 ml = *reinterpret_cast<const float2 *>(ws_ml + 2 * prow);
        m[s] = ml.x;
        l[s] = ml.y;
        // partial rows are stored per 128-dv block: [t][s][dc][h][128]
        const int dc = threadIdx.x >> 5, d = 4 * (threadIdx.x & 31);
        o[s] = *reinterpret_cast<const float4 *>(ws_o + ((((int64_t)t * S + s) * 4 + dc) * H + h) * 128 + d);
    }
    float mmax = -INFINITY;
#pragma unroll
    for (int s = 0; s < S; ++s)
        if (l[s] > 0.0f) mmax = fmaxf(mmax, m[s]);
    float L = 0.0f, acc0 = 0.0f, acc1 = 0.0f, acc2 = 0.0f, acc3 = 0.0f;
#pragma unroll
    for (int s = 0; s < S; ++s) {
        const float w = l[s] > 0.0f ? l[s] * ex2(m[s] - mmax) : 0.0f;
        L += w;
        acc0 += w * o[s].x;
        acc1 += w * o[s].y;
        acc2 += w * o[s].z;
        acc3 += w * o[s].w;
    }
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    __half2 *dst = reinterpret_cast<__half2 *>(out + (int64_t)th * kLatent + 4 * threadIdx.x);
    dst[0] = __floats2half2_rn(acc0 * inv, acc1 * inv);
    dst[1] = __floats2half2_rn(acc2 * inv, acc3 * inv);
    if (threadIdx.x == 0) lse[th] = L > 0.0f ? (mmax + lg2(L)) * 0.69314718055994531f : -INFINITY;
}

bool make_decode_plan(int32_t T, int32_t H, int32_t topk, DecodePlan *plan) {
    DecodePlan p{};
    if (H == 16 || H == 32 || H == 64) {
        p.heads_per_cta = H;
        p.head_groups = 1;
    } else if (H == 128) {
        p.heads_per_cta = 64;
        p.head_groups = 2;
    } else {
        return false;
    }
    if (topk < 1 || topk > kMaxTopk || T < 0) return false;
    const int64_t units = (int64_t)T * p.head_groups;
    const int max_s = std::min(16, (topk + dec::kTileRows - 1) / dec::kTileRows);
    int S = 1;
    while (S * 2 <= max_s && units * S * 2 <= 148) S *= 2;
    p.splits = S;
    p.workspace_bytes = S > 1 ? (size_t)T * S * H * (kLatent + 2) * sizeof(float) : 0;
    *plan = p;
    return true;
}

template <int HG, bool kStaged>
static cudaError_t launch_hg(const DecodeArgs &a, int64_t nblocks, cudaStream_t stream) {
    auto kern = sparse_mla_decode_kernel<HG, kStaged>;
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, dec::kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    kern<<<(unsigned)nblocks, dec::kThreads, dec::kSmemBytes, stream>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_sparse_mla_decode(bool staged, const void *q_nope, const void *q_rope, const uint8_t *src,
                                     int64_t num_slots, const int32_t *indices, int32_t topk, int32_t T,
                                     int32_t H, float sm_scale, void *out, float *lse, void *workspace,
                                     const DecodePlan &plan, int32_t *dev_status, cudaStream_t stream) {
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
    a.ws_o = static_cast<float *>(workspace);
    a.ws_ml = a.ws_o ? a.ws_o + (size_t)T * plan.splits * H * kLatent : nullptr;
    a.dev_status = dev_status;
    const int64_t nblocks = (int64_t)T * plan.head_groups * plan.splits;
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
    if (e != cudaSuccess || plan.splits == 1) return e;
    const unsigned cblocks = (unsigned)((int64_t)T * H);
    switch (plan.splits) {
        case 2: combine_splits_kernel<2><<<cblocks, 128, 0, stream>>>(a.ws_o, a.ws_ml, H, a.out, a.lse); break;
        case 4: combine_splits_kernel<4><<<cblocks, 128, 0, stream>>>(a.ws_o, a.ws_ml, H, a.out, a.lse); break;
        case 8: combine_splits_kernel<8><<<cblocks, 128, 0, stream>>>(a.ws_o, a.ws_ml, H, a.out, a.lse); break;
        case 16: combine_splits_kernel<16><<<cblocks, 128, 0, stream>>>(a.ws_o, a.ws_ml, H, a.out, a.lse); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

}  // namespace nvfp4mla
