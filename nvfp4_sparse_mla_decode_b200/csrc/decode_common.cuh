// decode_common.cuh -- pieces shared by the decode kernels: launch
// arguments, base-2 exp/log instructions, softmax-warp barriers, the in-warp
// transpose reduction and debug-only tracing.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>

#include "common.cuh"
#include "ptx.cuh"

namespace nvfp4mla {

struct DecodeArgs {
    const __half *q_nope;
    const __half *q_rope;
    const uint8_t *src;
    int64_t num_slots;
    const int32_t *indices;
    int topk, T, H, G, S;
    float scale_log2;
    __half *out;
    float *lse;
    float *ws_o;        // split partials, unnormalised FP32: [T][S][H][512] (FP8-row kernel) or
                        // [T][G][S][HG/4][512][4] (NVFP4 kernel: 4-head pieces, dv-major)
    float *ws_ml;       // split statistics: [T][S][H] x (max in log2 units, row sum)
    uint32_t *counters; // per (token, head group): arrivals, departures
    int32_t *dev_status;
    // Optional block table: when set, list entries are request-local token
    // positions and slot = table[t][pos >> page_shift] << page_shift | low bits.
    const int32_t *block_table;
    int64_t table_stride;  // entries per token row of the table
    int page_shift;        // log2 of the page size
    int64_t max_pos;       // table_stride << page_shift
    // FP8 (576-byte) rows only: true when `src` is a cache of rows addressed
    // by slot, false when it is the staging buffer [T][topk] addressed by
    // list position.
    bool rows_by_slot;
    // NVFP4 kernel: SM clock cycles after which any one wait gives up
    // (about a second by default), and a test hook that withholds one
    // arrival so that tests can drive the timeout paths (0 in every
    // product call; see DecodeTestHooks).
    unsigned long long wait_cycles;
    int test_withhold;
};

// Test-only settings for a decode launch (never set by the public API):
// withhold = 1: the softmax warps never publish P^T, so the output MMAs'
// wait runs out and every role that depends on it follows;
// withhold = 2: split 0 of each group never arrives on the merge counter, so
// the group's merge wait runs out and poisons the counter.
struct DecodeTestHooks {
    unsigned long long wait_cycles;
    int withhold;
};

#ifdef NVFP4MLA_TRACE
// Debug builds only: per-CTA phase timestamps (clock64 deltas) for the
// first 16 CTAs, 512 slots each.
// TRACE_SETUP() reads the buffer pointer once, so a stamp is a clock read
// and a store, not a global load after every wait.
static __device__ unsigned long long *g_trace;
#define TRACE_SETUP() unsigned long long *const trace_buf_ = blockIdx.x < 16 && g_trace ? g_trace + blockIdx.x * 512 : nullptr
#define TRACE(slot)                                                   \
    do {                                                              \
        if (trace_buf_) trace_buf_[(slot)] = clock64() - t_start;     \
    } while (0)
static inline void set_trace_local(unsigned long long *p) { cudaMemcpyToSymbol(g_trace, &p, sizeof(p)); }
// Every CTA: [start ns, end ns, SM id] from the global timer (comparable
// across SMs, unlike clock64).
static __device__ unsigned long long *g_trace_all;
static inline void set_trace_all_local(unsigned long long *p) { cudaMemcpyToSymbol(g_trace_all, &p, sizeof(p)); }
__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ unsigned sm_id() {
    unsigned r;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(r));
    return r;
}
#else
#define TRACE_SETUP() \
    do {              \
    } while (0)
#define TRACE(slot) \
    do {            \
    } while (0)
#endif

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float lg2(float x) {
    float y;
    asm("lg2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// Named barrier 1 over the 128 softmax threads, optionally OR-reducing a flag.
// Named barrier `id` over `n` threads, optionally OR-reducing a flag.
__device__ __forceinline__ void named_bar(uint32_t id, uint32_t n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
__device__ __forceinline__ bool named_bar_or(uint32_t id, uint32_t n, bool p) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\tsetp.ne.u32 pi, %3, 0;\n\tbar.red.or.pred po, %1, %2, pi;\n\tselp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"(id), "r"(n), "r"((uint32_t)p)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ uint32_t ldg32(const uint8_t *p) {
    return __ldg(reinterpret_cast<const unsigned int *>(p));
}
__device__ __forceinline__ uint2 ldg64(const uint8_t *p) { return __ldg(reinterpret_cast<const uint2 *>(p)); }

// In-warp transpose reduction: on entry each lane holds W column values; on
// exit lane l holds op-reduced columns [l*W/32, (l+1)*W/32) in v[0..W/32)
// (W == 16: column l/2 in v[0], duplicated in lane pairs).
template <int W, bool kMax>
__device__ __forceinline__ void warp_transpose_reduce(float (&v)[W], int lane) {
#pragma unroll
    for (int o = 16, w = W; o >= 1 && w >= 2; o >>= 1, w >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int j = 0; j < w / 2; ++j) {
            const float keep = upper ? v[j + w / 2] : v[j];
            const float send = upper ? v[j] : v[j + w / 2];
            const float got = __shfl_xor_sync(0xffffffffu, send, o);
            v[j] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
    if (W == 16) {
        const float got = __shfl_xor_sync(0xffffffffu, v[0], 1);
        v[0] = kMax ? fmaxf(v[0], got) : v[0] + got;
    }
}
template <int W>
__device__ __forceinline__ int transposed_col(int lane, int j) {
    return W >= 32 ? lane * (W / 32) + j : lane >> 1;
}
__host__ __device__ constexpr int cols_per_lane(int W) { return W >= 32 ? W / 32 : 1; }


// Tensor map for Q: a 2-D FP16 view [rows = T*H, cols] of q_nope (cols 512)
// or q_rope (cols 64), box 64 cols x box_rows rows, 128-byte swizzle; encoded
// maps are cached per host thread, keyed by (address, rows, cols, box rows).
bool make_q_map(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows);
// Tensor map over the NVFP4 kernel's split exchange area: FP32 rows of 2048
// (512 dv x 4 heads), box box_x floats x box_rows rows, no swizzle.
bool make_xch_map(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_x, uint32_t box_rows);
// Launch of the pipelined NVFP4 decode kernel (decode_nvfp4.cu).
cudaError_t launch_nvfp4_decode(const DecodeArgs &a, int heads_per_cta, int64_t nblocks, cudaStream_t stream);

// N consecutive TMEM columns (32 lanes x 32 bit) in one instruction.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
    if constexpr (N == 64) ptx::tmem_ld64(taddr, r);
    else if constexpr (N == 32) ptx::tmem_ld32(taddr, r);
    else ptx::tmem_ld16(taddr, r);
}

}  // namespace nvfp4mla
