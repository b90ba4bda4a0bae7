// kernels.h -- internal launchers of libnvfp4mla (host side, no checks:
// the C ABI in api.cu validates arguments before calling these).
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4mla {

cudaError_t launch_kv_append(const void *latent, int64_t latent_stride, const void *rope, int64_t rope_stride,
                             const int32_t *slot_mapping, int32_t n, uint8_t *cache, int64_t num_slots,
                             int32_t *dev_status, cudaStream_t stream);

// Work decomposition of one decode launch.
struct DecodePlan {
    int heads_per_cta;  // HG: heads handled by one CTA (N of the MMAs)
    int head_groups;    // G = H / HG
    int splits;         // S: CTAs sharing one token's list
    size_t workspace_bytes;
};
// Split launches keep one (arrivals, departures) pair of uint32 counters per
// (token, head group) at the start of the workspace; splitting needs
// T * G * S <= SMs, so a fixed 4 KB region (512 pairs) always suffices and
// sits at the same place for every shape.
constexpr size_t kSplitCounterBytes = 4096;
// sm_count: SMs of the device the launch will run on (one CTA per SM).
// splits / heads_per_cta: 0 picks them automatically; other values fix them
// (false when the shape cannot take them).
bool make_decode_plan(int32_t T, int32_t H, int32_t topk, int sm_count, DecodePlan *plan, int splits = 0,
                      int heads_per_cta = 0);
// SM count of the current device, or 148 when no device can be queried
// (pure host use, e.g. sizing a workspace on a machine without a GPU).
int current_device_sm_count();

cudaError_t launch_fp8_kv_append(const void *latent, int64_t latent_stride, const void *rope, int64_t rope_stride,
                                 const int32_t *slot_mapping, int32_t n, uint8_t *cache, int64_t num_slots,
                                 int32_t *dev_status, cudaStream_t stream);

struct DecodeTestHooks;  // test-only launch settings (decode_common.cuh)

// What the decode's `src` holds.
enum class RowSource {
    kNvfp4Cache,  // num_slots 352-byte NVFP4 rows; list entries are slots
    kFp8Staging,  // [T, topk] 576-byte E4M3 rows addressed by list position;
                  // entries outside [0, num_slots) are still the empty ones
    kFp8Cache,    // num_slots 576-byte E4M3 rows; list entries are slots
};

// Sparse MLA decode over `src` (see RowSource).  block_table (optional):
// list entries are then request-local positions, translated through
// table[t][pos >> page_shift] (table_stride entries per token) while the
// list is compacted.
cudaError_t launch_sparse_mla_decode(RowSource rows, const void *q_nope, const void *q_rope, const uint8_t *src,
                                     int64_t num_slots, const int32_t *indices, int32_t topk, int32_t T,
                                     int32_t H, float sm_scale, void *out, float *lse, void *workspace,
                                     const DecodePlan &plan, int32_t *dev_status, cudaStream_t stream,
                                     const int32_t *block_table = nullptr, int64_t table_stride = 0,
                                     int page_shift = 0, const DecodeTestHooks *hooks = nullptr);

cudaError_t launch_stage_fp8(const uint8_t *cache, int64_t num_slots, const int32_t *indices, int32_t topk,
                             int32_t T, uint8_t *staging, cudaStream_t stream);

// Sparse indexer (indexer.cu).  page_shift = log2(page size) >= 3.
int64_t indexer_score_stride(int32_t max_ctx);
cudaError_t launch_indexer_scores(const uint8_t *q, const float *w, const uint8_t *keys, int64_t num_slots,
                                  const int32_t *table, int64_t table_stride, int page_shift,
                                  const int32_t *ctx_lens, int32_t max_ctx, int32_t T, float *scores,
                                  int64_t score_stride, int32_t *dev_status, cudaStream_t stream);
// Selection splits each request's row over indexer_topk_parts(T) CTAs; more
// than one needs indexer_topk_workspace_bytes of workspace whose first T
// words are zero (every completed launch leaves them so).
int indexer_topk_parts(int32_t T, int sm_count);
size_t indexer_topk_workspace_bytes(int32_t T, int sm_count);
cudaError_t launch_indexer_topk(const float *scores, int64_t score_stride, const int32_t *ctx_lens, int32_t max_ctx,
                                int32_t T, int32_t topk, int32_t *positions, void *workspace, int32_t *dev_status,
                                cudaStream_t stream);

// Per-layer paged caches <-> block-major multi-layer cache (blhnc.cu).
cudaError_t launch_blhnc_convert(const uint64_t *layer_ptrs, int32_t layers, int64_t num_blocks, int32_t block_size,
                                 int32_t row_bytes, int32_t sub, const int32_t *block_ids, const int32_t *new_ids,
                                 int32_t nb, uint8_t *blhnc, int64_t num_new, bool to_blhnc, int32_t *dev_status,
                                 cudaStream_t stream);

// Bounded-wait self-test: a single CTA whose two waits run out (~1 ms each);
// `counter` must point at a zero uint32 in device memory.
cudaError_t launch_wait_timeout_selftest(uint32_t *counter, int32_t *dev_status, cudaStream_t stream);

}  // namespace nvfp4mla
