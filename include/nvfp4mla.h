/*
 * nvfp4mla.h -- C ABI of libnvfp4mla: sparse multi-head-latent-attention
 * (MLA) decode over a KV cache stored as NVFP4, for NVIDIA B200 (sm_100a).
 *
 * What the library computes follows page "Prime Intellect Launches Prime
 * Inference, Serving 600B Tokens Daily", section "Four-bit caches make room":
 * the MLA latent cache is compressed with NVFP4 (4-bit values, one FP8 scale
 * per group of 16), shrinking each row from 576 to 352 bytes; a native
 * sparse-attention kernel loads only the rows picked by the sparse indexer,
 * unpacks them on chip and runs attention with FP16 operands and FP32
 * accumulation; the index list has 2,048 positions and its empty entries
 * are zero-filled; a staged implementation that first unpacks NVFP4 into FP8
 * buffers in GPU memory is the comparison path.
 *
 * Row layout (352 bytes, the pages fix only the size and the grouping):
 *   [0,256)   latent dims 0..511 as E2M1 nibbles; byte b = dim 2b (low
 *             nibble) | dim 2b+1 (high nibble)
 *   [256,288) 32 E4M3 scales; scale g covers latent dims 16g..16g+15
 *   [288,352) 64 RoPE dims as E4M3, byte k = RoPE dim k
 * Latent dim d dequantizes to e2m1(nibble) * e4m3(scale[d/16]); RoPE dim k
 * to e4m3(byte k).  Both values are exact in FP16.
 *
 * Conventions for every call:
 *   - all data pointers are DEVICE pointers; the caller owns every buffer;
 *     the library allocates no device memory and keeps no global state;
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream); work is enqueued asynchronously on it;
 *   - arguments the host can check are checked before anything is enqueued;
 *     on error the call returns a non-OK status and launches nothing;
 *   - problems only the device can see (an index or slot out of range, a
 *     bounded wait that ran out) are OR-ed as status bits into *dev_status
 *     when dev_status is not NULL; read it after synchronizing the stream;
 *   - calls on different streams are independent; concurrent calls that
 *     write the same output or workspace race.
 */
#ifndef NVFP4MLA_H
#define NVFP4MLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define NVFP4MLA_ROW_BYTES 352        /* 256 nibble bytes + 32 scales + 64 RoPE */
#define NVFP4MLA_STAGED_ROW_BYTES 576 /* staged FP8 row: 512 latent + 64 RoPE */
#define NVFP4MLA_LATENT 512
#define NVFP4MLA_ROPE 64
#define NVFP4MLA_GROUP 16
#define NVFP4MLA_MAX_TOPK 2048        /* positions of one index list */
#define NVFP4MLA_MAX_HEADS 128
#define NVFP4MLA_INDEX_HEADS 64       /* sparse indexer heads */
#define NVFP4MLA_INDEX_DIM 128        /* dims (= E4M3 bytes) of an indexer key or query head */

typedef enum {
    NVFP4MLA_OK = 0,
    NVFP4MLA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size */
    NVFP4MLA_ERR_UNSUPPORTED = 2, /* shape outside what the kernels cover */
    NVFP4MLA_ERR_WORKSPACE = 3,   /* workspace/staging buffer too small */
    NVFP4MLA_ERR_CUDA = 4,        /* a CUDA runtime call failed */
    NVFP4MLA_ERR_TIMEOUT = 5,     /* device: a bounded wait ran out */
    NVFP4MLA_ERR_BAD_INDEX = 6    /* device: index/slot outside [0,num_slots) */
} nvfp4mla_status;

/* Device status bits OR-ed into *dev_status (int32). */
#define NVFP4MLA_DEV_TIMEOUT 1   /* a bounded wait ran out; results invalid */
#define NVFP4MLA_DEV_BAD_INDEX 2 /* an index/slot outside [-1, num_slots) */
#define NVFP4MLA_DEV_LAYOUT 4    /* shared memory base not 1 KB aligned */

/*
 * nvfp4_kv_append -- quantize n BF16 cache rows into NVFP4 rows at scattered
 * slots (page "Prime Intellect Launches Prime Inference, Serving 600B Tokens
 * Daily", section "Four-bit caches make room": 4-bit values with an FP8
 * scale shared by every 16 of them, 352-byte rows).
 *
 *   latent_bf16   [n, latent_stride] BF16, first 512 elements of a row used;
 *                 16-byte aligned, latent_stride % 8 == 0
 *   rope_bf16     [n, rope_stride] BF16, first 64 used; 16-byte aligned,
 *                 rope_stride % 8 == 0
 *   slot_mapping  [n] int32: row i goes to cache slot slot_mapping[i];
 *                 a negative slot skips the row; a slot >= num_slots skips
 *                 it and sets NVFP4MLA_DEV_BAD_INDEX
 *   cache         [num_slots, 352] bytes, 16-byte aligned
 * Per group of 16 latent values: a = max|x|, scale = E4M3 round-to-nearest-
 * even, saturating, of a/6 (FP32 division); each value becomes the E2M1
 * round-to-nearest-even, saturating, of x/scale (FP32 division), or +0 when
 * the scale is 0.  RoPE values are E4M3-rounded the same way, unscaled.
 * n == 0 is a no-op.  Returns INVALID_ARG for null pointers (when n > 0),
 * misalignment or negative sizes.
 */
nvfp4mla_status nvfp4_kv_append(const void *latent_bf16, int64_t latent_stride, const void *rope_bf16,
                                int64_t rope_stride, const int32_t *slot_mapping, int32_t n, uint8_t *cache,
                                int64_t num_slots, int32_t *dev_status, void *stream);

/*
 * nvfp4mla_fp8_kv_append -- the pre-NVFP4 cache row (same page and section:
 * a row took 576 bytes before the four-bit format): write n BF16 cache rows
 * as 576-byte E4M3 rows at scattered slots.  Bytes [0, 512) of a row are
 * the latent dims, [512, 576) the RoPE dims, each the E4M3 round-to-nearest-
 * even, saturating (to +-448), of the value, with no scale.
 *   latent_bf16, rope_bf16, slot_mapping, n, dev_status, stream: as
 *                 nvfp4_kv_append
 *   cache         [num_slots, 576] bytes, 16-byte aligned
 * Same error behaviour as nvfp4_kv_append.
 */
nvfp4mla_status nvfp4mla_fp8_kv_append(const void *latent_bf16, int64_t latent_stride, const void *rope_bf16,
                                       int64_t rope_stride, const int32_t *slot_mapping, int32_t n, uint8_t *cache,
                                       int64_t num_slots, int32_t *dev_status, void *stream);

/*
 * nvfp4_sparse_mla_num_splits -- how many CTAs the decode splits each
 * token's index list across: the largest power of two S <= 16 (and <= the
 * number of 128-row tiles of topk) with T * G * S no larger than the SM
 * count of the current device (148 when no device can be queried), where
 * G = H / HG head groups of HG heads each: HG = min(H, 64), or 32 when H >= 64
 * and T * (H / 32) * (the largest S the list takes) fits in the SMs.  The
 * pages size their SM clusters from the token batch in the same spirit (same
 * section).  Host-only; returns 0 for unsupported shapes.
 */
int32_t nvfp4_sparse_mla_num_splits(int32_t T, int32_t H, int32_t topk);

/*
 * nvfp4_sparse_mla_workspace_size -- bytes of device workspace
 * nvfp4_sparse_mla_decode needs for (T, H, topk) on the current device:
 * 0 when the lists are not split (S == 1), else 4096 bytes of split
 * counters followed by the softmax statistics and FP32 partial outputs of
 * the S splits.  Layout: [0, 4096) uint32 counter pairs, then [T][S][H][2]
 * FP32 (max, row sum), then [T][S][H][512] FP32.
 */
size_t nvfp4_sparse_mla_workspace_size(int32_t T, int32_t H, int32_t topk);

/*
 * nvfp4_sparse_mla_decode -- sparse MLA decode over the NVFP4 cache (same
 * page and section: only the rows the indexer selected are read, they are
 * unpacked on chip to FP16 MMA operands with FP32 accumulation, and list
 * entries that name no row contribute nothing).
 *
 *   q_nope_f16  [T, H, 512] FP16, contiguous, 16-byte aligned
 *   q_rope_f16  [T, H, 64]  FP16, contiguous, 16-byte aligned
 *   cache       [num_slots, 352] NVFP4 rows, 16-byte aligned
 *   indices     [T, topk] int32 slot ids, 16-byte aligned; an entry outside
 *               [0, num_slots) is empty: it takes no part in the softmax
 *               (entries < -1 or >= num_slots also set DEV_BAD_INDEX)
 *   sm_scale    softmax scale applied to q.k
 *   out_f16     [T, H, 512] FP16:  sum_j p_j V_j with p = softmax over the
 *               valid entries of sm_scale * (q_nope.k_lat + q_rope.k_rope),
 *               V_j = the 512 latent values of row j; all-empty -> 0
 *   lse         [T, H] FP32 natural-log sum-exp of the scaled scores;
 *               all-empty -> -inf
 *   workspace   device buffer of at least nvfp4_sparse_mla_workspace_size
 *               bytes (may be NULL when that size is 0), 256-byte aligned,
 *               owned by the caller.  Its first 4096 bytes (the split
 *               counters) must be zero before the first call that uses it
 *               (e.g. allocate it zero-filled); every call that completes
 *               leaves them zero again, for any shape.  After a call that
 *               raised NVFP4MLA_DEV_TIMEOUT they must be cleared again.
 *               When S > 1 the launch is cooperative: it fails with
 *               NVFP4MLA_ERR_CUDA if the device cannot hold all
 *               T * (H / min(H, 64)) * S CTAs at once.
 * Supported: 1 <= topk <= 2048; H in {16, 32, 64, 128}; T >= 0 (T == 0
 * is a no-op); num_slots >= 1.  Results are undefined for NaN/Inf queries.
 */
nvfp4mla_status nvfp4_sparse_mla_decode(const void *q_nope_f16, const void *q_rope_f16, const uint8_t *cache,
                                        int64_t num_slots, const int32_t *indices, int32_t topk, int32_t T,
                                        int32_t H, float sm_scale, void *out_f16, float *lse, void *workspace,
                                        size_t workspace_bytes, int32_t *dev_status, void *stream);

/*
 * nvfp4mla_tuning -- launch settings a caller may fix instead of the
 * automatic plan (sweeps, or forcing one path), for
 * nvfp4_sparse_mla_decode_tuned.  A zero field keeps the automatic choice.
 *   splits         CTAs sharing one token's list (S): a power of two no
 *                  larger than 16 nor than topk's 128-row tiles; with
 *                  S > 1, T * (H / heads_per_cta) * S must not exceed the
 *                  device's SMs (the merge needs every CTA resident) and
 *                  T * (H / heads_per_cta) must not exceed 512
 *   heads_per_cta  heads of one CTA (HG, the N of its MMAs): 16, 32 or 64,
 *                  at most H (automatic: min(H, 64))
 *   force_staged   nonzero: decode through the staged comparison path
 *                  (rows unpacked to 576-byte E4M3 in a staging buffer,
 *                  then attention over them) instead of the native kernel
 *   reserved       must be 0
 * The pages size the decode's SM clusters from the token batch (page
 * "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
 * section "Four-bit caches make room"); these fields let a caller set that
 * sizing by hand.
 */
typedef struct nvfp4mla_tuning {
    int32_t splits;
    int32_t heads_per_cta;
    int32_t force_staged;
    int32_t reserved;
} nvfp4mla_tuning;

/*
 * nvfp4_sparse_mla_workspace_size_tuned -- nvfp4_sparse_mla_workspace_size
 * for the plan `tuning` fixes (NULL: the automatic plan).  The staged path
 * needs its staging buffer besides (nvfp4_staged_fp8_staging_size).  Returns
 * 0 for a shape or setting the decode does not take.
 */
size_t nvfp4_sparse_mla_workspace_size_tuned(int32_t T, int32_t H, int32_t topk, const nvfp4mla_tuning *tuning);

/*
 * nvfp4_sparse_mla_decode_tuned -- nvfp4_sparse_mla_decode with the plan
 * `tuning` fixes (NULL: exactly nvfp4_sparse_mla_decode).
 *   workspace  as nvfp4_sparse_mla_decode, of at least
 *              nvfp4_sparse_mla_workspace_size_tuned bytes
 *   staging    with force_staged: [T, topk, 576] bytes, 16-byte aligned, at
 *              least nvfp4_staged_fp8_staging_size(T, topk); else unused
 *              (may be NULL)
 * Results are those of nvfp4_sparse_mla_decode (of the staged path with
 * force_staged); they differ only by FP32 rounding order between split
 * counts.  Errors: a setting the shape cannot take returns
 * NVFP4MLA_ERR_INVALID_ARG; the rest as nvfp4_sparse_mla_decode.
 */
nvfp4mla_status nvfp4_sparse_mla_decode_tuned(const void *q_nope_f16, const void *q_rope_f16, const uint8_t *cache,
                                              int64_t num_slots, const int32_t *indices, int32_t topk, int32_t T,
                                              int32_t H, float sm_scale, void *out_f16, float *lse, void *workspace,
                                              size_t workspace_bytes, uint8_t *staging, size_t staging_bytes,
                                              const nvfp4mla_tuning *tuning, int32_t *dev_status, void *stream);

/*
 * nvfp4_sparse_mla_decode_host -- nvfp4_sparse_mla_decode for inputs and
 * outputs in host memory: on `stream` it copies q_nope, q_rope and indices
 * from the host into the caller's device buffers (one cudaMemcpyAsync each),
 * runs the decode, and copies out and lse back to the host.  The pages'
 * serving loop moves each decode step's queries and lists to the GPU and its
 * results back; this call keeps those copies on the same stream as the
 * kernel, so a caller that alternates two streams (each with its own device
 * buffers and workspace) overlaps one step's copies with the other's kernel.
 *   *_host     host buffers with the shapes of nvfp4_sparse_mla_decode's
 *              arguments; page-locked memory (cudaHostAlloc) is needed for
 *              the copies to run asynchronously
 *   *_dev      device buffers of the same shapes, owned by the caller,
 *              16-byte aligned (lse_dev 4-byte)
 * The host output buffers are written when `stream` reaches the end of the
 * call; synchronize before reading them.  Other arguments, the workspace
 * contract and errors are those of nvfp4_sparse_mla_decode; a failed copy
 * returns NVFP4MLA_ERR_CUDA.
 */
nvfp4mla_status nvfp4_sparse_mla_decode_host(const void *q_nope_host, const void *q_rope_host,
                                             const int32_t *indices_host, void *out_host, float *lse_host,
                                             void *q_nope_dev, void *q_rope_dev, int32_t *indices_dev, void *out_dev,
                                             float *lse_dev, const uint8_t *cache, int64_t num_slots, int32_t topk,
                                             int32_t T, int32_t H, float sm_scale, void *workspace,
                                             size_t workspace_bytes, int32_t *dev_status, void *stream);

/*
 * nvfp4_sparse_mla_decode_paged -- nvfp4_sparse_mla_decode for lists of
 * request-local token positions instead of slot ids: the position -> slot
 * translation through each request's page table (the paged cache the pages'
 * deployment uses, same page and section) happens inside the launch, while
 * the list is compacted, so no translated list is ever written to memory.
 *
 *   positions    [T, topk] int32, 16-byte aligned: token positions in the
 *                request's context; -1 = empty
 *   block_table  [T, table_stride] int32, 4-byte aligned: page ids of token
 *                t's request in position order (slot = page * page_size +
 *                position % page_size); unused entries may hold -1
 *   table_stride entries per row of block_table (>= 1)
 *   page_size    slots per page, a power of two in [1, 2^20];
 *                table_stride * page_size must fit in int32
 * A position < -1 or >= table_stride * page_size, a page id < 0, or a slot
 * >= num_slots makes that entry empty and sets NVFP4MLA_DEV_BAD_INDEX.  Every
 * other argument, the workspace contract and the results are those of
 * nvfp4_sparse_mla_decode.
 */
nvfp4mla_status nvfp4_sparse_mla_decode_paged(const void *q_nope_f16, const void *q_rope_f16, const uint8_t *cache,
                                              int64_t num_slots, const int32_t *positions, int32_t topk,
                                              const int32_t *block_table, int32_t table_stride, int32_t page_size,
                                              int32_t T, int32_t H, float sm_scale, void *out_f16, float *lse,
                                              void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                              void *stream);

/*
 * nvfp4_sparse_mla_decode_noalloc -- nvfp4_sparse_mla_decode without a
 * caller-supplied workspace.  The pages have no counterpart: this is a
 * library convenience for callers that cannot hand out device memory per
 * call -- e.g. a serving engine that gave all free HBM to its paged KV cache
 * at start-up, or a code path that must not reach a device allocator.  The
 * split scratch is a static device array of 20 MiB per device (enough for
 * every plan on a device of up to 148 SMs); a plan that needs more returns
 * NVFP4MLA_ERR_WORKSPACE.  Nothing is allocated, no allocating library
 * routine is called.
 *
 *   Arguments, layouts and results: as nvfp4_sparse_mla_decode, minus the
 *   workspace.
 *   The first call on each device looks the scratch up
 *   (cudaGetSymbolAddress); make that call before any stream capture.
 *   The scratch's first 4096 bytes (split counters) start at zero when the
 *   library loads and every completed call leaves them zero; after a call
 *   that raised NVFP4MLA_DEV_TIMEOUT this entry point must not be used again
 *   in the process.
 *   All calls on one device share the scratch: calls that can overlap in time
 *   (different streams, or different host threads) race -- use
 *   nvfp4_sparse_mla_decode with separate workspaces for those.
 */
nvfp4mla_status nvfp4_sparse_mla_decode_noalloc(const void *q_nope_f16, const void *q_rope_f16,
                                                const uint8_t *cache, int64_t num_slots, const int32_t *indices,
                                                int32_t topk, int32_t T, int32_t H, float sm_scale, void *out_f16,
                                                float *lse, int32_t *dev_status, void *stream);

/*
 * nvfp4_staged_fp8_staging_size -- bytes of the FP8 staging buffer the
 * staged path writes: T * topk * 576.
 */
size_t nvfp4_staged_fp8_staging_size(int32_t T, int32_t topk);

/*
 * nvfp4_staged_fp8_mla_decode -- the staged comparison path (same page and
 * section: the earlier implementation expanded NVFP4 into FP8 buffers in GPU
 * memory before attention, which costs one more trip through HBM).  Kernel 1 gathers each
 * valid row, dequantizes it and re-encodes every value as E4M3 (round to
 * nearest even, saturating) into staging[t, j, 0:576] (512 latent then 64
 * RoPE); kernel 2 runs the same attention over the staging buffer.  Empty
 * entries leave their staging rows untouched and stay excluded.
 * Arguments as nvfp4_sparse_mla_decode, plus
 *   staging   [T, topk, 576] bytes, 16-byte aligned, at least
 *             nvfp4_staged_fp8_staging_size bytes
 * The result equals attention over the E4M3-rounded dequantized values.
 */
nvfp4mla_status nvfp4_staged_fp8_mla_decode(const void *q_nope_f16, const void *q_rope_f16, const uint8_t *cache,
                                            int64_t num_slots, const int32_t *indices, int32_t topk, int32_t T,
                                            int32_t H, float sm_scale, void *out_f16, float *lse,
                                            uint8_t *staging, size_t staging_bytes, void *workspace,
                                            size_t workspace_bytes, int32_t *dev_status, void *stream);

/*
 * nvfp4_staged_fp8_stage, nvfp4_staged_fp8_attend -- the two steps of
 * nvfp4_staged_fp8_mla_decode as separate calls (same page and section), so
 * each step can be launched, captured and timed on its own.  Calling
 * nvfp4_staged_fp8_stage and then nvfp4_staged_fp8_attend on the same
 * stream with the same arguments gives the result of
 * nvfp4_staged_fp8_mla_decode.
 *   stage:  cache, num_slots, indices, topk, T, staging, staging_bytes,
 *           stream as nvfp4_staged_fp8_mla_decode; writes the E4M3 rows of
 *           the valid entries into staging[t, j, 0:576]
 *   attend: every argument of nvfp4_staged_fp8_mla_decode except cache;
 *           reads staging[t, j] for the entries with 0 <= indices[t, j] <
 *           num_slots (the rows the stage step wrote)
 * Errors as nvfp4_staged_fp8_mla_decode.
 */
nvfp4mla_status nvfp4_staged_fp8_stage(const uint8_t *cache, int64_t num_slots, const int32_t *indices, int32_t topk,
                                       int32_t T, uint8_t *staging, size_t staging_bytes, void *stream);
nvfp4mla_status nvfp4_staged_fp8_attend(const void *q_nope_f16, const void *q_rope_f16, int64_t num_slots,
                                        const int32_t *indices, int32_t topk, int32_t T, int32_t H, float sm_scale,
                                        void *out_f16, float *lse, const uint8_t *staging, size_t staging_bytes,
                                        void *workspace, size_t workspace_bytes, int32_t *dev_status, void *stream);

/*
 * nvfp4mla_fp8_sparse_mla_decode -- the same attention as
 * nvfp4_sparse_mla_decode over a cache of 576-byte E4M3 rows (written by
 * nvfp4mla_fp8_kv_append): the "before" side of the 576 -> 352 byte row
 * change on the same page and section.  List entries are slots of
 * fp8_cache; keys are the E4M3 values of a row's 576 bytes, values its first
 * 512.  Arguments, workspace (nvfp4_sparse_mla_workspace_size), statuses and
 * the empty-entry rule are those of nvfp4_sparse_mla_decode, except
 *   fp8_cache  [num_slots, 576] bytes, 16-byte aligned
 */
nvfp4mla_status nvfp4mla_fp8_sparse_mla_decode(const void *q_nope_f16, const void *q_rope_f16,
                                               const uint8_t *fp8_cache, int64_t num_slots, const int32_t *indices,
                                               int32_t topk, int32_t T, int32_t H, float sm_scale, void *out_f16,
                                               float *lse, void *workspace, size_t workspace_bytes,
                                               int32_t *dev_status, void *stream);

/*
 * Sparse indexer: the step that produces the decode's index lists (same page
 * and section: a sparse indexer picks the rows each token's attention reads
 * and hands over 2,048 positions).  The page gives no scoring function; the
 * one computed here is the lightning-indexer form of DeepSeek sparse
 * attention:
 *   I[t, p] = sum_h w[t, h] * max(0, sum_d q[t, h, d] * k[slot(t, p), d])
 * over 64 heads h and 128 dims d, q and k E4M3 bytes, w FP32, for context
 * positions 0 <= p < ctx_lens[t], slot(t, p) = block_table[t][p / page] *
 * page + p % page.  The list of token t holds the min(topk, ctx_lens[t])
 * positions with the largest scores (equal scores: smaller position first;
 * -0 equals +0) in increasing position order, then -1 -- request-local
 * positions, the input of nvfp4_sparse_mla_decode_paged.
 *
 * Common arguments (device pointers, caller-owned):
 *   q_fp8        [T, 64, 128] E4M3 bytes, 16-byte aligned
 *   weights      [T, 64] FP32
 *   keys_fp8     [num_slots, 128] E4M3 bytes, 16-byte aligned; 1 <= num_slots <= INT32_MAX
 *   block_table  [T, table_stride] int32 page ids (negative = no page);
 *                a position whose page entry is negative or whose page
 *                leaves the key cache scores -inf and sets
 *                NVFP4MLA_DEV_BAD_INDEX
 *   page_size    a power of two in [8, 2^20]
 *   ctx_lens     [T] int32; a length outside [0, max_ctx] is clamped and
 *                sets NVFP4MLA_DEV_BAD_INDEX
 *   max_ctx      host-side bound on every ctx_lens[t];
 *                max_ctx <= table_stride * page_size
 *   scores       [T, score_stride] FP32, 16-byte aligned; score_stride >=
 *                max_ctx and a multiple of 4; only positions < ctx_lens[t]
 *                are written or read
 *   positions    [T, topk] int32, 1 <= topk <= 2048
 * Scores accumulate in FP32 on the tensor cores; which of two nearly equal
 * scores ranks first may differ from an exact evaluation.  NaN scores are
 * not supported.
 */

/* Workspace of nvfp4mla_indexer_topk for T requests on the current device:
 * 0 when each request's row is handled by one CTA (T >= SMs / 2), else
 * arrival counters, per-CTA candidate counts, thresholds and largest keys,
 * and candidate lists.  It must
 * be zero-filled before its first use; every completed call leaves the
 * counters at zero again. */
size_t nvfp4mla_indexer_topk_workspace_size(int32_t T);

/* Workspace of nvfp4mla_sparse_indexer: the score rows
 * (T * nvfp4mla_indexer_score_stride(max_ctx) floats, rounded up to 256
 * bytes) followed by nvfp4mla_indexer_topk_workspace_size(T) bytes; zero-fill
 * it before its first use (0 is returned for bad arguments). */
size_t nvfp4mla_indexer_workspace_size(int32_t T, int32_t max_ctx);
/* The score row stride (floats) nvfp4mla_sparse_indexer uses: max_ctx rounded up to 128. */
int64_t nvfp4mla_indexer_score_stride(int32_t max_ctx);

/* Scores of every context position of every token (first half of the
 * indexer). */
nvfp4mla_status nvfp4mla_indexer_scores(const uint8_t *q_fp8, const float *weights, const uint8_t *keys_fp8,
                                        int64_t num_slots, const int32_t *block_table, int32_t table_stride,
                                        int32_t page_size, const int32_t *ctx_lens, int32_t max_ctx, int32_t T,
                                        float *scores, int64_t score_stride, int32_t *dev_status, void *stream);

/* Selection over given scores (second half): positions[t] = the list
 * described above for scores[t, 0:ctx_lens[t]].  workspace: at least
 * nvfp4mla_indexer_topk_workspace_size(T) bytes, 256-byte aligned (NULL when
 * that is 0); WORKSPACE when missing or too small. */
nvfp4mla_status nvfp4mla_indexer_topk(const float *scores, int64_t score_stride, const int32_t *ctx_lens,
                                      int32_t max_ctx, int32_t T, int32_t topk, int32_t *positions,
                                      void *workspace, size_t workspace_bytes, int32_t *dev_status, void *stream);

/* Both halves; the scores and the selection's workspace live in
 * `workspace` (at least nvfp4mla_indexer_workspace_size bytes, 256-byte
 * aligned, zero-filled before its first use). */
nvfp4mla_status nvfp4mla_sparse_indexer(const uint8_t *q_fp8, const float *weights, const uint8_t *keys_fp8,
                                        int64_t num_slots, const int32_t *block_table, int32_t table_stride,
                                        int32_t page_size, const int32_t *ctx_lens, int32_t max_ctx, int32_t T,
                                        int32_t topk, int32_t *positions, void *workspace, size_t workspace_bytes,
                                        int32_t *dev_status, void *stream);

/*
 * Block-major multi-layer layout (same page, section "Fewer copies unlock
 * NVLink": the BLHNC layout keeps every layer of a block together, with
 * blocks a sixteenth of the earlier size, so moving a request needs about
 * ten times fewer copy descriptors).  The page gives no byte layout; the
 * one used here:
 *   per-layer caches   layer l: [num_blocks, block_size, row_bytes] bytes
 *   block-major cache  [num_new_blocks, layers, block_size / sub, row_bytes]
 * Positions j * (block_size/sub) .. (j+1) * (block_size/sub) - 1 of the
 * request's i-th block block_ids[i], every layer l, correspond to
 * block-major block new_block_ids[i * sub + j], layer slot l.
 *
 * nvfp4mla_blhnc_convert -- copies the request's data from the per-layer
 * caches to the block-major cache (to_blhnc = 1) or back (to_blhnc = 0).
 *   layer_caches   [layers] device array of the per-layer caches' device
 *                  addresses (each 16-byte aligned)
 *   block_ids      [nb] int32, new_block_ids [nb * sub] int32
 *   blhnc          the block-major cache, 16-byte aligned
 *   row_bytes      a multiple of 16; block_size a multiple of sub
 * A block id outside [0, num_blocks), a new id outside [0, num_new_blocks)
 * or a misaligned layer address skips that copy and sets
 * NVFP4MLA_DEV_BAD_INDEX.  Overlapping destinations race.
 */
nvfp4mla_status nvfp4mla_blhnc_convert(const uint64_t *layer_caches, int32_t layers, int64_t num_blocks,
                                       int32_t block_size, int32_t row_bytes, int32_t sub, const int32_t *block_ids,
                                       const int32_t *new_block_ids, int32_t nb, uint8_t *blhnc,
                                       int64_t num_new_blocks, int32_t to_blhnc, int32_t *dev_status, void *stream);

/*
 * nvfp4mla_copy_descriptors -- host-only descriptor model of a transfer:
 * layers * (number of runs of consecutive ids in ids[0:n]).  With the
 * request's block ids and its layer count it counts the copies of the
 * per-layer layout; with its block-major ids and layers = 1, those of the
 * block-major layout.  ids is a HOST pointer; returns -1 for bad arguments.
 */
int64_t nvfp4mla_copy_descriptors(const int32_t *ids, int32_t n, int32_t layers);

/*
 * nvfp4mla_selftest_wait_timeout -- checks, on the device, that the bounded
 * waits every kernel here uses end with a status instead of hanging: one CTA
 * waits on an mbarrier nothing arrives on and on *zero_word (which must stay
 * 0) reaching 1, each for about a millisecond, then ORs
 * NVFP4MLA_DEV_TIMEOUT into *dev_status and exits normally.  The context
 * stays usable.  Both pointers are device pointers owned by the caller.
 */
nvfp4mla_status nvfp4mla_selftest_wait_timeout(uint32_t *zero_word, int32_t *dev_status, void *stream);

/* The CUDA runtime error (a cudaError_t value) behind the last
 * NVFP4MLA_ERR_CUDA that a call of this library returned on the calling host
 * thread, or 0 if none has; and its description (static storage).  Neither
 * is reset by later successful calls. */
int32_t nvfp4mla_last_cuda_error(void);
const char *nvfp4mla_last_cuda_error_string(void);

/* Human-readable name of a status code (static storage). */
const char *nvfp4mla_status_string(nvfp4mla_status status);

/* Library ABI version: major*10000 + minor*100 + patch. */
int32_t nvfp4mla_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4MLA_H */
