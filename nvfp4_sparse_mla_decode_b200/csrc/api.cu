// api.cu -- the C ABI of libnvfp4mla (declared in include/nvfp4mla.h):
// argument checks, work planning, launches.  Nothing here allocates memory.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "../../include/nvfp4mla.h"
#include "decode_common.cuh"
#include "kernels.h"

using namespace nvfp4mla;

namespace {

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Scratch of nvfp4_sparse_mla_decode_noalloc: a file-scope device array, one
// per device, so that entry point never asks for memory.  Every split plan
// on a device with up to 148 SMs needs at most
// 4096 + 148 * 64 * (512 + 2) * 4 = 19,478,528 bytes; 20 MiB covers them, and
// a larger plan is refused.  Device globals are zero when the module loads,
// which is the state the split counters at its start must begin in.
constexpr size_t kNoAllocWorkspaceBytes = size_t(20) << 20;
static_assert(kSplitCounterBytes + size_t(148) * 64 * (NVFP4MLA_LATENT + 2) * 4 <= kNoAllocWorkspaceBytes,
              "the no-allocation scratch must hold every plan on a 148-SM device");
static __device__ __align__(256) uint8_t g_noalloc_workspace[kNoAllocWorkspaceBytes];

// Device address of the scratch on `dev`, looked up once per device.  The
// cache is read and written with acquire/release atomics, so first calls from
// several host threads at once are well defined (they may each look the
// address up; all of them store the same value).
void *noalloc_workspace(int dev) {
    static std::atomic<void *> addr[64] = {};
    if (dev < 0 || dev >= 64) return nullptr;
    void *cached = addr[dev].load(std::memory_order_acquire);
    if (!cached) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_workspace) != cudaSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        addr[dev].store(p, std::memory_order_release);
        cached = p;
    }
    return cached;
}

// The CUDA error behind the last NVFP4MLA_ERR_CUDA this host thread got.
thread_local cudaError_t g_last_cuda_error = cudaSuccess;

nvfp4mla_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return NVFP4MLA_OK;
    g_last_cuda_error = e;
    return NVFP4MLA_ERR_CUDA;
}

// The plan for (T, H, topk) with a caller's settings (tuning may be NULL):
// UNSUPPORTED for a shape the decode does not take, INVALID_ARG for settings
// the shape cannot take.
nvfp4mla_status decode_plan(int32_t T, int32_t H, int32_t topk, const nvfp4mla_tuning *tuning, DecodePlan *plan) {
    const int sms = current_device_sm_count();
    if (!make_decode_plan(T, H, topk, sms, plan)) return NVFP4MLA_ERR_UNSUPPORTED;
    if (!tuning) return NVFP4MLA_OK;
    if (tuning->reserved != 0 || tuning->splits < 0 || tuning->heads_per_cta < 0) return NVFP4MLA_ERR_INVALID_ARG;
    if (!make_decode_plan(T, H, topk, sms, plan, tuning->splits, tuning->heads_per_cta))
        return NVFP4MLA_ERR_INVALID_ARG;
    return NVFP4MLA_OK;
}

// Checks shared by the native and staged decode entry points.
nvfp4mla_status check_decode(const void *q_nope, const void *q_rope, const uint8_t *cache, int64_t num_slots,
                             const int32_t *indices, int32_t topk, int32_t T, int32_t H, float sm_scale,
                             const void *out, const float *lse, DecodePlan *plan,
                             const nvfp4mla_tuning *tuning = nullptr) {
    if (T < 0 || topk < 1 || topk > NVFP4MLA_MAX_TOPK || num_slots < 1 || num_slots > INT32_MAX)
        return NVFP4MLA_ERR_INVALID_ARG;
    if (!(sm_scale == sm_scale) || sm_scale > 3.0e38f || sm_scale < -3.0e38f) return NVFP4MLA_ERR_INVALID_ARG;
    const nvfp4mla_status pst = decode_plan(T, H, topk, tuning, plan);
    if (pst != NVFP4MLA_OK) return pst;
    if (T == 0) return NVFP4MLA_OK;
    if (!q_nope || !q_rope || !cache || !indices || !out || !lse) return NVFP4MLA_ERR_INVALID_ARG;
    if (!aligned(q_nope, 16) || !aligned(q_rope, 16) || !aligned(cache, 16) || !aligned(indices, 16) ||
        !aligned(out, 16) || !aligned(lse, 4))
        return NVFP4MLA_ERR_INVALID_ARG;
    return NVFP4MLA_OK;
}

}  // namespace

extern "C" {

nvfp4mla_status nvfp4_kv_append(const void *latent_bf16, int64_t latent_stride, const void *rope_bf16,
                                int64_t rope_stride, const int32_t *slot_mapping, int32_t n, uint8_t *cache,
                                int64_t num_slots, int32_t *dev_status, void *stream) {
    if (n < 0 || num_slots < 0 || latent_stride < NVFP4MLA_LATENT || rope_stride < NVFP4MLA_ROPE)
        return NVFP4MLA_ERR_INVALID_ARG;
    if (n == 0) return NVFP4MLA_OK;
    if (!latent_bf16 || !rope_bf16 || !slot_mapping || !cache) return NVFP4MLA_ERR_INVALID_ARG;
    if (latent_stride % 8 || rope_stride % 8 || !aligned(latent_bf16, 16) || !aligned(rope_bf16, 16) ||
        !aligned(cache, 16) || !aligned(slot_mapping, 4))
        return NVFP4MLA_ERR_INVALID_ARG;
    return from_cuda(launch_kv_append(latent_bf16, latent_stride, rope_bf16, rope_stride, slot_mapping, n, cache,
                                      num_slots, dev_status, static_cast<cudaStream_t>(stream)));
}

nvfp4mla_status nvfp4mla_fp8_kv_append(const void *latent_bf16, int64_t latent_stride, const void *rope_bf16,
                                       int64_t rope_stride, const int32_t *slot_mapping, int32_t n, uint8_t *cache,
                                       int64_t num_slots, int32_t *dev_status, void *stream) {
    if (n < 0 || num_slots < 0 || latent_stride < NVFP4MLA_LATENT || rope_stride < NVFP4MLA_ROPE)
        return NVFP4MLA_ERR_INVALID_ARG;
    if (n == 0) return NVFP4MLA_OK;
    if (!latent_bf16 || !rope_bf16 || !slot_mapping || !cache) return NVFP4MLA_ERR_INVALID_ARG;
    if (latent_stride % 8 || rope_stride % 8 || !aligned(latent_bf16, 16) || !aligned(rope_bf16, 16) ||
        !aligned(cache, 16) || !aligned(slot_mapping, 4))
        return NVFP4MLA_ERR_INVALID_ARG;
    return from_cuda(launch_fp8_kv_append(latent_bf16, latent_stride, rope_bf16, rope_stride, slot_mapping, n,
                                          cache, num_slots, dev_status, static_cast<cudaStream_t>(stream)));
}

int32_t nvfp4_sparse_mla_num_splits(int32_t T, int32_t H, int32_t topk) {
    DecodePlan p;
    return make_decode_plan(T, H, topk, current_device_sm_count(), &p) ? p.splits : 0;
}

size_t nvfp4_sparse_mla_workspace_size(int32_t T, int32_t H, int32_t topk) {
    DecodePlan p;
    return make_decode_plan(T, H, topk, current_device_sm_count(), &p) ? p.workspace_bytes : 0;
}

nvfp4mla_status nvfp4_sparse_mla_decode(const void *q_nope_f16, const void *q_rope_f16, const uint8_t *cache,
                                        int64_t num_slots, const int32_t *indices, int32_t topk, int32_t T,
                                        int32_t H, float sm_scale, void *out_f16, float *lse, void *workspace,
                                        size_t workspace_bytes, int32_t *dev_status, void *stream) {
    DecodePlan plan;
    nvfp4mla_status st =
        check_decode(q_nope_f16, q_rope_f16, cache, num_slots, indices, topk, T, H, sm_scale, out_f16, lse, &plan);
    if (st != NVFP4MLA_OK || T == 0) return st;
    if (plan.workspace_bytes > 0 && (!workspace || workspace_bytes < plan.workspace_bytes)) return NVFP4MLA_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 256)) return NVFP4MLA_ERR_INVALID_ARG;
    return from_cuda(launch_sparse_mla_decode(RowSource::kNvfp4Cache, q_nope_f16, q_rope_f16, cache, num_slots, indices, topk, T, H,
                                              sm_scale, out_f16, lse, workspace, plan, dev_status,
                                              static_cast<cudaStream_t>(stream)));
}

size_t nvfp4_sparse_mla_workspace_size_tuned(int32_t T, int32_t H, int32_t topk, const nvfp4mla_tuning *tuning) {
    DecodePlan p;
    if (T < 0 || topk < 1 || topk > NVFP4MLA_MAX_TOPK) return 0;
    return decode_plan(T, H, topk, tuning, &p) == NVFP4MLA_OK ? p.workspace_bytes : 0;
}

nvfp4mla_status nvfp4_sparse_mla_decode_tuned(const void *q_nope_f16, const void *q_rope_f16, const uint8_t *cache,
                                              int64_t num_slots, const int32_t *indices, int32_t topk, int32_t T,
                                              int32_t H, float sm_scale, void *out_f16, float *lse, void *workspace,
                                              size_t workspace_bytes, uint8_t *staging, size_t staging_bytes,
                                              const nvfp4mla_tuning *tuning, int32_t *dev_status, void *stream) {
    DecodePlan plan;
    nvfp4mla_status st = check_decode(q_nope_f16, q_rope_f16, cache, num_slots, indices, topk, T, H, sm_scale,
                                      out_f16, lse, &plan, tuning);
    if (st != NVFP4MLA_OK || T == 0) return st;
    if (plan.workspace_bytes > 0 && (!workspace || workspace_bytes < plan.workspace_bytes)) return NVFP4MLA_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 256)) return NVFP4MLA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (tuning && tuning->force_staged) {
        if (!staging || staging_bytes < nvfp4_staged_fp8_staging_size(T, topk)) return NVFP4MLA_ERR_WORKSPACE;
        if (!aligned(staging, 16)) return NVFP4MLA_ERR_INVALID_ARG;
        cudaError_t e = launch_stage_fp8(cache, num_slots, indices, topk, T, staging, s);
        if (e != cudaSuccess) return from_cuda(e);
        return from_cuda(launch_sparse_mla_decode(RowSource::kFp8Staging, q_nope_f16, q_rope_f16, staging, num_slots,
                                                  indices, topk, T, H, sm_scale, out_f16, lse, workspace, plan,
                                                  dev_status, s));
    }
    return from_cuda(launch_sparse_mla_decode(RowSource::kNvfp4Cache, q_nope_f16, q_rope_f16, cache, num_slots, indices,
                                              topk, T, H, sm_scale, out_f16, lse, workspace, plan, dev_status, s));
}

// Test-only (not in the public header): the NVFP4 decode with a chosen wait
// bound (SM clock cycles, > 0) and one arrival withheld (1: P^T is never
// published; 2: split 0 never arrives on the merge counter), so that tests
// can drive the kernel's timeout paths and check that it reports
// NVFP4MLA_DEV_TIMEOUT through dev_status and leaves the context usable.
nvfp4mla_status nvfp4mla_test_decode_hooks(const void *q_nope_f16, const void *q_rope_f16, const uint8_t *cache,
                                           int64_t num_slots, const int32_t *indices, int32_t topk, int32_t T,
                                           int32_t H, float sm_scale, void *out_f16, float *lse, void *workspace,
                                           size_t workspace_bytes, int32_t *dev_status, uint64_t wait_cycles,
                                           int32_t withhold, void *stream) {
    DecodePlan plan;
    nvfp4mla_status st =
        check_decode(q_nope_f16, q_rope_f16, cache, num_slots, indices, topk, T, H, sm_scale, out_f16, lse, &plan);
    if (st != NVFP4MLA_OK || T == 0) return st;
    if (wait_cycles == 0 || withhold < 0 || withhold > 2) return NVFP4MLA_ERR_INVALID_ARG;
    if (plan.workspace_bytes > 0 && (!workspace || workspace_bytes < plan.workspace_bytes)) return NVFP4MLA_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 256)) return NVFP4MLA_ERR_INVALID_ARG;
    DecodeTestHooks hooks{wait_cycles, withhold};
    return from_cuda(launch_sparse_mla_decode(RowSource::kNvfp4Cache, q_nope_f16, q_rope_f16, cache, num_slots, indices,
                                              topk, T, H, sm_scale, out_f16, lse, workspace, plan, dev_status,
                                              static_cast<cudaStream_t>(stream), nullptr, 0, 0, &hooks));
}

nvfp4mla_status nvfp4_sparse_mla_decode_host(const void *q_nope_host, const void *q_rope_host,
                                             const int32_t *indices_host, void *out_host, float *lse_host,
                                             void *q_nope_dev, void *q_rope_dev, int32_t *indices_dev, void *out_dev,
                                             float *lse_dev, const uint8_t *cache, int64_t num_slots, int32_t topk,
                                             int32_t T, int32_t H, float sm_scale, void *workspace,
                                             size_t workspace_bytes, int32_t *dev_status, void *stream) {
    DecodePlan plan;
    nvfp4mla_status st = check_decode(q_nope_dev, q_rope_dev, cache, num_slots, indices_dev, topk, T, H, sm_scale,
                                      out_dev, lse_dev, &plan);
    if (st != NVFP4MLA_OK || T == 0) return st;
    if (!q_nope_host || !q_rope_host || !indices_host || !out_host || !lse_host) return NVFP4MLA_ERR_INVALID_ARG;
    if (plan.workspace_bytes > 0 && (!workspace || workspace_bytes < plan.workspace_bytes)) return NVFP4MLA_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 256)) return NVFP4MLA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t th = (size_t)T * (size_t)H;
    cudaError_t e = cudaMemcpyAsync(q_nope_dev, q_nope_host, th * NVFP4MLA_LATENT * 2, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(q_rope_dev, q_rope_host, th * NVFP4MLA_ROPE * 2, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(indices_dev, indices_host, (size_t)T * topk * 4, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess)
        e = launch_sparse_mla_decode(RowSource::kNvfp4Cache, q_nope_dev, q_rope_dev, cache, num_slots, indices_dev, topk,
                                     T, H, sm_scale, out_dev, lse_dev, workspace, plan, dev_status, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(out_host, out_dev, th * NVFP4MLA_LATENT * 2, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaMemcpyAsync(lse_host, lse_dev, th * 4, cudaMemcpyDeviceToHost, s);
    return from_cuda(e);
}

nvfp4mla_status nvfp4_sparse_mla_decode_paged(const void *q_nope_f16, const void *q_rope_f16, const uint8_t *cache,
                                              int64_t num_slots, const int32_t *positions, int32_t topk,
                                              const int32_t *block_table, int32_t table_stride, int32_t page_size,
                                              int32_t T, int32_t H, float sm_scale, void *out_f16, float *lse,
                                              void *workspace, size_t workspace_bytes, int32_t *dev_status,
                                              void *stream) {
    DecodePlan plan;
    nvfp4mla_status st =
        check_decode(q_nope_f16, q_rope_f16, cache, num_slots, positions, topk, T, H, sm_scale, out_f16, lse, &plan);
    if (st != NVFP4MLA_OK) return st;
    int shift = 0;
    while (shift < 21 && (1 << shift) < page_size) ++shift;
    if (page_size < 1 || page_size > (1 << 20) || (1 << shift) != page_size || table_stride < 1 ||
        (int64_t)table_stride * page_size > INT32_MAX)
        return NVFP4MLA_ERR_INVALID_ARG;
    if (T == 0) return NVFP4MLA_OK;
    if (!block_table || !aligned(block_table, 4)) return NVFP4MLA_ERR_INVALID_ARG;
    if (plan.workspace_bytes > 0 && (!workspace || workspace_bytes < plan.workspace_bytes)) return NVFP4MLA_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 256)) return NVFP4MLA_ERR_INVALID_ARG;
    return from_cuda(launch_sparse_mla_decode(RowSource::kNvfp4Cache, q_nope_f16, q_rope_f16, cache, num_slots, positions, topk, T, H,
                                              sm_scale, out_f16, lse, workspace, plan, dev_status,
                                              static_cast<cudaStream_t>(stream), block_table, table_stride, shift));
}

nvfp4mla_status nvfp4_sparse_mla_decode_noalloc(const void *q_nope_f16, const void *q_rope_f16,
                                                const uint8_t *cache, int64_t num_slots, const int32_t *indices,
                                                int32_t topk, int32_t T, int32_t H, float sm_scale, void *out_f16,
                                                float *lse, int32_t *dev_status, void *stream) {
    DecodePlan plan;
    nvfp4mla_status st =
        check_decode(q_nope_f16, q_rope_f16, cache, num_slots, indices, topk, T, H, sm_scale, out_f16, lse, &plan);
    if (st != NVFP4MLA_OK || T == 0) return st;
    if (plan.workspace_bytes > kNoAllocWorkspaceBytes) return NVFP4MLA_ERR_WORKSPACE;
    void *ws = nullptr;
    if (plan.workspace_bytes > 0) {
        int dev = 0;
        const cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return from_cuda(e);
        ws = noalloc_workspace(dev);
        if (!ws) return from_cuda(cudaErrorMemoryAllocation);
    }
    return from_cuda(launch_sparse_mla_decode(RowSource::kNvfp4Cache, q_nope_f16, q_rope_f16, cache, num_slots, indices, topk, T, H,
                                              sm_scale, out_f16, lse, ws, plan, dev_status,
                                              static_cast<cudaStream_t>(stream)));
}

size_t nvfp4_staged_fp8_staging_size(int32_t T, int32_t topk) {
    if (T < 0 || topk < 0) return 0;
    return (size_t)T * (size_t)topk * NVFP4MLA_STAGED_ROW_BYTES;
}

nvfp4mla_status nvfp4_staged_fp8_mla_decode(const void *q_nope_f16, const void *q_rope_f16, const uint8_t *cache,
                                            int64_t num_slots, const int32_t *indices, int32_t topk, int32_t T,
                                            int32_t H, float sm_scale, void *out_f16, float *lse,
                                            uint8_t *staging, size_t staging_bytes, void *workspace,
                                            size_t workspace_bytes, int32_t *dev_status, void *stream) {
    DecodePlan plan;
    nvfp4mla_status st =
        check_decode(q_nope_f16, q_rope_f16, cache, num_slots, indices, topk, T, H, sm_scale, out_f16, lse, &plan);
    if (st != NVFP4MLA_OK || T == 0) return st;
    if (!staging || staging_bytes < nvfp4_staged_fp8_staging_size(T, topk)) return NVFP4MLA_ERR_WORKSPACE;
    if (!aligned(staging, 16)) return NVFP4MLA_ERR_INVALID_ARG;
    if (plan.workspace_bytes > 0 && (!workspace || workspace_bytes < plan.workspace_bytes)) return NVFP4MLA_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 256)) return NVFP4MLA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = launch_stage_fp8(cache, num_slots, indices, topk, T, staging, s);
    if (e != cudaSuccess) return from_cuda(e);
    return from_cuda(launch_sparse_mla_decode(RowSource::kFp8Staging, q_nope_f16, q_rope_f16, staging, num_slots, indices, topk, T, H,
                                              sm_scale, out_f16, lse, workspace, plan, dev_status, s));
}

nvfp4mla_status nvfp4_staged_fp8_stage(const uint8_t *cache, int64_t num_slots, const int32_t *indices, int32_t topk,
                                       int32_t T, uint8_t *staging, size_t staging_bytes, void *stream) {
    if (T < 0 || topk < 1 || topk > NVFP4MLA_MAX_TOPK || num_slots < 1 || num_slots > INT32_MAX)
        return NVFP4MLA_ERR_INVALID_ARG;
    if (T == 0) return NVFP4MLA_OK;
    if (!cache || !indices || !staging) return NVFP4MLA_ERR_INVALID_ARG;
    if (!aligned(cache, 16) || !aligned(indices, 4) || !aligned(staging, 16)) return NVFP4MLA_ERR_INVALID_ARG;
    if (staging_bytes < nvfp4_staged_fp8_staging_size(T, topk)) return NVFP4MLA_ERR_WORKSPACE;
    return from_cuda(launch_stage_fp8(cache, num_slots, indices, topk, T, staging, static_cast<cudaStream_t>(stream)));
}

nvfp4mla_status nvfp4_staged_fp8_attend(const void *q_nope_f16, const void *q_rope_f16, int64_t num_slots,
                                        const int32_t *indices, int32_t topk, int32_t T, int32_t H, float sm_scale,
                                        void *out_f16, float *lse, const uint8_t *staging, size_t staging_bytes,
                                        void *workspace, size_t workspace_bytes, int32_t *dev_status, void *stream) {
    DecodePlan plan;
    nvfp4mla_status st = check_decode(q_nope_f16, q_rope_f16, staging, num_slots, indices, topk, T, H, sm_scale,
                                      out_f16, lse, &plan);
    if (st != NVFP4MLA_OK || T == 0) return st;
    if (staging_bytes < nvfp4_staged_fp8_staging_size(T, topk)) return NVFP4MLA_ERR_WORKSPACE;
    if (plan.workspace_bytes > 0 && (!workspace || workspace_bytes < plan.workspace_bytes)) return NVFP4MLA_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 256)) return NVFP4MLA_ERR_INVALID_ARG;
    return from_cuda(launch_sparse_mla_decode(RowSource::kFp8Staging, q_nope_f16, q_rope_f16, staging, num_slots,
                                              indices, topk, T, H, sm_scale, out_f16, lse, workspace, plan,
                                              dev_status, static_cast<cudaStream_t>(stream)));
}

nvfp4mla_status nvfp4mla_fp8_sparse_mla_decode(const void *q_nope_f16, const void *q_rope_f16,
                                               const uint8_t *fp8_cache, int64_t num_slots, const int32_t *indices,
                                               int32_t topk, int32_t T, int32_t H, float sm_scale, void *out_f16,
                                               float *lse, void *workspace, size_t workspace_bytes,
                                               int32_t *dev_status, void *stream) {
    DecodePlan plan;
    nvfp4mla_status st = check_decode(q_nope_f16, q_rope_f16, fp8_cache, num_slots, indices, topk, T, H, sm_scale,
                                      out_f16, lse, &plan);
    if (st != NVFP4MLA_OK || T == 0) return st;
    if (plan.workspace_bytes > 0 && (!workspace || workspace_bytes < plan.workspace_bytes)) return NVFP4MLA_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 256)) return NVFP4MLA_ERR_INVALID_ARG;
    return from_cuda(launch_sparse_mla_decode(RowSource::kFp8Cache, q_nope_f16, q_rope_f16, fp8_cache, num_slots,
                                              indices, topk, T, H, sm_scale, out_f16, lse, workspace, plan,
                                              dev_status, static_cast<cudaStream_t>(stream)));
}

size_t nvfp4mla_indexer_topk_workspace_size(int32_t T) {
    return T < 0 ? 0 : indexer_topk_workspace_bytes(T, current_device_sm_count());
}

// Scores first, then the selection's workspace at a 256-byte boundary.
static size_t indexer_scores_bytes(int32_t T, int32_t max_ctx) {
    return ((size_t)T * (size_t)indexer_score_stride(max_ctx) * sizeof(float) + 255) / 256 * 256;
}

size_t nvfp4mla_indexer_workspace_size(int32_t T, int32_t max_ctx) {
    if (T < 0 || max_ctx < 0 || max_ctx > INT32_MAX - 128) return 0;
    return indexer_scores_bytes(T, max_ctx) + nvfp4mla_indexer_topk_workspace_size(T);
}

int64_t nvfp4mla_indexer_score_stride(int32_t max_ctx) {
    return (max_ctx < 0 || max_ctx > INT32_MAX - 128) ? 0 : indexer_score_stride(max_ctx);
}

nvfp4mla_status nvfp4mla_indexer_scores(const uint8_t *q_fp8, const float *weights, const uint8_t *keys_fp8,
                                        int64_t num_slots, const int32_t *block_table, int32_t table_stride,
                                        int32_t page_size, const int32_t *ctx_lens, int32_t max_ctx, int32_t T,
                                        float *scores, int64_t score_stride, int32_t *dev_status, void *stream) {
    if (T < 0 || max_ctx < 0 || max_ctx > INT32_MAX - 128 || num_slots < 1 || num_slots > INT32_MAX ||
        table_stride < 1)
        return NVFP4MLA_ERR_INVALID_ARG;
    int shift = 0;
    while (shift < 21 && (1 << shift) < page_size) ++shift;
    if (page_size < 8 || page_size > (1 << 20) || (1 << shift) != page_size ||
        (int64_t)max_ctx > (int64_t)table_stride * page_size)
        return NVFP4MLA_ERR_INVALID_ARG;
    if (score_stride < max_ctx || score_stride % 4) return NVFP4MLA_ERR_INVALID_ARG;
    if (T == 0 || max_ctx == 0) return NVFP4MLA_OK;
    if (!q_fp8 || !weights || !keys_fp8 || !block_table || !ctx_lens || !scores) return NVFP4MLA_ERR_INVALID_ARG;
    if (!aligned(q_fp8, 16) || !aligned(keys_fp8, 16) || !aligned(weights, 4) || !aligned(block_table, 4) ||
        !aligned(ctx_lens, 4) || !aligned(scores, 16))
        return NVFP4MLA_ERR_INVALID_ARG;
    return from_cuda(launch_indexer_scores(q_fp8, weights, keys_fp8, num_slots, block_table, table_stride, shift,
                                           ctx_lens, max_ctx, T, scores, score_stride, dev_status,
                                           static_cast<cudaStream_t>(stream)));
}

nvfp4mla_status nvfp4mla_indexer_topk(const float *scores, int64_t score_stride, const int32_t *ctx_lens,
                                      int32_t max_ctx, int32_t T, int32_t topk, int32_t *positions,
                                      void *workspace, size_t workspace_bytes, int32_t *dev_status, void *stream) {
    if (T < 0 || max_ctx < 0 || max_ctx > INT32_MAX - 128 || topk < 1 || topk > NVFP4MLA_MAX_TOPK ||
        score_stride < max_ctx || score_stride % 4)
        return NVFP4MLA_ERR_INVALID_ARG;
    if (T == 0) return NVFP4MLA_OK;
    if (!ctx_lens || !positions || (max_ctx > 0 && !scores)) return NVFP4MLA_ERR_INVALID_ARG;
    if (!aligned(scores, 16) || !aligned(ctx_lens, 4) || !aligned(positions, 4)) return NVFP4MLA_ERR_INVALID_ARG;
    const size_t need = nvfp4mla_indexer_topk_workspace_size(T);
    if (need > 0 && (!workspace || workspace_bytes < need)) return NVFP4MLA_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 256)) return NVFP4MLA_ERR_INVALID_ARG;
    return from_cuda(launch_indexer_topk(scores, score_stride, ctx_lens, max_ctx, T, topk, positions, workspace,
                                         dev_status, static_cast<cudaStream_t>(stream)));
}

nvfp4mla_status nvfp4mla_sparse_indexer(const uint8_t *q_fp8, const float *weights, const uint8_t *keys_fp8,
                                        int64_t num_slots, const int32_t *block_table, int32_t table_stride,
                                        int32_t page_size, const int32_t *ctx_lens, int32_t max_ctx, int32_t T,
                                        int32_t topk, int32_t *positions, void *workspace, size_t workspace_bytes,
                                        int32_t *dev_status, void *stream) {
    if (topk < 1 || topk > NVFP4MLA_MAX_TOPK) return NVFP4MLA_ERR_INVALID_ARG;
    const size_t need = nvfp4mla_indexer_workspace_size(T, max_ctx);
    if (T > 0 && max_ctx > 0 && (!workspace || workspace_bytes < need)) return NVFP4MLA_ERR_WORKSPACE;
    if (workspace && !aligned(workspace, 256)) return NVFP4MLA_ERR_INVALID_ARG;
    const int64_t stride = nvfp4mla_indexer_score_stride(max_ctx);
    float *sc = static_cast<float *>(workspace);
    nvfp4mla_status st = nvfp4mla_indexer_scores(q_fp8, weights, keys_fp8, num_slots, block_table, table_stride,
                                                 page_size, ctx_lens, max_ctx, T, sc, stride, dev_status, stream);
    if (st != NVFP4MLA_OK) return st;
    const size_t off = T > 0 ? indexer_scores_bytes(T, max_ctx) : 0;
    uint8_t *tw = workspace ? static_cast<uint8_t *>(workspace) + off : nullptr;
    return nvfp4mla_indexer_topk(sc, stride, ctx_lens, max_ctx, T, topk, positions, tw,
                                 workspace_bytes > off ? workspace_bytes - off : 0, dev_status, stream);
}

nvfp4mla_status nvfp4mla_blhnc_convert(const uint64_t *layer_caches, int32_t layers, int64_t num_blocks,
                                       int32_t block_size, int32_t row_bytes, int32_t sub, const int32_t *block_ids,
                                       const int32_t *new_block_ids, int32_t nb, uint8_t *blhnc,
                                       int64_t num_new_blocks, int32_t to_blhnc, int32_t *dev_status, void *stream) {
    if (layers < 1 || num_blocks < 1 || block_size < 1 || sub < 1 || block_size % sub || row_bytes < 16 ||
        row_bytes % 16 || nb < 0 || num_new_blocks < 1 || (to_blhnc != 0 && to_blhnc != 1))
        return NVFP4MLA_ERR_INVALID_ARG;
    if ((int64_t)block_size * row_bytes > INT32_MAX) return NVFP4MLA_ERR_INVALID_ARG;
    if (nb == 0) return NVFP4MLA_OK;
    if (!layer_caches || !block_ids || !new_block_ids || !blhnc) return NVFP4MLA_ERR_INVALID_ARG;
    if (!aligned(layer_caches, 8) || !aligned(block_ids, 4) || !aligned(new_block_ids, 4) || !aligned(blhnc, 16))
        return NVFP4MLA_ERR_INVALID_ARG;
    return from_cuda(launch_blhnc_convert(layer_caches, layers, num_blocks, block_size, row_bytes, sub, block_ids,
                                          new_block_ids, nb, blhnc, num_new_blocks, to_blhnc != 0, dev_status,
                                          static_cast<cudaStream_t>(stream)));
}

int64_t nvfp4mla_copy_descriptors(const int32_t *ids, int32_t n, int32_t layers) {
    if (n < 0 || layers < 1 || (n > 0 && !ids)) return -1;
    int64_t runs = 0;
    for (int32_t k = 0; k < n; ++k)
        if (k == 0 || (int64_t)ids[k] != (int64_t)ids[k - 1] + 1) ++runs;
    return runs * layers;
}

nvfp4mla_status nvfp4mla_selftest_wait_timeout(uint32_t *zero_word, int32_t *dev_status, void *stream) {
    if (!zero_word || !dev_status || !aligned(zero_word, 4) || !aligned(dev_status, 4))
        return NVFP4MLA_ERR_INVALID_ARG;
    return from_cuda(launch_wait_timeout_selftest(zero_word, dev_status, static_cast<cudaStream_t>(stream)));
}

int32_t nvfp4mla_last_cuda_error(void) { return (int32_t)g_last_cuda_error; }

const char *nvfp4mla_last_cuda_error_string(void) { return cudaGetErrorString(g_last_cuda_error); }

const char *nvfp4mla_status_string(nvfp4mla_status status) {
    switch (status) {
        case NVFP4MLA_OK: return "ok";
        case NVFP4MLA_ERR_INVALID_ARG: return "invalid argument";
        case NVFP4MLA_ERR_UNSUPPORTED: return "unsupported shape";
        case NVFP4MLA_ERR_WORKSPACE: return "workspace or staging buffer too small";
        case NVFP4MLA_ERR_CUDA: return "CUDA runtime error";
        case NVFP4MLA_ERR_TIMEOUT: return "device wait timed out";
        case NVFP4MLA_ERR_BAD_INDEX: return "index or slot out of range";
    }
    return "unknown status";
}

int32_t nvfp4mla_version(void) { return 100; }

}  // extern "C"
