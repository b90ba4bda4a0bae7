// append.cu -- nvfp4_kv_append: BF16 latent + RoPE rows -> 352-byte NVFP4
// rows at scattered cache slots (and nvfp4mla_fp8_kv_append: the same rows
// as 576-byte E4M3 rows).
//
// Page "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
// section "Four-bit caches make room": NVFP4 keeps an FP8 scale for every 16
// values and the cache row becomes 352 bytes.  Per group of 16 latent
// values: scale = E4M3_RNE_sat(max|x| / 6), value codes = E2M1_RNE_sat(x /
// scale) (all zero when the scale is 0); RoPE dims are E4M3_RNE_sat(x).
//
// One warp per row: lane g owns latent group g (16 values, 32 bytes of BF16
// in, 8 nibble bytes + 1 scale byte out) and RoPE dims 2g, 2g+1.  Every store
// of a warp is contiguous (256 B nibbles, 32 B scales, 64 B RoPE), so the
// kernel moves 1152 B in and 352 B out per row at streaming bandwidth.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4mla {

__global__ void __launch_bounds__(256) kv_append_kernel(const __nv_bfloat16 *__restrict__ latent,
                                                        int64_t latent_stride,
                                                        const __nv_bfloat16 *__restrict__ rope, int64_t rope_stride,
                                                        const int32_t *__restrict__ slot_mapping, int32_t n,
                                                        uint8_t *__restrict__ cache, int64_t num_slots,
                                                        int32_t *__restrict__ dev_status) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= n) return;
    const int64_t slot = slot_mapping[row];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (lane == 0 && dev_status) atomicOr(dev_status, NVFP4MLA_DEV_BAD_INDEX);
        return;
    }
    // 16 BF16 latent values of group `lane`
    const uint4 *src = reinterpret_cast<const uint4 *>(latent + row * latent_stride + lane * kGroup);
    const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    float x[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
    const uint32_t scode = e4m3_rne_sat(__fdiv_rn(amax, 6.0f));
    const float s = e4m3_to_float(scode);
    uint32_t lo = 0, hi = 0;
    if (s != 0.0f) {
#pragma unroll
        for (int i = 0; i < 8; ++i) lo |= e2m1_rne_sat(__fdiv_rn(x[i], s)) << (4 * i);
#pragma unroll
        for (int i = 0; i < 8; ++i) hi |= e2m1_rne_sat(__fdiv_rn(x[8 + i], s)) << (4 * i);
    }
    uint8_t *dst = cache + slot * kRowBytes;
    *reinterpret_cast<uint2 *>(dst + lane * 8) = make_uint2(lo, hi);
    dst[kScaleOff + lane] = (uint8_t)scode;
    // RoPE dims 2*lane, 2*lane+1
    const uint32_t rp = *reinterpret_cast<const uint32_t *>(rope + row * rope_stride + 2 * lane);
    const uint32_t r0 = e4m3_rne_sat(__uint_as_float(rp << 16));
    const uint32_t r1 = e4m3_rne_sat(__uint_as_float(rp & 0xFFFF0000u));
    *reinterpret_cast<uint16_t *>(dst + kRopeOff + 2 * lane) = (uint16_t)(r0 | (r1 << 8));
}

cudaError_t launch_kv_append(const void *latent, int64_t latent_stride, const void *rope, int64_t rope_stride,
                             const int32_t *slot_mapping, int32_t n, uint8_t *cache, int64_t num_slots,
                             int32_t *dev_status, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    const int rows_per_block = 8;
    const int blocks = (n + rows_per_block - 1) / rows_per_block;
    kv_append_kernel<<<blocks, 32 * rows_per_block, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(latent), latent_stride, static_cast<const __nv_bfloat16 *>(rope),
        rope_stride, slot_mapping, n, cache, num_slots, dev_status);
    return cudaGetLastError();
}

// The pre-NVFP4 row (same page and section: cache rows were 576 bytes before
// the four-bit format): every latent and RoPE value becomes its own E4M3
// byte, round to nearest even, saturating, with no scale.  One warp per row:
// lane g converts latent dims 16g..16g+15 (32 B in, one 16-byte store) and
// RoPE dims 2g, 2g+1.
__global__ void __launch_bounds__(256) fp8_kv_append_kernel(const __nv_bfloat16 *__restrict__ latent,
                                                            int64_t latent_stride,
                                                            const __nv_bfloat16 *__restrict__ rope,
                                                            int64_t rope_stride,
                                                            const int32_t *__restrict__ slot_mapping, int32_t n,
                                                            uint8_t *__restrict__ cache, int64_t num_slots,
                                                            int32_t *__restrict__ dev_status) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= n) return;
    const int64_t slot = slot_mapping[row];
    if (slot < 0) return;
    if (slot >= num_slots) {
        if (lane == 0 && dev_status) atomicOr(dev_status, NVFP4MLA_DEV_BAD_INDEX);
        return;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>(latent + row * latent_stride + lane * kGroup);
    const uint4 v0 = __ldg(src), v1 = __ldg(src + 1);
    const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t out[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t lo = w[2 * q], hi = w[2 * q + 1];
        out[q] = e4m3_rne_sat(__uint_as_float(lo << 16)) | (e4m3_rne_sat(__uint_as_float(lo & 0xFFFF0000u)) << 8) |
                 (e4m3_rne_sat(__uint_as_float(hi << 16)) << 16) |
                 (e4m3_rne_sat(__uint_as_float(hi & 0xFFFF0000u)) << 24);
    }
    uint8_t *dst = cache + slot * kStagedRowBytes;
    *reinterpret_cast<uint4 *>(dst + 16 * lane) = make_uint4(out[0], out[1], out[2], out[3]);
    const uint32_t rp = *reinterpret_cast<const uint32_t *>(rope + row * rope_stride + 2 * lane);
    const uint32_t r0 = e4m3_rne_sat(__uint_as_float(rp << 16));
    const uint32_t r1 = e4m3_rne_sat(__uint_as_float(rp & 0xFFFF0000u));
    *reinterpret_cast<uint16_t *>(dst + kLatent + 2 * lane) = (uint16_t)(r0 | (r1 << 8));
}

cudaError_t launch_fp8_kv_append(const void *latent, int64_t latent_stride, const void *rope, int64_t rope_stride,
                                 const int32_t *slot_mapping, int32_t n, uint8_t *cache, int64_t num_slots,
                                 int32_t *dev_status, cudaStream_t stream) {
    if (n <= 0) return cudaSuccess;
    const int rows_per_block = 8;
    const int blocks = (n + rows_per_block - 1) / rows_per_block;
    fp8_kv_append_kernel<<<blocks, 32 * rows_per_block, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(latent), latent_stride, static_cast<const __nv_bfloat16 *>(rope),
        rope_stride, slot_mapping, n, cache, num_slots, dev_status);
    return cudaGetLastError();
}

}  // namespace nvfp4mla
