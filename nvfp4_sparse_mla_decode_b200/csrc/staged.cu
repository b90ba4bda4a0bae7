// staged.cu -- the staged comparison path: expand the gathered NVFP4 rows
// into E4M3 rows in HBM, then run the same attention kernel over them.
//
// Page "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
// section "Four-bit caches make room": before the native kernel, the NVFP4
// cache was first expanded into FP8 buffers in GPU memory and attention ran
// on those, paying one more round trip through memory per layer.  The FP8
// row is the pre-NVFP4 576-byte row: 512 latent then 64 RoPE values, each
// the E4M3 (round to nearest even, saturating) re-encoding of the exact
// dequantized value.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4mla {

// One warp per list entry (t, j): lane g re-encodes latent group g (16
// values -> 16 bytes) and RoPE dims 2g, 2g+1.  Empty entries are skipped.
__global__ void __launch_bounds__(256) stage_fp8_kernel(const uint8_t *__restrict__ cache, int64_t num_slots,
                                                        const int32_t *__restrict__ indices, int32_t topk,
                                                        int64_t entries, uint8_t *__restrict__ staging) {
    const int lane = threadIdx.x & 31;
    const int64_t e = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (e >= entries) return;
    const int32_t slot = __ldg(indices + e);
    if (slot < 0 || (int64_t)slot >= num_slots) return;
    const uint8_t *row = cache + (int64_t)slot * kRowBytes;
    const uint2 nib = __ldg(reinterpret_cast<const uint2 *>(row + 8 * lane));
    const float s = e4m3_to_float(row[kScaleOff + lane]);
    uint32_t outw[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t src = q < 2 ? nib.x : nib.y;
        uint32_t w = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int i = (q & 1) * 4 + b;  // value index within the 8 of this word
            const uint32_t code = (src >> (4 * i)) & 0xFu;
            const uint32_t mag = code & 7u;
            float v = (mag < 2 ? 0.5f * (float)mag : (float)(1u << ((mag >> 1) - 1)) * (1.0f + 0.5f * (float)(mag & 1u)));
            v = (code & 8u) ? -v : v;
            w |= e4m3_rne_sat(v * s) << (8 * b);
        }
        outw[q] = w;
    }
    uint8_t *dst = staging + e * kStagedRowBytes;
    *reinterpret_cast<uint4 *>(dst + 16 * lane) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
    const uint32_t r0 = e4m3_rne_sat(e4m3_to_float(row[kRopeOff + 2 * lane]));
    const uint32_t r1 = e4m3_rne_sat(e4m3_to_float(row[kRopeOff + 2 * lane + 1]));
    *reinterpret_cast<uint16_t *>(dst + kLatent + 2 * lane) = (uint16_t)(r0 | (r1 << 8));
}

cudaError_t launch_stage_fp8(const uint8_t *cache, int64_t num_slots, const int32_t *indices, int32_t topk,
                             int32_t T, uint8_t *staging, cudaStream_t stream) {
    const int64_t entries = (int64_t)T * topk;
    if (entries == 0) return cudaSuccess;
    const int per_block = 8;
    stage_fp8_kernel<<<(unsigned)((entries + per_block - 1) / per_block), 32 * per_block, 0, stream>>>(
        cache, num_slots, indices, topk, entries, staging);
    return cudaGetLastError();
}

}  // namespace nvfp4mla
