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

// Two FP16 values -> two E4M3 bytes (round to nearest even, saturating to
// +-448), low half -> low byte.
__device__ __forceinline__ uint32_t f16x2_to_e4m3x2(uint32_t h2) {
    uint32_t d;
    asm("{\n\t.reg .b16 r;\n\tcvt.rn.satfinite.e4m3x2.f16x2 r, %1;\n\tcvt.u32.u16 %0, r;\n\t}" : "=r"(d) : "r"(h2));
    return d;
}

// Warps stride over the list entries (t, j); per entry lane g re-encodes
// latent group g (16 values -> 16 bytes) and copies RoPE bytes 2g, 2g+1 (an
// E4M3 value re-encodes to itself).  A latent value is formed exactly in
// FP16 (e2m1 x e4m3 has at most 6 significant bits) and rounded once to
// E4M3.  Empty entries are skipped.
__global__ void __launch_bounds__(256) stage_fp8_kernel(const uint8_t *__restrict__ cache, int64_t num_slots,
                                                        const int32_t *__restrict__ indices, int64_t entries,
                                                        uint8_t *__restrict__ staging) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t e = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); e < entries; e += warps) {
        const int32_t slot = __ldg(indices + e);
        if (slot < 0 || (int64_t)slot >= num_slots) continue;
        const uint8_t *row = cache + (int64_t)slot * kRowBytes;
        const uint2 nib = __ldg(reinterpret_cast<const uint2 *>(row + 8 * lane));
        const uint32_t sb = __ldg(row + kScaleOff + lane);
        const uint16_t rope = __ldg(reinterpret_cast<const uint16_t *>(row + kRopeOff + 2 * lane));
        const uint32_t s2 = e4m3x2_to_f16x2(sb | (sb << 8));
        uint32_t h[8];
        e2m1x8_to_f16x8(nib.x, *reinterpret_cast<uint32_t(*)[4]>(&h[0]));
        e2m1x8_to_f16x8(nib.y, *reinterpret_cast<uint32_t(*)[4]>(&h[4]));
        uint32_t outw[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t lo = f16x2_to_e4m3x2(hmul2_u32(h[2 * q], s2));
            const uint32_t hi = f16x2_to_e4m3x2(hmul2_u32(h[2 * q + 1], s2));
            outw[q] = lo | (hi << 16);
        }
        uint8_t *dst = staging + e * kStagedRowBytes;
        *reinterpret_cast<uint4 *>(dst + 16 * lane) = make_uint4(outw[0], outw[1], outw[2], outw[3]);
        *reinterpret_cast<uint16_t *>(dst + kLatent + 2 * lane) = rope;
    }
}

cudaError_t launch_stage_fp8(const uint8_t *cache, int64_t num_slots, const int32_t *indices, int32_t topk,
                             int32_t T, uint8_t *staging, cudaStream_t stream) {
    const int64_t entries = (int64_t)T * topk;
    if (entries == 0) return cudaSuccess;
    const int per_block = 8;  // warps per block
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    (void)cudaGetLastError();
    const int64_t want = (entries + per_block - 1) / per_block;
    const int64_t cap = (int64_t)sms * 8;  // 8 blocks of 8 warps per SM, each warp looping over entries
    stage_fp8_kernel<<<(unsigned)(want < cap ? want : cap), 32 * per_block, 0, stream>>>(cache, num_slots, indices,
                                                                                       entries, staging);
    return cudaGetLastError();
}

}  // namespace nvfp4mla
