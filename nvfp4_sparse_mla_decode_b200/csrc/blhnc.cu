// blhnc.cu -- conversion between per-layer paged caches and the block-major
// multi-layer layout (BLHNC).
//
// Page "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
// section "Fewer copies unlock NVLink": moving a request's KV layer by layer
// took tens of thousands of small copies; a block-major layout that keeps
// every layer of a block together, with blocks a sixteenth of the earlier
// size, cut the copy descriptors of a transfer about tenfold.  Layout used
// here (the page gives none):
//   per-layer caches   layer l: [num_blocks, N, C] bytes
//   block-major cache  [num_new_blocks, L, N / sub, C] bytes
// and positions j * N/sub .. (j+1) * N/sub - 1 of the request's i-th block
// b_i, every layer l, are block-major block d[i * sub + j], layer slot l.
//
// Each (i, j, l) is one contiguous run of N/sub * C bytes on both sides, so
// the conversion is a batch of equal-sized copies at computed addresses:
// one warp per run, 16-byte loads and stores, four in flight per lane.  It
// is HBM-bound: every byte is read once and written once.
#include <cuda_runtime.h>

#include "common.cuh"
#include "kernels.h"

namespace nvfp4mla {

struct BlhncArgs {
    const uint64_t *layer_ptrs;  // [L] device addresses of the per-layer caches
    int L;
    int64_t num_blocks;
    int N, C, sub;
    const int32_t *block_ids;  // [nb]
    const int32_t *new_ids;    // [nb * sub]
    int nb;
    uint8_t *blhnc;  // [num_new, L, N / sub, C]
    int64_t num_new;
    bool to_blhnc;
    int32_t *dev_status;
};

__global__ void __launch_bounds__(256) blhnc_convert_kernel(const BlhncArgs a) {
    const int lane = threadIdx.x & 31;
    const int64_t nruns = (int64_t)a.nb * a.sub * a.L;
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    const int n = a.N / a.sub;
    const int64_t run_bytes = (int64_t)n * a.C;
    const int nvec = (int)(run_bytes >> 4);
    bool bad = false;
    for (int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < nruns; r += warps) {
        // run r = ((i * sub + j) * L + l): consecutive warps take the layers
        // of one block-major block, which are adjacent in the destination
        const int l = (int)(r % a.L);
        const int64_t ij = r / a.L;
        const int j = (int)(ij % a.sub);
        const int i = (int)(ij / a.sub);
        const int32_t b = __ldg(a.block_ids + i);
        const int32_t d = __ldg(a.new_ids + ij);
        const uint64_t base = __ldg(a.layer_ptrs + l);
        if (b < 0 || b >= a.num_blocks || d < 0 || d >= a.num_new || (base & 15u)) {
            bad = true;
            continue;
        }
        uint8_t *layer = reinterpret_cast<uint8_t *>(base) + ((int64_t)b * a.N + (int64_t)j * n) * a.C;
        uint8_t *blk = a.blhnc + ((int64_t)d * a.L + l) * run_bytes;
        const uint4 *src = reinterpret_cast<const uint4 *>(a.to_blhnc ? layer : blk);
        uint4 *dst = reinterpret_cast<uint4 *>(a.to_blhnc ? blk : layer);
        for (int k = lane; k < nvec; k += 128) {
            uint4 v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (k + 32 * u < nvec) v[u] = __ldcs(src + k + 32 * u);
#pragma unroll
            for (int u = 0; u < 4; ++u)
                if (k + 32 * u < nvec) __stcs(dst + k + 32 * u, v[u]);
        }
    }
    if (bad && a.dev_status) atomicOr(a.dev_status, NVFP4MLA_DEV_BAD_INDEX);
}

cudaError_t launch_blhnc_convert(const uint64_t *layer_ptrs, int32_t layers, int64_t num_blocks, int32_t block_size,
                                 int32_t row_bytes, int32_t sub, const int32_t *block_ids, const int32_t *new_ids,
                                 int32_t nb, uint8_t *blhnc, int64_t num_new, bool to_blhnc, int32_t *dev_status,
                                 cudaStream_t stream) {
    const int64_t nruns = (int64_t)nb * sub * layers;
    if (nruns == 0) return cudaSuccess;
    BlhncArgs a;
    a.layer_ptrs = layer_ptrs;
    a.L = layers;
    a.num_blocks = num_blocks;
    a.N = block_size;
    a.C = row_bytes;
    a.sub = sub;
    a.block_ids = block_ids;
    a.new_ids = new_ids;
    a.nb = nb;
    a.blhnc = blhnc;
    a.num_new = num_new;
    a.to_blhnc = to_blhnc;
    a.dev_status = dev_status;
    // 8 warps per CTA, 8 CTAs per SM, grid-stride over the runs
    const int64_t want = (nruns + 7) / 8;
    const int64_t cap = (int64_t)current_device_sm_count() * 8;
    const unsigned blocks = (unsigned)(want < cap ? want : cap);
    blhnc_convert_kernel<<<blocks, 256, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace nvfp4mla
