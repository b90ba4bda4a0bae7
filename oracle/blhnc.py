"""Block-major multi-layer layout oracle -- test infrastructure only; the
CUDA library never imports this module and shares no code with it.

Page "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
section "Fewer copies unlock NVLink": moving a long request's KV between
workers layer by layer took tens of thousands of small copies; the
block-major layout called BLHNC keeps the data of every layer of a block
next to each other, with blocks a sixteenth of the earlier size, and cut the
copy descriptors of a transfer by about ten times.  The page gives no byte
layout.  The readings taken here:

* the usual layout has one paged cache per layer, [num_blocks, N, C]
  (N positions per block, C bytes per position, e.g. the 352-byte row);
* the block-major cache is [num_new_blocks, L, N / sub, C] (H, the head
  dimension of the name, is 1 for a latent cache): its blocks hold N / sub
  positions of every layer;
* converting a request: positions j * N/sub .. (j+1) * N/sub - 1 of its
  i-th block b_i, every layer, go to block-major block d[i * sub + j]
  (d: the request's new block ids, in order);
* a copy descriptor covers one run of contiguous bytes: per layer, one per
  run of consecutive block ids under the usual layout; one per run of
  consecutive new-block ids under the block-major layout, all layers at once.
"""
from __future__ import annotations

import numpy as np

__all__ = ["convert", "convert_back", "runs", "descriptors_layer_major", "descriptors_block_major"]


def convert(layer_caches, block_ids, sub: int, new_ids, num_new_blocks: int, fill: int = 0) -> np.ndarray:
    """layer_caches: L arrays uint8 [num_blocks, N, C]; block_ids: the
    request's nb blocks; new_ids: nb * sub block-major ids.  Returns the
    block-major cache uint8 [num_new_blocks, L, N // sub, C], `fill`
    elsewhere."""
    L = len(layer_caches)
    _, N, C = layer_caches[0].shape
    assert N % sub == 0
    n = N // sub
    out = np.full((num_new_blocks, L, n, C), fill, dtype=np.uint8)
    for i, b in enumerate(np.asarray(block_ids, dtype=np.int64)):
        for j in range(sub):
            d = int(new_ids[i * sub + j])
            for l in range(L):
                out[d, l] = layer_caches[l][b, j * n:(j + 1) * n]
    return out


def convert_back(blhnc: np.ndarray, layer_caches, block_ids, sub: int, new_ids):
    """The inverse: the request's blocks of every layer cache from the
    block-major cache (returns new arrays; the inputs are not modified)."""
    caches = [c.copy() for c in layer_caches]
    n = blhnc.shape[2]
    for i, b in enumerate(np.asarray(block_ids, dtype=np.int64)):
        for j in range(sub):
            d = int(new_ids[i * sub + j])
            for l in range(len(caches)):
                caches[l][b, j * n:(j + 1) * n] = blhnc[d, l]
    return caches


def runs(ids) -> int:
    """Number of maximal runs of consecutive increasing ids (id, id+1, ...)."""
    ids = np.asarray(ids, dtype=np.int64)
    if ids.size == 0:
        return 0
    return 1 + int(np.count_nonzero(ids[1:] != ids[:-1] + 1))


def descriptors_layer_major(block_ids, layers: int) -> int:
    """Copy descriptors of moving the request's blocks with one paged cache
    per layer: each layer moves each run of consecutive blocks once."""
    return layers * runs(block_ids)


def descriptors_block_major(new_ids) -> int:
    """Copy descriptors of moving the request's block-major blocks: one per
    run of consecutive new ids, all layers at once."""
    return runs(new_ids)
