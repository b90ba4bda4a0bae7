"""Sparse indexer oracle: scores over each request's context, then the
top-k position list.  Test infrastructure only -- the CUDA library never
imports this module and shares no code with it.

Page "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
section "Four-bit caches make room": a sparse indexer picks the cache rows
that each query token's attention reads, and the list it hands over has
2,048 positions.  The page gives neither the indexer's scoring function nor
its tie rule.  The readings taken here:

* scoring: the lightning-indexer form published with DeepSeek sparse
  attention,
      I[t, p] = sum_h w[t, h] * max(0, sum_d q[t, h, d] * k[slot(t, p), d])
  with 64 indexer heads of 128 dims, q and k stored as E4M3 bytes, w FP32;
  slot(t, p) = table[t][p // page] * page + p % page (the request's block
  table), for context positions 0 <= p < ctx[t];
* selection: the min(topk, ctx[t]) positions with the largest scores, equal
  scores taken in increasing position order; the list holds them in
  increasing position order and is padded with -1.  Scores compare as
  numbers, so -0 equals +0.

Everything is FP64: E4M3 values and their products are exact, and the sums
round far below the GPU's FP32 accumulation.
"""
from __future__ import annotations

import numpy as np

from . import oracle as _codec

INDEX_HEADS = 64
INDEX_DIM = 128

__all__ = ["INDEX_HEADS", "INDEX_DIM", "e4m3_table", "context_slots", "indexer_scores",
           "topk_positions", "sparse_indexer"]

_TABLE = None


def e4m3_table() -> np.ndarray:
    """float64 value of every E4M3 byte (NaN for the two NaN codes), from the
    codec's own decoder."""
    global _TABLE
    if _TABLE is None:
        _TABLE = np.array([_codec.e4m3_value(c) for c in range(256)], dtype=np.float64)
    return _TABLE


def context_slots(table_row: np.ndarray, ctx: int, page_size: int) -> np.ndarray:
    """Slot of every context position 0..ctx-1 through one request's block
    table (int64; -1 where the table entry is negative)."""
    p = np.arange(ctx, dtype=np.int64)
    blk = np.asarray(table_row, dtype=np.int64)[p // page_size]
    return np.where(blk >= 0, blk * page_size + p % page_size, -1)


def indexer_scores(q_codes: np.ndarray, w: np.ndarray, key_codes, block_table: np.ndarray,
                   ctx_lens, page_size: int, tokens=None, magnitude: bool = False):
    """FP64 indexer scores.

    q_codes uint8 [T, 64, 128] (E4M3 bytes), w float32 [T, 64], key_codes:
    uint8 [num_slots, 128] or a callable slots -> uint8 [n, 128] (rows of the
    key cache), block_table int32 [T, width], ctx_lens [T].  Returns a list
    (one entry per token in ``tokens``) of float64 [ctx[t]] score vectors;
    with ``magnitude`` also the list of sum_h |w_h| * sum_d |q_hd * k_d|, the
    scale of the rounding error of any evaluation of the same sums."""
    lut = e4m3_table()
    tokens = range(q_codes.shape[0]) if tokens is None else tokens
    rows = key_codes if callable(key_codes) else (lambda s: key_codes[s])
    scores, mags = [], []
    for t in tokens:
        ctx = int(ctx_lens[t])
        slots = context_slots(block_table[t], ctx, page_size)
        assert np.all(slots >= 0), "context position without a page"
        K = lut[np.asarray(rows(slots), dtype=np.uint8)]            # [ctx, 128]
        Q = lut[np.asarray(q_codes[t], dtype=np.uint8)]              # [64, 128]
        wt = np.asarray(w[t], dtype=np.float32).astype(np.float64)   # [64]
        S = K @ Q.T                                                  # [ctx, 64]
        scores.append(np.maximum(S, 0.0) @ wt)
        if magnitude:
            mags.append((np.abs(K) @ np.abs(Q).T) @ np.abs(wt))
    return (scores, mags) if magnitude else scores


def topk_positions(scores, topk: int) -> np.ndarray:
    """Selection step: scores is a list of per-token score vectors (length =
    that token's context).  Returns int32 [T, topk]: the chosen positions in
    increasing order, then -1."""
    out = np.full((len(scores), topk), -1, dtype=np.int32)
    for i, s in enumerate(scores):
        s = np.asarray(s, dtype=np.float64)
        n = s.shape[0]
        if n <= topk:
            out[i, :n] = np.arange(n, dtype=np.int32)
            continue
        pos = np.arange(n)
        order = np.lexsort((pos, -s))      # by score descending, then position
        out[i] = np.sort(order[:topk]).astype(np.int32)
    return out


def sparse_indexer(q_codes, w, key_codes, block_table, ctx_lens, page_size: int, topk: int, tokens=None):
    """Scores then selection; returns (positions int32 [len(tokens), topk],
    scores list)."""
    sc = indexer_scores(q_codes, w, key_codes, block_table, ctx_lens, page_size, tokens)
    return topk_positions(sc, topk), sc
