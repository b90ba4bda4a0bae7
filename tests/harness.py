"""Shared helpers for the GPU parity tests and the benchmark's checks.

Builds caches through the product path (``kv_append``) from the seeded
generators, and builds the oracle's inputs independently: the oracle gets the
same BF16 source rows, quantizes them itself, and never sees a byte produced
by the CUDA library.
"""
from __future__ import annotations

import numpy as np
import torch

import nvfp4_sparse_mla_decode_b200 as nv
from nvfp4_sparse_mla_decode_b200 import synth


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


from nvfp4_sparse_mla_decode_b200.cache import build_cache, build_fp8_cache  # noqa: E402,F401


def oracle_inputs(w: synth.Workload, tokens, fp8_rows=False):
    """Compact oracle problem for the given tokens: oracle-quantized rows of
    every valid slot they reference (NVFP4, or 576-byte E4M3 rows with
    fp8_rows) and their lists remapped onto them."""
    import oracle
    tokens = list(tokens)
    idx = w.indices[tokens].cpu().numpy().astype(np.int64)
    valid = (idx >= 0) & (idx < w.num_slots)
    slots = np.unique(idx[valid])
    lat, rope = w.source_rows(torch.from_numpy(slots).to(w.indices.device))
    quantize = oracle.quantize_fp8_rows if fp8_rows else oracle.quantize_rows
    rows = quantize(bf16_bits(lat), bf16_bits(rope))
    pos = np.searchsorted(slots, np.where(valid, idx, 0))
    remap = np.where(valid, pos, -1).astype(np.int32)
    qn = w.q_nope[tokens].cpu().numpy()
    qr = w.q_rope[tokens].cpu().numpy()
    return qn, qr, rows, remap, slots


def oracle_decode(w: synth.Workload, tokens, staged=False, fp8_rows=False):
    import oracle
    qn, qr, rows, remap, _ = oracle_inputs(w, tokens, fp8_rows=fp8_rows)
    return oracle.sparse_mla(qn, qr, rows, remap, w.sm_scale, staged=staged, fp8_rows=fp8_rows)


def check_close(out: torch.Tensor, lse: torch.Tensor, ref_out: np.ndarray, ref_lse: np.ndarray,
                rel=2e-3, abs_=1e-4, lse_tol=1e-3):
    """Per (token, head): max|out-ref| <= rel*max|ref| + abs_, |lse-ref| <= lse_tol
    (both -inf for an empty list).  Returns the worst ratios for reporting."""
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.float().cpu().numpy().astype(np.float64)
    err = np.abs(o - ref_out).max(axis=-1)
    bound = rel * np.abs(ref_out).max(axis=-1) + abs_
    assert np.all(np.isfinite(o)), "non-finite output"
    worst = float((err / bound).max())
    assert np.all(err <= bound), "out mismatch: worst err/bound %.3f at %s" % (
        worst, np.unravel_index(np.argmax(err / bound), err.shape))
    both_inf = np.isneginf(l) & np.isneginf(ref_lse)
    with np.errstate(invalid="ignore"):
        lerr = np.where(both_inf, 0.0, np.abs(l - ref_lse))
    assert not np.any(np.isnan(lerr)), "lse: one side -inf, the other finite" 
    assert np.all(lerr <= lse_tol), "lse mismatch: max %.3g" % np.nanmax(lerr)
    return worst, float(lerr.max())


def translate(positions: np.ndarray, table: np.ndarray, page: int, num_slots: int) -> np.ndarray:
    """Plain definition: slot = table[t, pos // page] * page + pos % page;
    -1, out-of-range positions and missing pages give -1."""
    T, K = positions.shape
    out = np.full((T, K), -1, dtype=np.int64)
    for t in range(T):
        for j in range(K):
            p = int(positions[t, j])
            if p < 0 or p >= table.shape[1] * page:
                continue
            blk = int(table[t, p // page])
            if blk < 0:
                continue
            slot = blk * page + p % page
            if slot < num_slots:
                out[t, j] = slot
    return out
