"""Fill a paged cache on the GPU from a synthetic workload, through the
library's own append kernels (``nvfp4_kv_append`` for 352-byte NVFP4 rows,
``nvfp4mla_fp8_kv_append`` for 576-byte E4M3 rows)."""
from __future__ import annotations

import torch

from . import ROW_BYTES, STAGED_ROW_BYTES, fp8_kv_append, kv_append
from .synth import Workload


def _fill(w: Workload, row_bytes: int, append, dev_status) -> torch.Tensor:
    cache = torch.zeros(w.num_slots, row_bytes, dtype=torch.uint8, device="cuda")
    for lo, lat, rope in w.rows.chunks():
        slots = torch.arange(lo, lo + lat.shape[0], dtype=torch.int32, device="cuda")
        append(lat, rope, slots, cache, dev_status)
        del lat, rope
    if w.new_slots is not None:
        append(w.new_lat, w.new_rope, w.new_slots, cache, dev_status)
    return cache


def build_cache(w: Workload, dev_status=None) -> torch.Tensor:
    """[num_slots, 352] uint8 cache on the current CUDA device holding every
    slot's row of ``w`` (base content, then any appended rows)."""
    return _fill(w, ROW_BYTES, kv_append, dev_status)


def build_fp8_cache(w: Workload, dev_status=None) -> torch.Tensor:
    """The same rows as 576-byte E4M3 rows: [num_slots, 576] uint8."""
    return _fill(w, STAGED_ROW_BYTES, fp8_kv_append, dev_status)
