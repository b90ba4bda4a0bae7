"""Fill a paged NVFP4 cache on the GPU from a synthetic workload, through
the library's own append kernel (``nvfp4_kv_append``)."""
from __future__ import annotations

import torch

from . import ROW_BYTES, kv_append
from .synth import Workload


def build_cache(w: Workload, dev_status=None) -> torch.Tensor:
    """[num_slots, 352] uint8 cache on the current CUDA device holding every
    slot's row of ``w`` (base content, then any appended rows)."""
    cache = torch.zeros(w.num_slots, ROW_BYTES, dtype=torch.uint8, device="cuda")
    for lo, lat, rope in w.rows.chunks():
        slots = torch.arange(lo, lo + lat.shape[0], dtype=torch.int32, device="cuda")
        kv_append(lat, rope, slots, cache, dev_status)
        del lat, rope
    if w.new_slots is not None:
        kv_append(w.new_lat, w.new_rope, w.new_slots, cache, dev_status)
    return cache
