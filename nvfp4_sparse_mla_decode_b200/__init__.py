"""Python binding of libnvfp4mla (NVFP4 sparse MLA decode on B200, sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libnvfp4mla.so`` behind the C ABI of ``include/nvfp4mla.h``.
PyTorch supplies device memory and the current stream.  There is no CPU or
PyTorch fallback: if the shared library is missing or the device is not a
CUDA GPU, calls raise.

Build the library with ``python -m nvfp4_sparse_mla_decode_b200.build``.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

__all__ = [
    "ROW_BYTES", "STAGED_ROW_BYTES", "LATENT", "ROPE", "MAX_TOPK", "NVFP4MLAError",
    "lib", "lib_path", "kv_append", "decode", "decode_host", "decode_paged", "decode_noalloc", "staged_decode", "staged_stage",
    "staged_attend",
    "fp8_kv_append", "fp8_decode", "indexer_scores", "indexer_topk", "sparse_indexer", "blhnc_convert",
    "copy_descriptors", "num_splits",
    "workspace_size", "staging_size", "status_string", "version",
    "DEV_TIMEOUT", "DEV_BAD_INDEX", "DEV_LAYOUT",
]

ROW_BYTES = 352
STAGED_ROW_BYTES = 576
LATENT = 512
ROPE = 64
MAX_TOPK = 2048
DEV_TIMEOUT = 1
DEV_BAD_INDEX = 2
DEV_LAYOUT = 4

_HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(_HERE, "libnvfp4mla.so")
_lib = None

_vp, _i32, _i64, _f32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t


class Tuning(ctypes.Structure):
    """nvfp4mla_tuning: fixed split count, heads per CTA, forced staged path
    (0 = the automatic choice; `reserved` must stay 0)."""
    _fields_ = [("splits", _i32), ("heads_per_cta", _i32), ("force_staged", _i32), ("reserved", _i32)]


class NVFP4MLAError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str | None = None):
        msg = "%s: %s (status %d)" % (what, status_string(status), status)
        super().__init__(msg + (": " + detail if detail else ""))
        self.status = status
        self.detail = detail


def lib() -> ctypes.CDLL:
    """Load libnvfp4mla.so from the package directory (raises if absent)."""
    global _lib
    if _lib is None:
        if not os.path.exists(lib_path):
            raise RuntimeError("libnvfp4mla.so is not built; run `python -m nvfp4_sparse_mla_decode_b200.build`")
        L = ctypes.CDLL(lib_path)
        L.nvfp4_kv_append.restype = _i32
        L.nvfp4_kv_append.argtypes = [_vp, _i64, _vp, _i64, _vp, _i32, _vp, _i64, _vp, _vp]
        L.nvfp4_sparse_mla_num_splits.restype = _i32
        L.nvfp4_sparse_mla_num_splits.argtypes = [_i32, _i32, _i32]
        L.nvfp4_sparse_mla_workspace_size.restype = _sz
        L.nvfp4_sparse_mla_workspace_size.argtypes = [_i32, _i32, _i32]
        L.nvfp4_sparse_mla_decode.restype = _i32
        L.nvfp4_sparse_mla_decode.argtypes = [_vp, _vp, _vp, _i64, _vp, _i32, _i32, _i32, _f32, _vp, _vp, _vp,
                                              _sz, _vp, _vp]
        L.nvfp4_sparse_mla_workspace_size_tuned.restype = _sz
        L.nvfp4_sparse_mla_workspace_size_tuned.argtypes = [_i32, _i32, _i32, ctypes.POINTER(Tuning)]
        L.nvfp4_sparse_mla_decode_tuned.restype = _i32
        L.nvfp4_sparse_mla_decode_tuned.argtypes = [_vp, _vp, _vp, _i64, _vp, _i32, _i32, _i32, _f32, _vp, _vp, _vp,
                                                    _sz, _vp, _sz, ctypes.POINTER(Tuning), _vp, _vp]
        L.nvfp4_sparse_mla_decode_paged.restype = _i32
        L.nvfp4_sparse_mla_decode_paged.argtypes = [_vp, _vp, _vp, _i64, _vp, _i32, _vp, _i32, _i32, _i32, _i32,
                                                    _f32, _vp, _vp, _vp, _sz, _vp, _vp]
        L.nvfp4_sparse_mla_decode_noalloc.restype = _i32
        L.nvfp4_sparse_mla_decode_noalloc.argtypes = [_vp, _vp, _vp, _i64, _vp, _i32, _i32, _i32, _f32, _vp, _vp,
                                                      _vp, _vp]
        L.nvfp4_staged_fp8_staging_size.restype = _sz
        L.nvfp4_staged_fp8_staging_size.argtypes = [_i32, _i32]
        L.nvfp4_staged_fp8_mla_decode.restype = _i32
        L.nvfp4_staged_fp8_mla_decode.argtypes = [_vp, _vp, _vp, _i64, _vp, _i32, _i32, _i32, _f32, _vp, _vp,
                                                  _vp, _sz, _vp, _sz, _vp, _vp]
        L.nvfp4_sparse_mla_decode_host.restype = _i32
        L.nvfp4_sparse_mla_decode_host.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32,
                                                   _i32, _i32, _f32, _vp, _sz, _vp, _vp]
        L.nvfp4_staged_fp8_stage.restype = _i32
        L.nvfp4_staged_fp8_stage.argtypes = [_vp, _i64, _vp, _i32, _i32, _vp, _sz, _vp]
        L.nvfp4_staged_fp8_attend.restype = _i32
        L.nvfp4_staged_fp8_attend.argtypes = [_vp, _vp, _i64, _vp, _i32, _i32, _i32, _f32, _vp, _vp, _vp, _sz, _vp,
                                              _sz, _vp, _vp]
        L.nvfp4mla_fp8_kv_append.restype = _i32
        L.nvfp4mla_fp8_kv_append.argtypes = [_vp, _i64, _vp, _i64, _vp, _i32, _vp, _i64, _vp, _vp]
        L.nvfp4mla_fp8_sparse_mla_decode.restype = _i32
        L.nvfp4mla_fp8_sparse_mla_decode.argtypes = [_vp, _vp, _vp, _i64, _vp, _i32, _i32, _i32, _f32, _vp, _vp,
                                                     _vp, _sz, _vp, _vp]
        L.nvfp4mla_indexer_workspace_size.restype = _sz
        L.nvfp4mla_indexer_workspace_size.argtypes = [_i32, _i32]
        L.nvfp4mla_indexer_score_stride.restype = _i64
        L.nvfp4mla_indexer_score_stride.argtypes = [_i32]
        L.nvfp4mla_indexer_scores.restype = _i32
        L.nvfp4mla_indexer_scores.argtypes = [_vp, _vp, _vp, _i64, _vp, _i32, _i32, _vp, _i32, _i32, _vp, _i64,
                                              _vp, _vp]
        L.nvfp4mla_indexer_topk.restype = _i32
        L.nvfp4mla_indexer_topk.argtypes = [_vp, _i64, _vp, _i32, _i32, _i32, _vp, _vp, _sz, _vp, _vp]
        L.nvfp4mla_indexer_topk_workspace_size.restype = _sz
        L.nvfp4mla_indexer_topk_workspace_size.argtypes = [_i32]
        L.nvfp4mla_sparse_indexer.restype = _i32
        L.nvfp4mla_sparse_indexer.argtypes = [_vp, _vp, _vp, _i64, _vp, _i32, _i32, _vp, _i32, _i32, _i32, _vp,
                                              _vp, _sz, _vp, _vp]
        L.nvfp4mla_blhnc_convert.restype = _i32
        L.nvfp4mla_blhnc_convert.argtypes = [_vp, _i32, _i64, _i32, _i32, _i32, _vp, _vp, _i32, _vp, _i64, _i32,
                                             _vp, _vp]
        L.nvfp4mla_copy_descriptors.restype = _i64
        L.nvfp4mla_copy_descriptors.argtypes = [_vp, _i32, _i32]
        L.nvfp4mla_selftest_wait_timeout.restype = _i32
        L.nvfp4mla_selftest_wait_timeout.argtypes = [_vp, _vp, _vp]
        L.nvfp4mla_status_string.restype = ctypes.c_char_p
        L.nvfp4mla_status_string.argtypes = [_i32]
        L.nvfp4mla_last_cuda_error.restype = _i32
        L.nvfp4mla_last_cuda_error.argtypes = []
        L.nvfp4mla_last_cuda_error_string.restype = ctypes.c_char_p
        L.nvfp4mla_last_cuda_error_string.argtypes = []
        L.nvfp4mla_version.restype = _i32
        L.nvfp4mla_version.argtypes = []
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().nvfp4mla_status_string(int(status)).decode()


def version() -> int:
    return int(lib().nvfp4mla_version())


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _need_cuda(*ts: torch.Tensor) -> torch.device:
    dev = ts[0].device
    for t in ts:
        if t.device.type != "cuda" or t.device != dev:
            raise ValueError("all tensors must live on the same CUDA device")
    return dev


def _check(status: int, what: str) -> None:
    if status != 0:
        detail = None
        if status == 4:  # NVFP4MLA_ERR_CUDA: name the CUDA error behind it
            detail = lib().nvfp4mla_last_cuda_error_string().decode()
        raise NVFP4MLAError(status, what, detail)


def num_splits(T: int, H: int, topk: int = MAX_TOPK) -> int:
    return int(lib().nvfp4_sparse_mla_num_splits(T, H, topk))


def workspace_size(T: int, H: int, topk: int = MAX_TOPK, tuning: Optional[Tuning] = None) -> int:
    if tuning is not None:
        return int(lib().nvfp4_sparse_mla_workspace_size_tuned(T, H, topk, ctypes.byref(tuning)))
    return int(lib().nvfp4_sparse_mla_workspace_size(T, H, topk))


def staging_size(T: int, topk: int = MAX_TOPK) -> int:
    return int(lib().nvfp4_staged_fp8_staging_size(T, topk))


def _append(fn, name, latent, rope, slot_mapping, cache, dev_status):
    dev = _need_cuda(latent, rope, slot_mapping, cache)
    assert latent.dtype == torch.bfloat16 and rope.dtype == torch.bfloat16
    assert slot_mapping.dtype == torch.int32 and cache.dtype == torch.uint8 and cache.is_contiguous()
    assert latent.stride(-1) == 1 and rope.stride(-1) == 1 and slot_mapping.is_contiguous()
    n = slot_mapping.numel()
    assert latent.shape[0] == n and rope.shape[0] == n
    st = fn(_ptr(latent), latent.stride(0) if n else LATENT, _ptr(rope), rope.stride(0) if n else ROPE,
            _ptr(slot_mapping), n, _ptr(cache), cache.shape[0], _ptr(dev_status), _stream(dev))
    _check(st, name)


def kv_append(latent: torch.Tensor, rope: torch.Tensor, slot_mapping: torch.Tensor, cache: torch.Tensor,
              dev_status: Optional[torch.Tensor] = None) -> None:
    """Quantize BF16 rows latent [n, >=512] / rope [n, >=64] (row strides in
    elements, unit inner stride) into ``cache`` uint8 [num_slots, 352] at
    ``slot_mapping`` int32 [n]."""
    assert cache.dim() == 2 and cache.shape[1] == ROW_BYTES
    _append(lib().nvfp4_kv_append, "nvfp4_kv_append", latent, rope, slot_mapping, cache, dev_status)


def fp8_kv_append(latent: torch.Tensor, rope: torch.Tensor, slot_mapping: torch.Tensor, cache: torch.Tensor,
                  dev_status: Optional[torch.Tensor] = None) -> None:
    """kv_append() into a cache of 576-byte E4M3 rows, uint8 [num_slots, 576]."""
    assert cache.dim() == 2 and cache.shape[1] == STAGED_ROW_BYTES
    _append(lib().nvfp4mla_fp8_kv_append, "nvfp4mla_fp8_kv_append", latent, rope, slot_mapping, cache,
            dev_status)


def _decode_args(q_nope, q_rope, cache, indices, out, lse):
    dev = _need_cuda(q_nope, q_rope, cache, indices)
    T, H = q_nope.shape[0], q_nope.shape[1]
    assert q_nope.dtype == torch.float16 and q_rope.dtype == torch.float16
    assert q_nope.shape == (T, H, LATENT) and q_rope.shape == (T, H, ROPE)
    assert q_nope.is_contiguous() and q_rope.is_contiguous()
    assert indices.dtype == torch.int32 and indices.dim() == 2 and indices.shape[0] == T and indices.is_contiguous()
    assert cache.dtype == torch.uint8 and cache.is_contiguous()
    if out is None:
        out = torch.empty(T, H, LATENT, dtype=torch.float16, device=dev)
    if lse is None:
        lse = torch.empty(T, H, dtype=torch.float32, device=dev)
    return dev, T, H, indices.shape[1], out, lse


def decode(q_nope: torch.Tensor, q_rope: torch.Tensor, cache: torch.Tensor, indices: torch.Tensor,
           sm_scale: float, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
           workspace: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None,
           num_slots: Optional[int] = None, tuning: Optional[Tuning] = None,
           staging: Optional[torch.Tensor] = None):
    """Sparse MLA decode over the NVFP4 cache; returns (out [T,H,512] f16, lse [T,H] f32).

    A caller-supplied `workspace` must start zero-filled (its first 4096
    bytes hold split counters that every completed call leaves at zero).
    `tuning` fixes the plan (nvfp4_sparse_mla_decode_tuned); with
    force_staged the staged path runs through `staging` (allocated here when
    not given)."""
    dev, T, H, topk, out, lse = _decode_args(q_nope, q_rope, cache, indices, out, lse)
    ws_need = workspace_size(T, H, topk, tuning)
    if workspace is None and ws_need:
        workspace = torch.zeros(ws_need, dtype=torch.uint8, device=dev)
    if tuning is not None:
        if tuning.force_staged and staging is None:
            staging = torch.empty(max(1, staging_size(T, topk)), dtype=torch.uint8, device=dev)
        st = lib().nvfp4_sparse_mla_decode_tuned(
            _ptr(q_nope), _ptr(q_rope), _ptr(cache), num_slots if num_slots is not None else cache.shape[0],
            _ptr(indices), topk, T, H, float(sm_scale), _ptr(out), _ptr(lse), _ptr(workspace),
            workspace.numel() * workspace.element_size() if workspace is not None else 0, _ptr(staging),
            staging.numel() * staging.element_size() if staging is not None else 0, ctypes.byref(tuning),
            _ptr(dev_status), _stream(dev))
        _check(st, "nvfp4_sparse_mla_decode_tuned")
        return out, lse
    st = lib().nvfp4_sparse_mla_decode(_ptr(q_nope), _ptr(q_rope), _ptr(cache),
                                       num_slots if num_slots is not None else cache.shape[0], _ptr(indices),
                                       topk, T, H, float(sm_scale), _ptr(out), _ptr(lse), _ptr(workspace),
                                       workspace.numel() * workspace.element_size() if workspace is not None else 0,
                                       _ptr(dev_status), _stream(dev))
    _check(st, "nvfp4_sparse_mla_decode")
    return out, lse


def decode_host(h_q_nope: torch.Tensor, h_q_rope: torch.Tensor, h_indices: torch.Tensor, h_out: torch.Tensor,
                h_lse: torch.Tensor, d_q_nope: torch.Tensor, d_q_rope: torch.Tensor, d_indices: torch.Tensor,
                d_out: torch.Tensor, d_lse: torch.Tensor, cache: torch.Tensor, sm_scale: float,
                workspace: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> None:
    """decode() with inputs and outputs in (pinned) host tensors; the library
    copies them to and from the given device tensors on `stream` around the
    kernel.  Host outputs are valid once the stream has been synchronized."""
    for h in (h_q_nope, h_q_rope, h_indices, h_out, h_lse):
        assert h.device.type == "cpu" and h.is_contiguous()
    dev, T, H, topk, d_out, d_lse = _decode_args(d_q_nope, d_q_rope, cache, d_indices, d_out, d_lse)
    assert h_q_nope.shape == d_q_nope.shape and h_q_rope.shape == d_q_rope.shape
    assert h_indices.shape == d_indices.shape and h_out.shape == d_out.shape and h_lse.shape == d_lse.shape
    ws_need = workspace_size(T, H, topk)
    if workspace is None and ws_need:
        workspace = torch.zeros(ws_need, dtype=torch.uint8, device=dev)
    s = stream.cuda_stream if stream is not None else _stream(dev)
    st = lib().nvfp4_sparse_mla_decode_host(
        h_q_nope.data_ptr(), h_q_rope.data_ptr(), h_indices.data_ptr(), h_out.data_ptr(), h_lse.data_ptr(),
        _ptr(d_q_nope), _ptr(d_q_rope), _ptr(d_indices), _ptr(d_out), _ptr(d_lse), _ptr(cache), cache.shape[0],
        topk, T, H, float(sm_scale), _ptr(workspace),
        workspace.numel() * workspace.element_size() if workspace is not None else 0, _ptr(dev_status), s)
    _check(st, "nvfp4_sparse_mla_decode_host")


def decode_paged(q_nope: torch.Tensor, q_rope: torch.Tensor, cache: torch.Tensor, positions: torch.Tensor,
                 block_table: torch.Tensor, page_size: int, sm_scale: float, out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 dev_status: Optional[torch.Tensor] = None):
    """decode() over request-local positions translated through block_table
    ([T, stride] int32 page ids) inside the launch."""
    dev, T, H, topk, out, lse = _decode_args(q_nope, q_rope, cache, positions, out, lse)
    assert block_table.dtype == torch.int32 and block_table.dim() == 2 and block_table.is_contiguous()
    assert block_table.shape[0] == T
    ws_need = workspace_size(T, H, topk)
    if workspace is None and ws_need:
        workspace = torch.zeros(ws_need, dtype=torch.uint8, device=dev)
    st = lib().nvfp4_sparse_mla_decode_paged(_ptr(q_nope), _ptr(q_rope), _ptr(cache), cache.shape[0],
                                             _ptr(positions), topk, _ptr(block_table), block_table.shape[1],
                                             int(page_size), T, H, float(sm_scale), _ptr(out), _ptr(lse),
                                             _ptr(workspace),
                                             workspace.numel() * workspace.element_size() if workspace is not None
                                             else 0, _ptr(dev_status), _stream(dev))
    _check(st, "nvfp4_sparse_mla_decode_paged")
    return out, lse


def decode_noalloc(q_nope: torch.Tensor, q_rope: torch.Tensor, cache: torch.Tensor, indices: torch.Tensor,
                   sm_scale: float, out: torch.Tensor, lse: torch.Tensor,
                   dev_status: Optional[torch.Tensor] = None, num_slots: Optional[int] = None):
    """decode() without a workspace: the library's static per-device scratch
    is used, so calls that may overlap in time must not use it.  `out` and
    `lse` are caller-provided so nothing is allocated on this path."""
    dev, T, H, topk, out, lse = _decode_args(q_nope, q_rope, cache, indices, out, lse)
    st = lib().nvfp4_sparse_mla_decode_noalloc(_ptr(q_nope), _ptr(q_rope), _ptr(cache),
                                               num_slots if num_slots is not None else cache.shape[0],
                                               _ptr(indices), topk, T, H, float(sm_scale), _ptr(out), _ptr(lse),
                                               _ptr(dev_status), _stream(dev))
    _check(st, "nvfp4_sparse_mla_decode_noalloc")
    return out, lse


def staged_decode(q_nope: torch.Tensor, q_rope: torch.Tensor, cache: torch.Tensor, indices: torch.Tensor,
                  sm_scale: float, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                  staging: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  dev_status: Optional[torch.Tensor] = None):
    """The staged FP8 comparison path; returns (out, lse)."""
    dev, T, H, topk, out, lse = _decode_args(q_nope, q_rope, cache, indices, out, lse)
    if staging is None:
        staging = torch.empty(max(1, staging_size(T, topk)), dtype=torch.uint8, device=dev)
    ws_need = workspace_size(T, H, topk)
    if workspace is None and ws_need:
        workspace = torch.zeros(ws_need, dtype=torch.uint8, device=dev)
    st = lib().nvfp4_staged_fp8_mla_decode(_ptr(q_nope), _ptr(q_rope), _ptr(cache), cache.shape[0], _ptr(indices),
                                           topk, T, H, float(sm_scale), _ptr(out), _ptr(lse), _ptr(staging),
                                           staging.numel(), _ptr(workspace),
                                           workspace.numel() if workspace is not None else 0,
                                           _ptr(dev_status), _stream(dev))
    _check(st, "nvfp4_staged_fp8_mla_decode")
    return out, lse


def staged_stage(cache: torch.Tensor, indices: torch.Tensor, staging: torch.Tensor) -> None:
    """Step 1 of the staged path: E4M3 rows of the valid entries into staging."""
    assert indices.dtype == torch.int32 and indices.dim() == 2 and indices.is_contiguous()
    T, topk = indices.shape
    st = lib().nvfp4_staged_fp8_stage(_ptr(cache), cache.shape[0], _ptr(indices), topk, T, _ptr(staging),
                                      staging.numel(), _stream(cache.device))
    _check(st, "nvfp4_staged_fp8_stage")


def staged_attend(q_nope: torch.Tensor, q_rope: torch.Tensor, num_slots: int, indices: torch.Tensor,
                  staging: torch.Tensor, sm_scale: float, out: Optional[torch.Tensor] = None,
                  lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                  dev_status: Optional[torch.Tensor] = None):
    """Step 2 of the staged path: attention over the staged E4M3 rows."""
    dev, T, H, topk, out, lse = _decode_args(q_nope, q_rope, staging, indices, out, lse)
    ws_need = workspace_size(T, H, topk)
    if workspace is None and ws_need:
        workspace = torch.zeros(ws_need, dtype=torch.uint8, device=dev)
    st = lib().nvfp4_staged_fp8_attend(_ptr(q_nope), _ptr(q_rope), num_slots, _ptr(indices), topk, T, H,
                                       float(sm_scale), _ptr(out), _ptr(lse), _ptr(staging), staging.numel(),
                                       _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                       _ptr(dev_status), _stream(dev))
    _check(st, "nvfp4_staged_fp8_attend")
    return out, lse


def fp8_decode(q_nope: torch.Tensor, q_rope: torch.Tensor, fp8_cache: torch.Tensor, indices: torch.Tensor,
               sm_scale: float, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
               workspace: Optional[torch.Tensor] = None, dev_status: Optional[torch.Tensor] = None):
    """decode() over a cache of 576-byte E4M3 rows (uint8 [num_slots, 576])."""
    assert fp8_cache.dim() == 2 and fp8_cache.shape[1] == STAGED_ROW_BYTES
    dev, T, H, topk, out, lse = _decode_args(q_nope, q_rope, fp8_cache, indices, out, lse)
    ws_need = workspace_size(T, H, topk)
    if workspace is None and ws_need:
        workspace = torch.zeros(ws_need, dtype=torch.uint8, device=dev)
    st = lib().nvfp4mla_fp8_sparse_mla_decode(_ptr(q_nope), _ptr(q_rope), _ptr(fp8_cache), fp8_cache.shape[0],
                                              _ptr(indices), topk, T, H, float(sm_scale), _ptr(out), _ptr(lse),
                                              _ptr(workspace),
                                              workspace.numel() * workspace.element_size()
                                              if workspace is not None else 0, _ptr(dev_status), _stream(dev))
    _check(st, "nvfp4mla_fp8_sparse_mla_decode")
    return out, lse


def _indexer_inputs(q, w, keys, block_table, ctx_lens):
    dev = _need_cuda(q, w, keys, block_table, ctx_lens)
    T = q.shape[0]
    assert q.dtype == torch.uint8 and q.shape == (T, 64, 128) and q.is_contiguous()
    assert w.dtype == torch.float32 and w.shape == (T, 64) and w.is_contiguous()
    assert keys.dtype == torch.uint8 and keys.dim() == 2 and keys.shape[1] == 128 and keys.is_contiguous()
    assert block_table.dtype == torch.int32 and block_table.dim() == 2 and block_table.shape[0] == T
    assert block_table.is_contiguous()
    assert ctx_lens.dtype == torch.int32 and ctx_lens.shape == (T,) and ctx_lens.is_contiguous()
    return dev, T


def indexer_score_stride(max_ctx: int) -> int:
    return int(lib().nvfp4mla_indexer_score_stride(max_ctx))


def indexer_scores(q: torch.Tensor, w: torch.Tensor, keys: torch.Tensor, block_table: torch.Tensor,
                   page_size: int, ctx_lens: torch.Tensor, max_ctx: int, scores: Optional[torch.Tensor] = None,
                   dev_status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Indexer scores float32 [T, stride] (positions >= ctx_lens[t] untouched).
    q uint8 [T,64,128] E4M3, w float32 [T,64], keys uint8 [num_slots,128]
    E4M3, block_table int32 [T, width], ctx_lens int32 [T]."""
    dev, T = _indexer_inputs(q, w, keys, block_table, ctx_lens)
    if scores is None:
        scores = torch.empty(T, max(1, indexer_score_stride(max_ctx)), dtype=torch.float32, device=dev)
    assert scores.dtype == torch.float32 and scores.dim() == 2 and scores.stride(1) == 1
    st = lib().nvfp4mla_indexer_scores(_ptr(q), _ptr(w), _ptr(keys), keys.shape[0], _ptr(block_table),
                                       block_table.shape[1], int(page_size), _ptr(ctx_lens), int(max_ctx), T,
                                       _ptr(scores), scores.stride(0), _ptr(dev_status), _stream(dev))
    _check(st, "nvfp4mla_indexer_scores")
    return scores


def indexer_topk(scores: torch.Tensor, ctx_lens: torch.Tensor, max_ctx: int, topk: int = MAX_TOPK,
                 positions: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 dev_status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Top-k positions int32 [T, topk] of scores float32 [T, stride].  A
    caller-supplied `workspace` must start zero-filled (completed calls leave
    its counters at zero)."""
    dev = _need_cuda(scores, ctx_lens)
    T = ctx_lens.shape[0]
    assert scores.dtype == torch.float32 and scores.dim() == 2 and scores.stride(1) == 1 and scores.shape[0] == T
    assert ctx_lens.dtype == torch.int32 and ctx_lens.is_contiguous()
    if positions is None:
        positions = torch.empty(T, topk, dtype=torch.int32, device=dev)
    need = int(lib().nvfp4mla_indexer_topk_workspace_size(T))
    if workspace is None and need:
        workspace = torch.zeros(need, dtype=torch.uint8, device=dev)
    st = lib().nvfp4mla_indexer_topk(_ptr(scores), scores.stride(0), _ptr(ctx_lens), int(max_ctx), T, int(topk),
                                     _ptr(positions), _ptr(workspace),
                                     workspace.numel() * workspace.element_size() if workspace is not None else 0,
                                     _ptr(dev_status), _stream(dev))
    _check(st, "nvfp4mla_indexer_topk")
    return positions


def sparse_indexer(q: torch.Tensor, w: torch.Tensor, keys: torch.Tensor, block_table: torch.Tensor,
                   page_size: int, ctx_lens: torch.Tensor, max_ctx: int, topk: int = MAX_TOPK,
                   positions: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                   dev_status: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Scores and selection in one call: request-local positions int32
    [T, topk] (increasing, -1 padded), the input of decode_paged."""
    dev, T = _indexer_inputs(q, w, keys, block_table, ctx_lens)
    if positions is None:
        positions = torch.empty(T, topk, dtype=torch.int32, device=dev)
    need = int(lib().nvfp4mla_indexer_workspace_size(T, int(max_ctx)))
    if workspace is None:
        workspace = torch.zeros(max(256, need), dtype=torch.uint8, device=dev)
    st = lib().nvfp4mla_sparse_indexer(_ptr(q), _ptr(w), _ptr(keys), keys.shape[0], _ptr(block_table),
                                       block_table.shape[1], int(page_size), _ptr(ctx_lens), int(max_ctx), T,
                                       int(topk), _ptr(positions), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _ptr(dev_status),
                                       _stream(dev))
    _check(st, "nvfp4mla_sparse_indexer")
    return positions


def blhnc_convert(layer_caches, block_ids: torch.Tensor, new_block_ids: torch.Tensor, blhnc: torch.Tensor,
                  sub: int, to_blhnc: bool = True, layer_ptrs: Optional[torch.Tensor] = None,
                  dev_status: Optional[torch.Tensor] = None) -> None:
    """Per-layer caches (list of uint8 [num_blocks, N, C] tensors, equal
    shapes) <-> block-major cache uint8 [num_new, L, N // sub, C] for the
    request's blocks.  `layer_ptrs` (int64 device tensor of the caches'
    addresses) may be passed to avoid rebuilding it per call."""
    dev = _need_cuda(block_ids, new_block_ids, blhnc, *layer_caches)
    L = len(layer_caches)
    nblk, N, C = layer_caches[0].shape
    assert all(c.shape == (nblk, N, C) and c.dtype == torch.uint8 and c.is_contiguous() for c in layer_caches)
    assert blhnc.dtype == torch.uint8 and blhnc.is_contiguous() and blhnc.shape[1:] == (L, N // sub, C)
    assert block_ids.dtype == torch.int32 and new_block_ids.dtype == torch.int32
    assert block_ids.is_contiguous() and new_block_ids.is_contiguous()
    assert new_block_ids.numel() == block_ids.numel() * sub
    if layer_ptrs is None:
        layer_ptrs = torch.tensor([c.data_ptr() for c in layer_caches], dtype=torch.int64, device=dev)
    st = lib().nvfp4mla_blhnc_convert(_ptr(layer_ptrs), L, nblk, N, C, int(sub), _ptr(block_ids),
                                      _ptr(new_block_ids), block_ids.numel(), _ptr(blhnc), blhnc.shape[0],
                                      1 if to_blhnc else 0, _ptr(dev_status), _stream(dev))
    _check(st, "nvfp4mla_blhnc_convert")


def copy_descriptors(ids, layers: int = 1) -> int:
    """Host-side descriptor model: layers x runs of consecutive ids."""
    import numpy as np
    a = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
    r = lib().nvfp4mla_copy_descriptors(a.ctypes.data if a.size else None, a.size, int(layers))
    if r < 0:
        raise ValueError("bad arguments")
    return int(r)


def selftest_wait_timeout(device="cuda") -> int:
    """Run the bounded-wait self-test; returns the device status word it set
    (NVFP4MLA_DEV_TIMEOUT when the waits ended as designed)."""
    zero = torch.zeros(1, dtype=torch.int32, device=device)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    _check(lib().nvfp4mla_selftest_wait_timeout(_ptr(zero), _ptr(status), _stream(zero.device)),
           "nvfp4mla_selftest_wait_timeout")
    torch.cuda.synchronize(zero.device)
    return int(status.item())


def default_sm_scale() -> float:
    return 1.0 / math.sqrt(LATENT + ROPE)
