"""ctypes wrapper around ``nvfp4_oracle.c`` (plain C, FP64 attention).

Test infrastructure only: the CUDA product path never imports this module.
See ``nvfp4_oracle.c`` for the definitions each function follows and the
pages' passages they cite (page "Prime Intellect Launches Prime Inference,
Serving 600B Tokens Daily", section "Four-bit caches make room").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

__all__ = [
    "build_oracle", "lib", "ROW_BYTES", "STAGED_ROW_BYTES",
    "e2m1_value", "e4m3_value", "e2m1_encode", "e4m3_encode",
    "f16_to_double", "quantize_group", "quantize_rows", "quantize_fp8_rows", "dequant_rows",
    "stage_rows", "sparse_mla", "max_threads",
]

ROW_BYTES = 352
STAGED_ROW_BYTES = 576
_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nvfp4_oracle.c")
_SO = os.path.join(_HERE, "libnvfp4_oracle.so")
_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE arithmetic, OpenMP) if stale."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp.%d" % os.getpid()
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
            "-ffp-contract=off", "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm",
        ])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build_oracle())
        L = _lib
        L.oracle_e2m1_value.restype = ctypes.c_double
        L.oracle_e2m1_value.argtypes = [ctypes.c_int]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e4m3_value.argtypes = [ctypes.c_int]
        L.oracle_e2m1_encode.restype = ctypes.c_int
        L.oracle_e2m1_encode.argtypes = [ctypes.c_float]
        L.oracle_e4m3_encode.restype = ctypes.c_int
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_f16_to_double.restype = ctypes.c_double
        L.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
        L.oracle_quantize_group.restype = None
        L.oracle_quantize_group.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_quantize_rows.restype = None
        L.oracle_quantize_rows.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                           ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        L.oracle_quantize_fp8_rows.restype = None
        L.oracle_quantize_fp8_rows.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                               ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p]
        L.oracle_dequant_row.restype = None
        L.oracle_dequant_row.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_stage_row.restype = None
        L.oracle_stage_row.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_sparse_mla.restype = ctypes.c_int
        L.oracle_sparse_mla.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_float,
            ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        L.oracle_max_threads.restype = ctypes.c_int
        L.oracle_max_threads.argtypes = []
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(int(code))


def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(int(code))


def e2m1_encode(y: float) -> int:
    return lib().oracle_e2m1_encode(float(np.float32(y)))


def e4m3_encode(y: float) -> int:
    return lib().oracle_e4m3_encode(float(np.float32(y)))


def f16_to_double(bits: int) -> float:
    return lib().oracle_f16_to_double(int(bits))


def quantize_group(x16) -> tuple[np.ndarray, int]:
    """Quantize 16 FP32 values -> (16 nibble codes, scale code)."""
    x = np.ascontiguousarray(np.asarray(x16, dtype=np.float32))
    assert x.shape == (16,)
    nib = np.zeros(16, dtype=np.uint8)
    sc = np.zeros(1, dtype=np.uint8)
    lib().oracle_quantize_group(_ptr(x), _ptr(nib), _ptr(sc))
    return nib, int(sc[0])


def quantize_rows(latent_bf16_bits: np.ndarray, rope_bf16_bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns (uint16) [n,512] and [n,64] -> packed rows uint8 [n,352]."""
    lat = np.ascontiguousarray(latent_bf16_bits, dtype=np.uint16)
    rope = np.ascontiguousarray(rope_bf16_bits, dtype=np.uint16)
    n = lat.shape[0]
    assert lat.shape == (n, 512) and rope.shape == (n, 64)
    out = np.zeros((n, ROW_BYTES), dtype=np.uint8)
    if n:
        lib().oracle_quantize_rows(_ptr(lat), 512, _ptr(rope), 64, n, _ptr(out))
    return out


def quantize_fp8_rows(latent_bf16_bits: np.ndarray, rope_bf16_bits: np.ndarray) -> np.ndarray:
    """BF16 bit patterns [n,512] and [n,64] -> 576-byte E4M3 rows uint8 [n,576]."""
    lat = np.ascontiguousarray(latent_bf16_bits, dtype=np.uint16)
    rope = np.ascontiguousarray(rope_bf16_bits, dtype=np.uint16)
    n = lat.shape[0]
    assert lat.shape == (n, 512) and rope.shape == (n, 64)
    out = np.zeros((n, STAGED_ROW_BYTES), dtype=np.uint8)
    if n:
        lib().oracle_quantize_fp8_rows(_ptr(lat), 512, _ptr(rope), 64, n, _ptr(out))
    return out


def dequant_rows(rows: np.ndarray) -> np.ndarray:
    """Packed rows uint8 [n,352] -> float64 [n,576] (512 latent + 64 RoPE)."""
    rows = np.ascontiguousarray(rows, dtype=np.uint8)
    n = rows.shape[0]
    out = np.zeros((n, 576), dtype=np.float64)
    L = lib()
    for r in range(n):
        L.oracle_dequant_row(_ptr(rows[r]), _ptr(out[r]))
    return out


def stage_rows(rows: np.ndarray) -> np.ndarray:
    """Packed rows uint8 [n,352] -> staged E4M3 rows uint8 [n,576]."""
    rows = np.ascontiguousarray(rows, dtype=np.uint8)
    n = rows.shape[0]
    out = np.zeros((n, STAGED_ROW_BYTES), dtype=np.uint8)
    L = lib()
    for r in range(n):
        L.oracle_stage_row(_ptr(rows[r]), _ptr(out[r]))
    return out


def sparse_mla(q_nope_f16: np.ndarray, q_rope_f16: np.ndarray, cache: np.ndarray,
               indices: np.ndarray, sm_scale: float, staged: bool = False,
               nthreads: int = 0, num_slots: int | None = None, fp8_rows: bool = False):
    """FP64 sparse MLA decode.  q: float16 [T,H,512] / [T,H,64]; cache uint8
    [num_slots,352] (or [num_slots,576] E4M3 rows with fp8_rows); indices
    int32 [T,topk].  Returns (out f64 [T,H,512], lse f64 [T,H])."""
    qn = np.ascontiguousarray(q_nope_f16, dtype=np.float16)
    qr = np.ascontiguousarray(q_rope_f16, dtype=np.float16)
    cache = np.ascontiguousarray(cache, dtype=np.uint8)
    idx = np.ascontiguousarray(indices, dtype=np.int32)
    T, H = qn.shape[0], qn.shape[1]
    assert qn.shape == (T, H, 512) and qr.shape == (T, H, 64)
    assert idx.ndim == 2 and idx.shape[0] == T
    topk = idx.shape[1]
    if num_slots is None:
        num_slots = cache.shape[0]
    assert cache.ndim == 2 and cache.shape[1] == (STAGED_ROW_BYTES if fp8_rows else ROW_BYTES)
    assert cache.shape[0] >= num_slots
    out = np.zeros((T, H, 512), dtype=np.float64)
    lse = np.zeros((T, H), dtype=np.float64)
    rc = lib().oracle_sparse_mla(_ptr(qn.view(np.uint16)), _ptr(qr.view(np.uint16)), _ptr(cache),
                                 int(num_slots), _ptr(idx), int(topk), int(T), int(H),
                                 float(np.float32(sm_scale)), 2 if fp8_rows else int(bool(staged)),
                                 _ptr(out), _ptr(lse), int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_sparse_mla failed (%d)" % rc)
    return out, lse


def max_threads() -> int:
    return int(lib().oracle_max_threads())
