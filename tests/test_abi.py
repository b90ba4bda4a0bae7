"""Host-side checks of the C ABI (no GPU needed): the library builds and
loads, exports every function include/nvfp4mla.h declares, plans work, and
rejects bad arguments before touching the device."""
import ctypes
import os
import re

import pytest

import nvfp4_sparse_mla_decode_b200 as nv
from nvfp4_sparse_mla_decode_b200 import build as nvbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    nvbuild.build()
    return nv.lib()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "nvfp4mla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4\w*)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = declared_functions()
    assert "nvfp4_sparse_mla_decode" in names and "nvfp4_kv_append" in names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for s in range(7):
        assert nv.status_string(s)
    assert nv.status_string(0) == "ok"
    assert nv.version() >= 100


def test_plan_splits_fill_the_gpu(L):
    assert nv.num_splits(35, 64) == 4          # 140 CTAs on 148 SMs
    assert nv.num_splits(1, 16) == 16
    assert nv.num_splits(1, 128) == 16         # 2 head groups x 16
    assert nv.num_splits(64, 128) == 1
    assert nv.num_splits(4000, 64) == 1
    assert nv.num_splits(1, 64, 100) == 1      # a 100-entry list is one tile
    assert nv.num_splits(1, 48) == 0           # unsupported head count
    assert nv.workspace_size(35, 64) == 4096 + 35 * 4 * 64 * 514 * 4
    assert nv.workspace_size(4000, 64) == 0
    assert nv.staging_size(35) == 35 * 2048 * 576


def test_tuned_plan_workspace(L):
    # nvfp4mla_tuning fixes S and HG; 0 keeps the automatic choice; settings
    # a shape cannot take give 0 bytes (and INVALID_ARG from the decode)
    ws = lambda T, H, topk=2048, **kw: nv.workspace_size(T, H, topk, nv.Tuning(**kw))
    per = lambda T, S, H: 4096 + T * S * H * 514 * 4
    assert ws(35, 64) == nv.workspace_size(35, 64) == per(35, 4, 64)
    assert ws(35, 64, splits=1) == 0                       # one CTA per list: no merge
    assert ws(35, 64, splits=2) == per(35, 2, 64)
    assert ws(1, 64, splits=16) == per(1, 16, 64)
    assert ws(1, 64, splits=16, heads_per_cta=16) == per(1, 16, 64)  # 4 groups x 16 splits = 64 CTAs
    assert ws(35, 64, heads_per_cta=32) == per(35, 2, 64)  # automatic S for 70 units: 2
    assert ws(35, 64, splits=8) == 0                       # 280 CTAs cannot all be resident
    assert ws(1, 64, splits=3) == 0                        # not a power of two
    assert ws(1, 64, 100, splits=2) == 0                   # a 100-entry list is one tile
    assert ws(1, 64, heads_per_cta=48) == 0
    assert ws(1, 32, heads_per_cta=64) == 0                # more heads per CTA than H
    assert ws(1, 64, reserved=1) == 0
    assert ws(1, 48) == 0                                  # unsupported head count
    t = nv.Tuning(splits=3)
    args = [1 << 20, 1 << 20, 1 << 20, 100, 1 << 20, 2048, 1, 64, 0.1, 1 << 20, 1 << 20, 1 << 20, 1 << 30,
            None, 0]
    assert L.nvfp4_sparse_mla_decode_tuned(*args, ctypes.byref(t), None, None) == 1        # INVALID_ARG
    t = nv.Tuning(force_staged=1)
    assert L.nvfp4_sparse_mla_decode_tuned(*args, ctypes.byref(t), None, None) == 3        # no staging: WS
    args[7] = 48
    assert L.nvfp4_sparse_mla_decode_tuned(*args, None, None, None) == 2                    # UNSUPPORTED
    args[7], args[6] = 64, 0
    assert L.nvfp4_sparse_mla_decode_tuned(*args, None, None, None) == 0                    # T = 0: no-op


def _decode(L, **kw):
    a = dict(q=1 << 20, qr=1 << 20, cache=1 << 20, ns=100, idx=1 << 20, topk=2048, T=1, H=64, sc=0.1,
             out=1 << 20, lse=1 << 20, ws=1 << 20, wsb=1 << 30, st=None, stream=None)
    a.update(kw)
    return L.nvfp4_sparse_mla_decode(a["q"], a["qr"], a["cache"], a["ns"], a["idx"], a["topk"], a["T"], a["H"],
                                     a["sc"], a["out"], a["lse"], a["ws"], a["wsb"], a["st"], a["stream"])


def test_last_cuda_error_query(L):
    # the CUDA error behind the last NVFP4MLA_ERR_CUDA of this thread (0 and
    # "no error" until one happens); its text is what NVFP4MLAError shows
    code = L.nvfp4mla_last_cuda_error()
    text = L.nvfp4mla_last_cuda_error_string()
    assert code >= 0 and isinstance(text, bytes) and text
    if code == 0:
        assert text == b"no error"
    err = nv.NVFP4MLAError(4, "call", "an illegal memory access was encountered")
    assert "CUDA runtime error" in str(err) and "illegal memory access" in str(err) and err.status == 4


def test_decode_argument_errors(L):
    INVALID, UNSUP, WS = 1, 2, 3
    assert _decode(L, T=0) == 0                      # nothing to do, nothing launched
    assert _decode(L, q=None) == INVALID
    assert _decode(L, q=(1 << 20) + 8) == INVALID    # misaligned
    assert _decode(L, topk=0) == INVALID
    assert _decode(L, topk=4096) == INVALID
    assert _decode(L, ns=0) == INVALID
    assert _decode(L, H=48) == UNSUP
    assert _decode(L, H=256) == UNSUP
    assert _decode(L, T=35, ws=None, wsb=0) == WS
    assert _decode(L, T=35, wsb=1000) == WS
    assert _decode(L, sc=float("nan")) == INVALID


def test_append_argument_errors(L):
    f = L.nvfp4_kv_append
    assert f(None, 512, None, 64, None, 0, None, 10, None, None) == 0
    assert f(None, 512, 1 << 20, 64, 1 << 20, 4, 1 << 20, 10, None, None) == 1
    assert f(1 << 20, 500, 1 << 20, 64, 1 << 20, 4, 1 << 20, 10, None, None) == 1
    assert f(1 << 20, 512, 1 << 20, 60, 1 << 20, 4, 1 << 20, 10, None, None) == 1


def test_staged_argument_errors(L):
    f = L.nvfp4_staged_fp8_mla_decode
    base = [1 << 20, 1 << 20, 1 << 20, 100, 1 << 20, 2048, 1, 64, 0.1, 1 << 20, 1 << 20]
    assert f(*base, None, 0, None, 0, None, None) == 3            # no staging buffer
    assert f(*base, 1 << 20, 1000, None, 0, None, None) == 3      # staging too small
    assert f(*base, (1 << 20) + 4, 1 << 30, None, 0, None, None) == 1


def test_library_is_sm100a_only():
    log = os.path.join(ROOT, "nvfp4_sparse_mla_decode_b200", "build.log")
    if os.path.exists(log):
        assert "arch=compute_100a,code=sm_100a" in open(log).read()


def test_noalloc_argument_errors(L):
    # the same host checks as the workspace entry point, all before any
    # device call; the largest plan on 148 SMs fits the static scratch
    INVALID, UNSUP = 1, 2
    f = L.nvfp4_sparse_mla_decode_noalloc

    def call(**kw):
        a = dict(q=1 << 20, qr=1 << 20, cache=1 << 20, ns=100, idx=1 << 20, topk=2048, T=1, H=64, sc=0.1,
                 out=1 << 20, lse=1 << 20, st=None, stream=None)
        a.update(kw)
        return f(a["q"], a["qr"], a["cache"], a["ns"], a["idx"], a["topk"], a["T"], a["H"], a["sc"], a["out"],
                 a["lse"], a["st"], a["stream"])

    assert call(T=0) == 0
    assert call(q=None) == INVALID
    assert call(out=(1 << 20) + 4) == INVALID
    assert call(topk=0) == INVALID
    assert call(H=48) == UNSUP
    assert call(sc=float("inf")) == INVALID
    worst = max(nv.workspace_size(T, H) for T in range(1, 149) for H in (16, 32, 64, 128))
    assert worst <= 20 << 20


def test_selftest_argument_errors(L):
    f = L.nvfp4mla_selftest_wait_timeout
    assert f(None, 1 << 20, None) == 1
    assert f(1 << 20, None, None) == 1
    assert f((1 << 20) + 2, 1 << 20, None) == 1


def test_paged_argument_errors(L):
    f = L.nvfp4_sparse_mla_decode_paged
    INVALID = 1

    def call(**kw):
        a = dict(q=1 << 20, qr=1 << 20, cache=1 << 20, ns=100, pos=1 << 20, topk=2048, tb=1 << 20, stride=8,
                 page=64, T=1, H=64, sc=0.1, out=1 << 20, lse=1 << 20, ws=1 << 20, wsb=1 << 30, st=None,
                 stream=None)
        a.update(kw)
        return f(a["q"], a["qr"], a["cache"], a["ns"], a["pos"], a["topk"], a["tb"], a["stride"], a["page"],
                 a["T"], a["H"], a["sc"], a["out"], a["lse"], a["ws"], a["wsb"], a["st"], a["stream"])

    assert call(T=0) == 0
    assert call(page=48) == INVALID
    assert call(page=0) == INVALID
    assert call(page=1 << 21) == INVALID
    assert call(stride=0) == INVALID
    assert call(tb=None) == INVALID
    assert call(tb=(1 << 20) + 2) == INVALID
    assert call(stride=1 << 20, page=1 << 12) == INVALID   # positions would overflow int32


def test_fp8_append_argument_errors(L):
    f = L.nvfp4mla_fp8_kv_append
    assert f(None, 512, None, 64, None, 0, None, 10, None, None) == 0
    assert f(None, 512, 1 << 20, 64, 1 << 20, 4, 1 << 20, 10, None, None) == 1
    assert f(1 << 20, 500, 1 << 20, 64, 1 << 20, 4, 1 << 20, 10, None, None) == 1
    assert f(1 << 20, 512, 1 << 20, 64, 1 << 20, 4, (1 << 20) + 8, 10, None, None) == 1   # cache misaligned
    assert f(1 << 20, 512, 1 << 20, 64, 1 << 20, -1, 1 << 20, 10, None, None) == 1


def test_fp8_decode_argument_errors(L):
    INVALID, UNSUP, WS = 1, 2, 3
    f = L.nvfp4mla_fp8_sparse_mla_decode

    def call(**kw):
        a = dict(q=1 << 20, qr=1 << 20, cache=1 << 20, ns=100, idx=1 << 20, topk=2048, T=1, H=64, sc=0.1,
                 out=1 << 20, lse=1 << 20, ws=1 << 20, wsb=1 << 30, st=None, stream=None)
        a.update(kw)
        return f(a["q"], a["qr"], a["cache"], a["ns"], a["idx"], a["topk"], a["T"], a["H"], a["sc"], a["out"],
                 a["lse"], a["ws"], a["wsb"], a["st"], a["stream"])

    assert call(T=0) == 0
    assert call(cache=None) == INVALID
    assert call(cache=(1 << 20) + 4) == INVALID
    assert call(ns=0) == INVALID
    assert call(topk=4096) == INVALID
    assert call(H=80) == UNSUP
    assert call(T=35, ws=None, wsb=0) == WS
    assert call(T=35, ws=(1 << 20) + 16) == INVALID   # workspace not 256-byte aligned


def test_indexer_argument_errors(L):
    INVALID, WS = 1, 3
    f = L.nvfp4mla_indexer_scores

    def call(**kw):
        a = dict(q=1 << 20, w=1 << 20, k=1 << 20, ns=4096, tb=1 << 20, tbs=64, page=64, lens=1 << 20,
                 maxc=4096, T=2, sc=1 << 20, scs=4096, st=None, stream=None)
        a.update(kw)
        return f(a["q"], a["w"], a["k"], a["ns"], a["tb"], a["tbs"], a["page"], a["lens"], a["maxc"], a["T"],
                 a["sc"], a["scs"], a["st"], a["stream"])

    assert call(T=0) == 0
    assert call(maxc=0) == 0
    assert call(page=48) == INVALID           # not a power of two
    assert call(page=4) == INVALID            # below the 8-row copy
    assert call(maxc=64 * 64 + 1) == INVALID  # more positions than the table can map
    assert call(scs=4095) == INVALID
    assert call(scs=4098) == INVALID          # not a multiple of 4
    assert call(k=(1 << 20) + 8) == INVALID   # key cache misaligned
    assert call(sc=(1 << 20) + 4) == INVALID
    assert call(q=None) == INVALID
    t = L.nvfp4mla_indexer_topk
    args = [1 << 20, 4096, 1 << 20, 4096, 2]
    assert t(*args, 0, 1 << 20, 1 << 20, 1 << 30, None, None) == INVALID       # topk 0
    assert t(*args, 4096, 1 << 20, 1 << 20, 1 << 30, None, None) == INVALID    # topk > 2048
    assert t(1 << 20, 4096, 1 << 20, 4096, 0, 2048, 1 << 20, None, 0, None, None) == 0
    # with 148 SMs, 2 requests split their rows over 8 CTAs each: workspace needed
    need = L.nvfp4mla_indexer_topk_workspace_size(2)
    assert need == 256 + 256 + 2 * 8 * 8192 * 8  # 16 bytes of counts per CTA; 8192 8-byte candidates per CTA
    assert t(*args, 2048, 1 << 20, None, 0, None, None) == WS
    assert t(*args, 2048, 1 << 20, 1 << 20, need - 1, None, None) == WS
    assert t(*args, 2048, 1 << 20, (1 << 20) + 16, need, None, None) == INVALID  # not 256-byte aligned
    assert L.nvfp4mla_indexer_topk_workspace_size(148) == 0                     # one CTA per request
    s = L.nvfp4mla_sparse_indexer
    base = [1 << 20, 1 << 20, 1 << 20, 4096, 1 << 20, 64, 64, 1 << 20, 4096, 2, 2048, 1 << 20]
    assert s(*base, None, 0, None, None) == WS
    assert s(*base, 1 << 20, 1000, None, None) == WS
    assert L.nvfp4mla_indexer_workspace_size(35, 140000) == (35 * 140032 * 4 + 255) // 256 * 256 + \
        L.nvfp4mla_indexer_topk_workspace_size(35)
    # 35 requests x 4 CTAs: counters (140 B -> 256), 16 bytes of counts per CTA (2240 B -> 2304), candidates
    assert L.nvfp4mla_indexer_topk_workspace_size(35) == 256 + 2304 + 35 * 4 * 8192 * 8
    assert L.nvfp4mla_indexer_score_stride(140000) == 140032


def test_blhnc_argument_errors(L):
    INVALID = 1
    f = L.nvfp4mla_blhnc_convert

    def call(**kw):
        a = dict(lp=1 << 20, L=4, nblk=100, N=64, C=352, sub=16, ids=1 << 20, nids=1 << 20, nb=5, out=1 << 20,
                 nnew=1000, dirn=1, st=None, stream=None)
        a.update(kw)
        return f(a["lp"], a["L"], a["nblk"], a["N"], a["C"], a["sub"], a["ids"], a["nids"], a["nb"], a["out"],
                 a["nnew"], a["dirn"], a["st"], a["stream"])

    assert call(nb=0) == 0
    assert call(sub=3) == INVALID           # 64 positions do not split in 3
    assert call(C=350) == INVALID           # rows must be whole 16-byte units
    assert call(L=0) == INVALID
    assert call(dirn=2) == INVALID
    assert call(out=(1 << 20) + 8) == INVALID
    assert call(lp=None) == INVALID


def test_copy_descriptor_model_matches_oracle():
    import numpy as np
    from oracle import blhnc
    rng = np.random.default_rng(3)
    for _ in range(50):
        ids = rng.integers(0, 50, size=int(rng.integers(0, 40)))
        layers = int(rng.integers(1, 100))
        assert nv.copy_descriptors(ids, layers) == blhnc.descriptors_layer_major(ids, layers)
        assert nv.copy_descriptors(ids) == blhnc.descriptors_block_major(ids)
