"""Failure detection without a fault: the bounded waits every kernel uses
must end with NVFP4MLA_DEV_TIMEOUT when nothing ever completes them, and the
CUDA context must stay usable afterwards."""
import pytest
import torch

import nvfp4_sparse_mla_decode_b200 as nv
from nvfp4_sparse_mla_decode_b200 import synth
from harness import build_cache, check_close, oracle_decode

pytestmark = pytest.mark.gpu


def test_waits_run_out_and_report_timeout():
    assert nv.selftest_wait_timeout() == nv.DEV_TIMEOUT


def test_context_usable_after_timeouts():
    for _ in range(2):
        assert nv.selftest_wait_timeout() == nv.DEV_TIMEOUT
    w = synth.tiny("cuda", seed=71)
    cache = build_cache(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o, l = oracle_decode(w, [0])
    check_close(out, lse, o, l)


# The decode kernel's own timeout paths, driven through the library's
# test-only entry point: a short wait bound (about 0.1 ms of clocks) and one
# arrival withheld.  Nothing faults or hangs: every wait runs out, the kernel
# reports NVFP4MLA_DEV_TIMEOUT through dev_status and exits.
_WAIT_CYCLES = 200_000


def _hooked_decode(w, cache, workspace, status, withhold):
    import ctypes
    L = nv.lib()
    fn = L.nvfp4mla_test_decode_hooks
    fn.restype = ctypes.c_int32
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                   ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_float, ctypes.c_void_p,
                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_uint64,
                   ctypes.c_int32, ctypes.c_void_p]
    T, H = w.T, w.H
    out = torch.empty(T, H, 512, dtype=torch.float16, device="cuda")
    lse = torch.empty(T, H, dtype=torch.float32, device="cuda")
    st = fn(w.q_nope.data_ptr(), w.q_rope.data_ptr(), cache.data_ptr(), cache.shape[0], w.indices.data_ptr(),
            w.indices.shape[1], T, H, float(w.sm_scale), out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
            workspace.numel(), status.data_ptr(), _WAIT_CYCLES, withhold,
            torch.cuda.current_stream().cuda_stream)
    assert st == 0, nv.status_string(st)
    torch.cuda.synchronize()
    return out, lse


def _normal_decode(w, cache, workspace):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, workspace=workspace, dev_status=status)
    torch.cuda.synchronize()
    return int(status.item()), out, lse


def test_decode_withheld_p_times_out_then_recovers():
    # P^T is never published: the output MMAs' wait runs out, the softmax's
    # wait for them too; the merge still meets (every split arrives), so the
    # same workspace serves the next call unchanged
    w = synth.decode35("cuda")
    cache = build_cache(w)
    assert nv.num_splits(w.T, w.H) == 4
    ws = torch.zeros(nv.workspace_size(w.T, w.H), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _hooked_decode(w, cache, ws, status, withhold=1)
    assert int(status.item()) & nv.DEV_TIMEOUT
    code, out, lse = _normal_decode(w, cache, ws)
    assert code == 0
    tokens = [0, 17, 34]
    o, l = oracle_decode(w, tokens)
    check_close(out[tokens], lse[tokens], o, l)


def test_decode_merge_timeout_poisons_until_counters_cleared():
    # split 0 never arrives: every split's merge wait runs out, the group's
    # counter is poisoned and the slices are NaN; a later call on the same
    # workspace reports the timeout again instead of merging stale partials,
    # and zeroing the counter region restores normal use
    w = synth.decode35("cuda")
    cache = build_cache(w)
    ws = torch.zeros(nv.workspace_size(w.T, w.H), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = _hooked_decode(w, cache, ws, status, withhold=2)
    assert int(status.item()) & nv.DEV_TIMEOUT
    assert torch.isnan(out.float()).all()
    code, out, _ = _normal_decode(w, cache, ws)
    assert code & nv.DEV_TIMEOUT
    assert torch.isnan(out.float()).all()
    ws[:4096].zero_()
    code, out, lse = _normal_decode(w, cache, ws)
    assert code == 0
    tokens = [0, 34]
    o, l = oracle_decode(w, tokens)
    check_close(out[tokens], lse[tokens], o, l)
