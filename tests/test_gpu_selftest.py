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
