"""The no-allocation decode entry point (static per-device scratch) against
nvfp4_sparse_mla_decode with its own workspace: the same kernel runs on both,
so two calls in a row must give bit-identical out and lse, and leave the
scratch's split counters at zero for the next call.  Named to run last, so it
also runs after every other GPU test has used the library."""
import pytest
import torch

import nvfp4_sparse_mla_decode_b200 as nv
from nvfp4_sparse_mla_decode_b200 import synth
from harness import build_cache, check_close, oracle_decode

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", ["decode35x64", "tiny", "sweep8x128", "no_split", "t1x128", "t2x64"])
def test_noalloc_matches_workspace_entry_point_twice(shape):
    if shape == "t1x128":
        w = synth.per_request("cuda", [6000], 128, seed=65, name="na1")        # 32 heads per CTA, S = 16
    elif shape == "t2x64":
        w = synth.per_request("cuda", [6000] * 2, 64, seed=66, name="na2")     # 32 heads per CTA, S = 16
    elif shape == "decode35x64":
        w = synth.per_request("cuda", [6000] * 35, 64, seed=61, name="na35")   # S = 4
    elif shape == "tiny":
        w = synth.tiny("cuda", seed=62)                                        # S = 16
    elif shape == "sweep8x128":
        w = synth.per_request("cuda", [6000] * 8, 128, seed=63, name="na8")    # S = 8
    else:
        w = synth.per_request("cuda", [3000] * 160, 64, seed=64, name="na160")  # S = 1
    cache = build_cache(w)
    ref_out, ref_lse = nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        nv.decode_noalloc(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, out, lse, dev_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    tokens = [0, w.T - 1]
    o, l = oracle_decode(w, tokens)
    check_close(out[tokens], lse[tokens], o, l)


def test_noalloc_zero_tokens_is_noop():
    cache = torch.zeros(16, nv.ROW_BYTES, dtype=torch.uint8, device="cuda")
    qn = torch.empty(0, 64, 512, dtype=torch.float16, device="cuda")
    qr = torch.empty(0, 64, 64, dtype=torch.float16, device="cuda")
    idx = torch.empty(0, 2048, dtype=torch.int32, device="cuda")
    out = torch.empty(0, 64, 512, dtype=torch.float16, device="cuda")
    lse = torch.empty(0, 64, dtype=torch.float32, device="cuda")
    nv.decode_noalloc(qn, qr, cache, idx, 0.1, out, lse)
