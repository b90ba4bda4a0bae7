"""Sparse MLA decode on the GPU vs the FP64 CPU oracle.

Tolerance (from the target stated for this path): per (token, head)
max|out - ref| <= 2e-3 * max|ref| + 1e-4 and |lse - ref| <= 1e-3; all-empty
lists give out = 0 and lse = -inf on both sides.  The oracle sees only the
BF16 source rows (it quantizes them itself) and the index lists."""
import math

import numpy as np
import pytest
import torch

import oracle
import nvfp4_sparse_mla_decode_b200 as nv
from nvfp4_sparse_mla_decode_b200 import synth
from harness import build_cache, check_close, oracle_decode, oracle_inputs

pytestmark = pytest.mark.gpu


def run(w, cache, staged=False, tokens=None):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn = nv.staged_decode if staged else nv.decode
    out, lse = fn(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    tokens = list(range(w.T)) if tokens is None else list(tokens)
    ref_o, ref_l = oracle_decode(w, tokens, staged=staged)
    return check_close(out[tokens], lse[tokens], ref_o, ref_l)


def test_tiny_1500_valid_of_2048():
    w = synth.tiny("cuda")
    run(w, build_cache(w))


@pytest.mark.parametrize("H", [16, 32, 64, 128])
def test_ragged_tiles_all_head_counts(H):
    # lists of 1, 100, 128, 129, 700, 2048 valid entries, -1 elsewhere
    T = 6
    w = synth.per_request("cuda", [9000] * T, H, seed=11, name="ragged")
    counts = [1, 100, 128, 129, 700, 2048]
    for t, n in enumerate(counts):
        w.indices[t, n:] = -1
    run(w, build_cache(w))


def test_decode35x64_full():
    w = synth.decode35("cuda")
    assert nv.num_splits(w.T, w.H) == 4
    run(w, build_cache(w))


@pytest.mark.parametrize("H,splits,hg,staged", [
    (64, 1, 64, 0), (64, 2, 64, 0), (64, 16, 64, 0), (64, 0, 32, 0), (64, 4, 32, 0), (64, 0, 16, 0),
    (64, 4, 16, 0), (64, 1, 16, 0), (64, 2, 32, 1), (128, 16, 32, 0), (128, 0, 16, 0), (32, 8, 16, 0),
])
def test_tuned_plans_match_oracle(H, splits, hg, staged):
    # a caller's split count, heads per CTA and forced staged path: every
    # token against the oracle (the staged one for the staged path)
    T = 6 if H <= 64 else 2
    w = synth.per_request("cuda", [20000] * T, H, seed=29 + H + splits, name="tuned")
    cache = build_cache(w)
    tuning = nv.Tuning(splits=splits, heads_per_cta=hg, force_staged=staged)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, dev_status=status, tuning=tuning)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref_o, ref_l = oracle_decode(w, range(T), staged=bool(staged))
    check_close(out, lse, ref_o, ref_l)


def test_staged_path_matches_staged_oracle():
    w = synth.decode35("cuda", T=6, ctx=20000)
    run(w, build_cache(w), staged=True)


def test_staged_rows_bit_exact_against_oracle():
    # the stage kernel's 576-byte E4M3 rows, entry by entry, equal the
    # oracle's re-encoding of its own dequantized rows; empty entries are
    # left untouched
    w = synth.decode35("cuda", T=5, ctx=20000)
    w.indices[1, 1500:] = -1
    w.indices[3, ::3] = -1
    cache = build_cache(w)
    topk = w.indices.shape[1]
    staging = torch.full((nv.staging_size(w.T, topk),), 0xA5, dtype=torch.uint8, device="cuda")
    nv.staged_decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, staging=staging)
    torch.cuda.synchronize()
    _, _, rows, remap, _ = oracle_inputs(w, range(w.T))
    ref = oracle.stage_rows(rows)
    got = staging.view(w.T * topk, nv.STAGED_ROW_BYTES).cpu().numpy()
    flat = remap.reshape(-1)
    valid = flat >= 0
    assert np.array_equal(got[valid], ref[flat[valid]])
    assert np.all(got[~valid] == 0xA5)


def test_staged_two_steps_equal_one_call():
    # stage + attend as separate calls reproduce the one-call staged path bit for bit
    w = synth.decode35("cuda", T=6, ctx=20000)
    w.indices[2, 700:] = -1
    cache = build_cache(w)
    topk = w.indices.shape[1]
    staging = torch.empty(nv.staging_size(w.T, topk), dtype=torch.uint8, device="cuda")
    out1, lse1 = nv.staged_decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, staging=staging)
    out1, lse1 = out1.clone(), lse1.clone()
    staging2 = torch.empty_like(staging)
    nv.staged_stage(cache, w.indices, staging2)
    out2, lse2 = nv.staged_attend(w.q_nope, w.q_rope, cache.shape[0], w.indices, staging2, w.sm_scale)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_staged_tiny():
    w = synth.tiny("cuda")
    run(w, build_cache(w), staged=True)


@pytest.mark.parametrize("T,H", [(1, 128), (2, 64)])
def test_small_batches_32_heads_per_cta(T, H):
    # the automatic plan takes 32 heads per CTA here; native and staged paths
    w = synth.per_request("cuda", [9000] * T, H, seed=71 + T, name="small")
    cache = build_cache(w)
    run(w, cache)
    run(w, cache, staged=True)


@pytest.mark.parametrize("T", [1, 8, 32, 64, 128, 256])
def test_sweep_h128(T):
    # every token and both head groups of every token are compared
    w = synth.sweep("cuda", T)
    cache = build_cache(w)
    run(w, cache)
    del cache
    torch.cuda.empty_cache()


def test_padded_lists_256x64():
    # all 256 tokens: half the lists sorted (empty entries first), half in
    # random order, lengths from 16 to 2048 valid entries
    w = synth.padded("cuda")
    cache = build_cache(w)
    run(w, cache)


def test_append_then_prefill_4000x64():
    # all 4000 tokens of the prefill budget (about 1.1 TFLOP of FP64 work
    # for the oracle)
    w = synth.append_prefill("cuda")
    cache = build_cache(w)
    run(w, cache)


def test_all_empty_and_out_of_range_entries():
    w = synth.per_request("cuda", [5000] * 4, 64, seed=21, name="empty")
    w.indices[0, :] = -1
    w.indices[1, 5:] = -1
    w.indices[2, ::2] = w.num_slots + 7       # out of range: empty, flagged
    w.indices[3, ::3] = -(2 ** 31)
    cache = build_cache(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & nv.DEV_BAD_INDEX
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))
    ref_o, ref_l = oracle_decode(w, range(4))
    check_close(out, lse, ref_o, ref_l)


@pytest.mark.parametrize("topk", [1, 64, 100, 777, 2047])
def test_short_lists(topk):
    w = synth.per_request("cuda", [4000] * 3, 64, seed=31, name="short")
    w.indices = w.indices[:, :topk].contiguous()
    run(w, build_cache(w))


def test_duplicates_and_permutation():
    w = synth.per_request("cuda", [3000] * 2, 64, seed=41, name="dup")
    w.indices[0, 1000:] = w.indices[0, :1048].clone()   # duplicates count per position
    perm = torch.randperm(2048, device="cuda")
    w.indices[1] = w.indices[1][perm]
    run(w, build_cache(w))


def test_zero_tokens_is_noop():
    cache = torch.zeros(16, nv.ROW_BYTES, dtype=torch.uint8, device="cuda")
    qn = torch.empty(0, 64, 512, dtype=torch.float16, device="cuda")
    qr = torch.empty(0, 64, 64, dtype=torch.float16, device="cuda")
    idx = torch.empty(0, 2048, dtype=torch.int32, device="cuda")
    out, lse = nv.decode(qn, qr, cache, idx, 0.1)
    assert out.numel() == 0 and lse.numel() == 0


def test_split_workspace_reused_across_shapes_and_calls():
    # One zero-filled workspace serves split launches of different shapes
    # (S = 4, 8 and 16 here); every call must leave the 4096-byte counter
    # region at zero and repeat its results bit for bit.
    shapes = [(synth.per_request("cuda", [6000] * 35, 64, seed=51, name="ws35"), [0, 17, 34]),
              (synth.per_request("cuda", [6000] * 6, 128, seed=52, name="ws6"), [0, 5]),
              (synth.tiny("cuda", seed=53), [0])]
    need = max(nv.workspace_size(w.T, w.H) for w, _ in shapes)
    assert [nv.num_splits(w.T, w.H) for w, _ in shapes] == [4, 8, 16]
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for w, tokens in shapes:
        cache = build_cache(w)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        first = None
        for _ in range(2):
            out, lse = nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, workspace=ws, dev_status=status)
            torch.cuda.synchronize()
            assert int(status.item()) == 0
            assert int(ws[:4096].count_nonzero().item()) == 0, "split counters not reset"
            if first is None:
                first = (out.clone(), lse.clone())
            else:
                assert torch.equal(out, first[0]) and torch.equal(lse, first[1])
        ref_o, ref_l = oracle_decode(w, tokens)
        check_close(out[tokens], lse[tokens], ref_o, ref_l)
        del cache


def test_host_buffer_call_matches_device_call():
    # the call that copies host inputs in and results out on its stream gives
    # the device call's results bit for bit, on two streams with their own
    # device buffers and workspaces
    w = synth.decode35("cuda", T=6, ctx=20000)
    cache = build_cache(w)
    ref_out, ref_lse = nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale)
    torch.cuda.synchronize()
    h_qn, h_qr, h_ix = w.q_nope.cpu().pin_memory(), w.q_rope.cpu().pin_memory(), w.indices.cpu().pin_memory()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = []
    for s in streams:
        d = dict(d_q_nope=torch.empty_like(w.q_nope), d_q_rope=torch.empty_like(w.q_rope),
                 d_indices=torch.empty_like(w.indices), d_out=torch.empty(w.T, w.H, 512, dtype=torch.float16,
                                                                          device="cuda"),
                 d_lse=torch.empty(w.T, w.H, dtype=torch.float32, device="cuda"))
        h_out = torch.empty(w.T, w.H, 512, dtype=torch.float16).pin_memory()
        h_lse = torch.empty(w.T, w.H, dtype=torch.float32).pin_memory()
        ws = torch.zeros(max(1, nv.workspace_size(w.T, w.H)), dtype=torch.uint8, device="cuda")
        nv.decode_host(h_qn, h_qr, h_ix, h_out, h_lse, cache=cache, sm_scale=w.sm_scale, workspace=ws, stream=s, **d)
        outs.append((h_out, h_lse))
    torch.cuda.synchronize()
    for h_out, h_lse in outs:
        assert torch.equal(h_out, ref_out.cpu()) and torch.equal(h_lse, ref_lse.cpu())
