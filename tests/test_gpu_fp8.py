"""The 576-byte E4M3 row cache on the GPU vs the CPU oracle.

Page "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
section "Four-bit caches make room": before NVFP4 a cache row took 576
bytes, one FP8 byte per latent or RoPE dim.  nvfp4mla_fp8_kv_append must
match the oracle's quantize_fp8_rows bit for bit; nvfp4mla_fp8_sparse_mla_decode
must match the oracle's attention over those rows within the decode
tolerance (max|out - ref| <= 2e-3 * max|ref| + 1e-4, |lse - ref| <= 1e-3)."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_sparse_mla_decode_b200 as nv
from nvfp4_sparse_mla_decode_b200 import synth
from harness import bf16_bits, build_fp8_cache, check_close, oracle_decode

pytestmark = pytest.mark.gpu


def _append_and_compare(lat, rope, slots, num_slots):
    cache = torch.full((num_slots, nv.STAGED_ROW_BYTES), 0xAB, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.fp8_kv_append(lat, rope, slots, cache, status)
    torch.cuda.synchronize()
    got = cache[slots.long()].cpu().numpy()
    ref = oracle.quantize_fp8_rows(bf16_bits(lat), bf16_bits(rope))
    bad = np.nonzero((got != ref).any(axis=1))[0]
    assert bad.size == 0, "rows differ: %s" % bad[:8]
    assert int(status.item()) == 0
    return cache


def test_fp8_append_random_rows_bit_exact():
    scale = synth.channel_scale(31, "cuda")
    lat, rope = synth.source_rows(20000, scale, 32, "cuda", special=True)
    slots = torch.randperm(50000, device="cuda")[:20000].to(torch.int32)
    _append_and_compare(lat, rope, slots, 50000)


def test_fp8_append_ties_subnormals_saturation_bit_exact():
    # every E4M3 code's value, the midpoints between neighbours (ties to
    # even), values past the largest finite code, in both signs
    codes = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    mids = (codes[1:] + codes[:-1]) / 2
    vals = np.concatenate([codes, mids, [449.0, 464.0, 480.0, 1e5, 3e38, 0.0]])
    vals = np.concatenate([vals, -vals])
    flat = torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)
    n = -(-flat.numel() // 576)
    rows = torch.zeros(n * 576, dtype=torch.bfloat16)
    rows[:flat.numel()] = flat
    rows = rows.view(n, 576).cuda()
    slots = torch.arange(n, dtype=torch.int32, device="cuda")
    _append_and_compare(rows[:, :512], rows[:, 512:], slots, n)


def test_fp8_append_skips_negative_and_flags_out_of_range_slots():
    scale = synth.channel_scale(33, "cuda")
    lat, rope = synth.source_rows(8, scale, 34, "cuda")
    slots = torch.tensor([0, -1, 2, 99, 4, -5, 6, 7], dtype=torch.int32, device="cuda")
    cache = torch.full((8, nv.STAGED_ROW_BYTES), 0xAB, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.fp8_kv_append(lat, rope, slots, cache, status)
    torch.cuda.synchronize()
    assert int(status.item()) & nv.DEV_BAD_INDEX
    c = cache.cpu().numpy()
    ref = oracle.quantize_fp8_rows(bf16_bits(lat), bf16_bits(rope))
    for i, s in enumerate(slots.tolist()):
        if 0 <= s < 8:
            assert np.array_equal(c[s], ref[i])
    for untouched in (1, 3, 5):
        assert np.all(c[untouched] == 0xAB)


def run(w, cache, tokens=None):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = nv.fp8_decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    tokens = list(range(w.T)) if tokens is None else list(tokens)
    ref_o, ref_l = oracle_decode(w, tokens, fp8_rows=True)
    return check_close(out[tokens], lse[tokens], ref_o, ref_l)


def test_fp8_decode_tiny():
    w = synth.tiny("cuda")
    run(w, build_fp8_cache(w))


@pytest.mark.parametrize("H", [16, 32, 64, 128])
def test_fp8_decode_ragged_tiles_all_head_counts(H):
    T = 6
    w = synth.per_request("cuda", [9000] * T, H, seed=35, name="ragged")
    for t, n in enumerate([1, 100, 128, 129, 700, 2048]):
        w.indices[t, n:] = -1
    run(w, build_fp8_cache(w))


@pytest.mark.parametrize("T,H", [(1, 64), (2, 128), (4, 64)])
def test_fp8_decode_small_batches(T, H):
    # small batches take 32 heads per CTA and 16 splits: every token
    w = synth.per_request("cuda", [9000] * T, H, seed=37 + T, name="small")
    run(w, build_fp8_cache(w))


def test_fp8_decode35x64_full():
    w = synth.decode35("cuda")
    assert nv.num_splits(w.T, w.H) == 4
    run(w, build_fp8_cache(w))


def test_fp8_decode_empty_and_out_of_range_entries():
    w = synth.per_request("cuda", [5000] * 4, 64, seed=36, name="edge")
    w.indices[0, :] = -1                       # all empty: out 0, lse -inf
    w.indices[1, 5:] = -1
    w.indices[2, ::2] = w.num_slots + 7        # out of range: empty, flagged
    w.indices[3, ::3] = -(2 ** 31)
    cache = build_fp8_cache(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = nv.fp8_decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & nv.DEV_BAD_INDEX
    assert torch.all(out[0] == 0) and torch.all(torch.isneginf(lse[0]))
    ref_o, ref_l = oracle_decode(w, range(4), fp8_rows=True)
    check_close(out, lse, ref_o, ref_l)
