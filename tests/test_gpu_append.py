"""nvfp4_kv_append on the GPU vs the CPU oracle's quantizer: bit-exact.

Page "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
section "Four-bit caches make room" (352-byte rows, one FP8 scale per 16
values).  Inputs come from the seeded generators; the oracle quantizes the
same BF16 rows on the CPU."""
import numpy as np
import pytest
import torch

import oracle
import nvfp4_sparse_mla_decode_b200 as nv
from nvfp4_sparse_mla_decode_b200 import synth
from harness import bf16_bits

pytestmark = pytest.mark.gpu


def _append_and_compare(lat, rope, slots, num_slots):
    cache = torch.full((num_slots, nv.ROW_BYTES), 0xAB, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.kv_append(lat, rope, slots, cache, status)
    torch.cuda.synchronize()
    got = cache[slots.long()].cpu().numpy()
    ref = oracle.quantize_rows(bf16_bits(lat), bf16_bits(rope))
    bad = np.nonzero((got != ref).any(axis=1))[0]
    assert bad.size == 0, "rows differ: %s; first row bytes differ at %s" % (
        bad[:8], np.nonzero(got[bad[0]] != ref[bad[0]])[0][:16] if bad.size else None)
    assert int(status.item()) == 0
    return cache


def test_append_prefill_rows_bit_exact():
    w = synth.append_prefill("cuda")
    _append_and_compare(w.new_lat, w.new_rope, w.new_slots, w.num_slots)


def test_append_random_rows_bit_exact():
    scale = synth.channel_scale(77, "cuda")
    lat, rope = synth.source_rows(20000, scale, 78, "cuda")
    slots = torch.randperm(50000, device="cuda")[:20000].to(torch.int32)
    _append_and_compare(lat, rope, slots, 50000)


def _tie_rows():
    rows = []
    mids = [6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, 0.0]
    for e in range(-9, 9):
        s = 2.0 ** e
        rows.append([m * s for m in mids] * 32)
    # scales that saturate / overflow E4M3 and tiny scales
    for amax in [3000.0, 2688.0, 2700.0, 448.0 * 6, 1e-3, 6e-3, 2 ** -12, 2 ** -20, 0.0]:
        g = [amax * f for f in [1.0, -0.5, 0.3, -0.9, 0.77, 0.01, -0.02, 0.6, 0.1, 0.2, -1.0, 0.45, 0.55, 0.65, 0.75, 0.0]]
        rows.append(g * 32)
    lat = torch.tensor(rows, dtype=torch.float32).to(torch.bfloat16)
    rope_vals = [0.0, -0.0, 448.0, -448.0, 460.0, 464.0, 470.0, 1e6, 2 ** -9, 2 ** -10, 3 * 2 ** -11, 1.0625, 1.1875,
                 -1.0625, 0.015625, 0.0146484375] * 4
    rope = torch.tensor([rope_vals] * lat.shape[0], dtype=torch.float32).to(torch.bfloat16)
    return lat.cuda(), rope.cuda()


def test_append_ties_saturation_subnormals_bit_exact():
    lat, rope = _tie_rows()
    slots = torch.arange(lat.shape[0], dtype=torch.int32, device="cuda")
    _append_and_compare(lat, rope, slots, lat.shape[0])


def test_append_strided_inputs():
    scale = synth.channel_scale(5, "cuda")
    lat, rope = synth.source_rows(1000, scale, 6, "cuda")
    both = torch.cat([lat, rope], dim=1).contiguous()  # [n, 576]: strides 576 for both views
    slots = torch.arange(1000, dtype=torch.int32, device="cuda")
    cache = torch.zeros(1000, nv.ROW_BYTES, dtype=torch.uint8, device="cuda")
    nv.kv_append(both[:, :512], both[:, 512:], slots, cache)
    ref = oracle.quantize_rows(bf16_bits(lat), bf16_bits(rope))
    assert np.array_equal(cache.cpu().numpy(), ref)


def test_append_skips_negative_and_flags_out_of_range_slots():
    scale = synth.channel_scale(9, "cuda")
    lat, rope = synth.source_rows(8, scale, 10, "cuda")
    slots = torch.tensor([0, -1, 2, 99, 4, -5, 6, 7], dtype=torch.int32, device="cuda")
    cache = torch.full((8, nv.ROW_BYTES), 0xAB, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.kv_append(lat, rope, slots, cache, status)
    torch.cuda.synchronize()
    assert int(status.item()) & nv.DEV_BAD_INDEX
    c = cache.cpu().numpy()
    ref = oracle.quantize_rows(bf16_bits(lat), bf16_bits(rope))
    for i, s in enumerate(slots.tolist()):
        if 0 <= s < 8:
            assert np.array_equal(c[s], ref[i])
    for untouched in (1, 3, 5):
        assert np.all(c[untouched] == 0xAB)


def test_append_empty_is_noop():
    cache = torch.zeros(4, nv.ROW_BYTES, dtype=torch.uint8, device="cuda")
    e = torch.empty(0, 512, dtype=torch.bfloat16, device="cuda")
    r = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
    nv.kv_append(e, r, torch.empty(0, dtype=torch.int32, device="cuda"), cache)
    torch.cuda.synchronize()
    assert int(cache.sum()) == 0
