"""Pins for the CPU oracle (no GPU).

Every check compares the oracle with something other than itself: the
format tables of the OCP FP4/FP8 specifications (golden files), torch's own
float8_e4m3fn conversion, closed-form rounding bounds, dense softmax
attention computed with numpy, invariances of the definition, and brute
force on tiny inputs.  Page "Prime Intellect Launches Prime Inference,
Serving 600B Tokens Daily", section "Four-bit caches make room", is the
source of the row sizes, the group size and the 2,048-position list.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden

RNG = np.random.default_rng(12345)


def f32(x):
    return float(np.float32(x))


# ---------------------------------------------------------------- formats

def test_e2m1_value_table_matches_spec():
    for code, val in read_golden("e2m1_values.txt"):
        got = oracle.e2m1_value(int(code))
        assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val)), code


def test_e4m3_decode_all_codes_match_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(got), hex(c)
        else:
            assert got == ref[c] and math.copysign(1, got) == math.copysign(1, ref[c]), hex(c)


def test_e4m3_anchor_values():
    for code, val in read_golden("e4m3_anchors.txt"):
        got = oracle.e4m3_value(int(code, 16))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val)


def _torch_e4m3_code(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_in_range():
    # random magnitudes over the whole finite range incl. subnormals
    mags = np.exp(RNG.uniform(np.log(1e-4), np.log(460.0), 4000)).astype(np.float32)
    signs = RNG.choice([-1.0, 1.0], size=mags.size).astype(np.float32)
    xs = mags * signs
    # exact midpoints between neighbouring codes (ties) and the codes themselves
    vals = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    mids = ((vals[1:] + vals[:-1]) / 2).astype(np.float32)
    xs = np.concatenate([xs, vals.astype(np.float32), mids, -mids, [0.0, -0.0]]).astype(np.float32)
    ref = _torch_e4m3_code(xs)
    got = np.array([oracle.e4m3_encode(x) for x in xs], dtype=np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(xs[i], got[i], ref[i]) for i in bad[:10]]


def test_e4m3_encode_saturates():
    for x in [448.0, 463.99, 464.0, 465.0, 1e6, 3e38]:
        assert oracle.e4m3_encode(x) == 0x7E
        assert oracle.e4m3_encode(-x) == 0xFE


def test_e2m1_rounding_table():
    for x, code in read_golden("e2m1_rounding.txt"):
        assert oracle.e2m1_encode(float(x)) == int(code), x


def test_e2m1_encode_brute_force_nearest_even():
    table = np.array([float(v) for _, v in read_golden("e2m1_values.txt")[:8]])
    xs = np.concatenate([RNG.uniform(-8, 8, 5000), np.linspace(-7, 7, 2801)]).astype(np.float32)
    for x in xs:
        code = oracle.e2m1_encode(x)
        mag = abs(float(x))
        assert (code >> 3) == (1 if np.signbit(x) else 0)
        err = np.abs(table - min(mag, 6.0))
        best = np.flatnonzero(err == err.min())
        if best.size == 1:
            assert (code & 7) == best[0], x
        else:  # a tie: the even code wins
            assert (code & 7) in best and (code & 1) == 0, x


# -------------------------------------------------------------- quantizer

def _half_spacing(mag):
    return 0.25 if mag <= 2 else (0.5 if mag <= 4 else 1.0)


def test_group_quantizer_closed_form_bound_and_scale():
    for trial in range(3000):
        kind = trial % 4
        if kind == 0:
            x = RNG.standard_normal(16) * RNG.uniform(0.25, 4)
        elif kind == 1:
            x = RNG.standard_normal(16) * 10.0 ** RNG.uniform(-4, 2.5)
        elif kind == 2:
            x = RNG.standard_normal(16)
            x[RNG.integers(16)] = RNG.choice([-448.0, 448.0])
        else:
            x = np.zeros(16)
            x[RNG.integers(16)] = RNG.uniform(-3, 3)
        x = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).to(torch.float32).numpy()
        nib, sc = oracle.quantize_group(x)
        a = np.float32(np.max(np.abs(x)))
        # the scale is torch's E4M3 conversion of a/6 (both in FP32)
        assert sc == _torch_e4m3_code(np.array([np.float32(a) / np.float32(6.0)], np.float32))[0]
        s = oracle.e4m3_value(sc)
        if s == 0:
            assert np.all(nib == 0)
            continue
        for i in range(16):
            q = oracle.e2m1_value(int(nib[i]))
            y = float(np.float32(x[i]) / np.float32(s))
            if abs(y) > 6:
                assert abs(q) == 6.0 and np.sign(q) == np.sign(y)
            else:
                assert abs(y - q) <= _half_spacing(abs(y)) + 1e-12
            v = q * s
            assert float(np.float16(v)) == v  # exact in FP16


def test_all_zero_group():
    nib, sc = oracle.quantize_group(np.zeros(16, np.float32))
    assert sc == 0 and np.all(nib == 0)
    nib, sc = oracle.quantize_group(-np.zeros(16, np.float32))
    assert sc == 0 and np.all(nib == 0)


def test_rope_bytes_match_torch_e4m3():
    lat = torch.randn(64, 512).to(torch.bfloat16)
    rope = (torch.randn(64, 64) * 30).to(torch.bfloat16)
    rows = oracle.quantize_rows(lat.view(torch.int16).numpy().view(np.uint16),
                                rope.view(torch.int16).numpy().view(np.uint16))
    ref = rope.to(torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(rows[:, 288:], ref)


def test_row_layout_worked_example():
    # dim 0 -> code 1 (0.5), dim 1 -> code 2 (1.0) in byte 0; scale 0 = 2.0
    row = np.zeros((1, 352), np.uint8)
    row[0, 0] = 0x21
    row[0, 256] = 0x40  # E4M3 2.0
    row[0, 257] = 0x38  # E4M3 1.0 for dims 16..31
    row[0, 8] = 0xF7    # dims 16 (code 7 = 6.0) and 17 (code 15 = -6.0)
    row[0, 288] = 0xB8  # rope dim 0 = -1.0
    v = oracle.dequant_rows(row)[0]
    assert v[0] == 1.0 and v[1] == 2.0 and v[16] == 6.0 and v[17] == -6.0 and v[512] == -1.0
    assert np.count_nonzero(v) == 5


def test_quantize_dequantize_roundtrip_exact_fp16():
    lat = (torch.randn(200, 512) * (0.25 + 3.75 * torch.rand(512))).to(torch.bfloat16)
    rope = torch.randn(200, 64).to(torch.bfloat16)
    rows = oracle.quantize_rows(lat.view(torch.int16).numpy().view(np.uint16),
                                rope.view(torch.int16).numpy().view(np.uint16))
    v = oracle.dequant_rows(rows)
    assert np.array_equal(v.astype(np.float16).astype(np.float64), v)
    # relative error of the 4-bit format stays within its half-spacing bound
    ref = lat.to(torch.float64).numpy()
    scales = np.array([[oracle.e4m3_value(c) for c in r] for r in rows[:, 256:288]])
    bound = np.repeat(scales, 16, axis=1) * 1.0 + 1e-30
    assert np.all(np.abs(v[:, :512] - ref) <= bound * 1.0 + np.abs(ref) * 0.07)


def test_row_size_matches_pages():
    consts = {k: float(v) for k, v in read_golden("pages_constants.txt")}
    nibble_bytes = 512 // 2
    scale_bytes = 512 // int(consts["group_size"]) * int(consts["scales_per_group"])
    rope_bytes = 64
    assert nibble_bytes + scale_bytes + rope_bytes == consts["row_bytes_after"] == oracle.ROW_BYTES
    assert 512 + 64 == consts["row_bytes_before"] == oracle.STAGED_ROW_BYTES
    assert consts["row_bytes_before"] / consts["row_bytes_after"] == pytest.approx(18 / 11)


def test_capacity_ratio_consistent_with_row_sizes():
    consts = {k: float(v) for k, v in read_golden("pages_constants.txt")}
    ratio = consts["capacity_tokens_after"] / consts["capacity_tokens_before"]
    assert 1.0 < ratio <= consts["row_bytes_before"] / consts["row_bytes_after"]
    # the pages round to 3 significant digits: ~ +50%
    assert ratio == pytest.approx(1.5, abs=0.01)


# -------------------------------------------------------------- attention

def _cache(n, seed=0, scale=None):
    g = torch.Generator().manual_seed(seed)
    sc = scale if scale is not None else 0.25 + 3.75 * torch.rand(576, generator=g)
    x = (torch.randn(n, 576, generator=g) * sc).to(torch.bfloat16)
    lat = x[:, :512].contiguous().view(torch.int16).numpy().view(np.uint16)
    rope = x[:, 512:].contiguous().view(torch.int16).numpy().view(np.uint16)
    return oracle.quantize_rows(lat, rope)


def _q(T, H, seed=1):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(T, H, 576, generator=g).to(torch.float16).numpy()
    return np.ascontiguousarray(q[..., :512]), np.ascontiguousarray(q[..., 512:])


def _dense(qn, qr, K, scale):
    q = np.concatenate([qn, qr], axis=-1).astype(np.float64)
    s = scale * (q @ K.T)
    m = s.max(axis=-1, keepdims=True)
    p = np.exp(s - m)
    l = p.sum(axis=-1, keepdims=True)
    return (p @ K[:, :512]) / l, (m + np.log(l))[..., 0]


def test_full_selection_equals_dense_attention():
    n, H = 300, 4
    cache = _cache(n)
    qn, qr = _q(1, H)
    idx = np.arange(n, dtype=np.int32)[None, :]
    sm = 1 / math.sqrt(576)
    out, lse = oracle.sparse_mla(qn, qr, cache, idx, sm)
    K = oracle.dequant_rows(cache)
    ref_o, ref_l = _dense(qn[0], qr[0], K, f32(sm))
    np.testing.assert_allclose(out[0], ref_o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse[0], ref_l, rtol=1e-12, atol=1e-12)


def test_staged_variant_equals_dense_over_e4m3_values():
    n, H = 200, 3
    cache = _cache(n, seed=5)
    qn, qr = _q(1, H, seed=6)
    idx = np.arange(n, dtype=np.int32)[None, :]
    sm = 1 / math.sqrt(576)
    out, lse = oracle.sparse_mla(qn, qr, cache, idx, sm, staged=True)
    K = oracle.dequant_rows(cache)
    K8 = torch.from_numpy(K.astype(np.float32)).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref_o, ref_l = _dense(qn[0], qr[0], K8, f32(sm))
    np.testing.assert_allclose(out[0], ref_o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse[0], ref_l, rtol=1e-12, atol=1e-12)
    st = oracle.stage_rows(cache)
    assert np.array_equal(st, torch.from_numpy(K.astype(np.float32)).to(torch.float8_e4m3fn)
                          .view(torch.uint8).numpy())


def _bf16_rows(n, seed, scale):
    g = torch.Generator().manual_seed(seed)
    x = (torch.randn(n, 576, generator=g) * scale).to(torch.bfloat16)
    lat = x[:, :512].contiguous().view(torch.int16).numpy().view(np.uint16)
    rope = x[:, 512:].contiguous().view(torch.int16).numpy().view(np.uint16)
    return x.to(torch.float32), lat, rope


def test_fp8_rows_match_torch_e4m3_layout_and_saturation():
    # one E4M3 byte per dim, latent dims first then RoPE; values spread over
    # subnormals .. beyond the largest finite code
    sc = torch.exp(torch.linspace(math.log(1e-3), math.log(300.0), 576))
    x, lat, rope = _bf16_rows(64, 21, sc)
    rows = oracle.quantize_fp8_rows(lat, rope)
    assert rows.shape == (64, 576) and rows.dtype == np.uint8
    xs = x.numpy()
    inside = np.abs(xs) <= 448.0
    ref = _torch_e4m3_code(np.where(inside, xs, 0.0))
    assert np.array_equal(rows[inside], ref[inside])
    big = ~inside
    assert big.any()
    assert np.all(rows[big & (xs > 0)] == 0x7E) and np.all(rows[big & (xs < 0)] == 0xFE)
    assert oracle.quantize_fp8_rows(lat[:0], rope[:0]).shape == (0, 576)


def test_fp8_row_attention_equals_dense_over_selected_rows():
    n, H = 300, 3
    _, lat, rope = _bf16_rows(n, 22, 0.25 + 3.75 * torch.rand(576, generator=torch.Generator().manual_seed(23)))
    rows = oracle.quantize_fp8_rows(lat, rope)
    qn, qr = _q(1, H, seed=24)
    sel = np.random.default_rng(25).permutation(n)[:170].astype(np.int32)
    idx = np.concatenate([sel, -np.ones(30, np.int32)])[None, :]
    sm = 1 / math.sqrt(576)
    out, lse = oracle.sparse_mla(qn, qr, rows, idx, sm, fp8_rows=True)
    K = torch.from_numpy(rows[sel]).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ref_o, ref_l = _dense(qn[0], qr[0], K, f32(sm))
    np.testing.assert_allclose(out[0], ref_o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse[0], ref_l, rtol=1e-12, atol=1e-12)


def test_permutation_and_empty_entry_invariance():
    n, H, topk = 1000, 2, 2048
    cache = _cache(n, seed=2)
    qn, qr = _q(1, H, seed=3)
    sel = RNG.choice(n, 700, replace=False).astype(np.int32)
    idx = np.full((1, topk), -1, np.int32)
    idx[0, :700] = sel
    sm = 0.05
    o1, l1 = oracle.sparse_mla(qn, qr, cache, idx, sm)
    idx2 = idx.copy()
    idx2[0] = RNG.permutation(idx2[0])
    idx2[0, idx2[0] == -1] = RNG.choice([-1, -7, n, n + 5, -2**31], size=(idx2[0] == -1).sum())
    o2, l2 = oracle.sparse_mla(qn, qr, cache, idx2, sm)
    np.testing.assert_allclose(o1, o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(l1, l2, rtol=1e-12, atol=1e-12)


def test_single_valid_row_brute_force():
    cache = _cache(8, seed=4)
    K = oracle.dequant_rows(cache)
    qn = np.zeros((1, 1, 512), np.float16)
    qr = np.zeros((1, 1, 64), np.float16)
    qn[0, 0, 3] = 1.0
    qr[0, 0, 1] = -2.0
    idx = np.full((1, 2048), -1, np.int32)
    idx[0, 1000] = 5
    out, lse = oracle.sparse_mla(qn, qr, cache, idx, 0.5)
    assert np.array_equal(out[0, 0], K[5, :512])
    assert lse[0, 0] == 0.5 * (K[5, 3] - 2.0 * K[5, 513])


def test_two_equal_scores_average_and_ln2():
    cache = _cache(4, seed=7)
    K = oracle.dequant_rows(cache)
    qn = np.zeros((1, 1, 512), np.float16)
    qr = np.zeros((1, 1, 64), np.float16)
    idx = np.array([[1, 2] + [-1] * 2046], np.int32)
    out, lse = oracle.sparse_mla(qn, qr, cache, idx, 1.0)
    np.testing.assert_allclose(out[0, 0], (K[1, :512] + K[2, :512]) / 2, rtol=0, atol=1e-12)
    assert lse[0, 0] == pytest.approx(math.log(2), abs=1e-15)


def test_duplicate_index_counts_per_position():
    cache = _cache(4, seed=8)
    K = oracle.dequant_rows(cache)
    qn = np.zeros((1, 1, 512), np.float16)
    qr = np.zeros((1, 1, 64), np.float16)
    idx = np.array([[1, 1, 2]], np.int32)
    out, lse = oracle.sparse_mla(qn, qr, cache, idx, 1.0)
    np.testing.assert_allclose(out[0, 0], (2 * K[1, :512] + K[2, :512]) / 3, atol=1e-12)
    assert lse[0, 0] == pytest.approx(math.log(3), abs=1e-15)


def test_all_empty_list():
    cache = _cache(4, seed=9)
    qn, qr = _q(2, 2)
    idx = np.full((2, 2048), -1, np.int32)
    out, lse = oracle.sparse_mla(qn, qr, cache, idx, 1.0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_multi_token_heads_independent():
    # each (t, h) equals the single-token single-head computation
    cache = _cache(500, seed=10)
    qn, qr = _q(3, 5, seed=11)
    idx = np.stack([RNG.choice(500, 2048, replace=True).astype(np.int32) for _ in range(3)])
    idx[1, ::3] = -1
    out, lse = oracle.sparse_mla(qn, qr, cache, idx, 0.07)
    for t in range(3):
        for h in range(5):
            o1, l1 = oracle.sparse_mla(qn[t:t + 1, h:h + 1], qr[t:t + 1, h:h + 1], cache,
                                       idx[t:t + 1], 0.07)
            assert np.array_equal(o1[0, 0], out[t, h]) and l1[0, 0] == lse[t, h]
