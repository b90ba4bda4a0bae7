"""Pins of the sparse indexer oracle (CPU).

Page "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
section "Four-bit caches make room": the indexer picks each token's rows and
hands over 2,048 positions.  The scoring form and the tie rule are readings
(stated in oracle/indexer.py); every check below compares the oracle with
something other than itself: brute force over all subsets, torch's own
E4M3 decoder and contraction, closed forms and invariants."""
import itertools

import numpy as np
import torch

from oracle import indexer

RNG = np.random.default_rng(2024)


def _dominates(s, a, b):
    # position a must come before position b in the selection order
    return s[a] > s[b] or (s[a] == s[b] and a < b)


def test_selection_equals_brute_force_over_all_subsets():
    for trial in range(60):
        n = int(RNG.integers(2, 9))
        k = int(RNG.integers(1, n))
        s = RNG.integers(-2, 3, size=n).astype(np.float64)    # many ties
        winners = []
        for sub in itertools.combinations(range(n), k):
            rest = [u for u in range(n) if u not in sub]
            if all(_dominates(s, a, b) for a in sub for b in rest):
                winners.append(sub)
        assert len(winners) == 1
        got = indexer.topk_positions([s], k)[0]
        assert list(got) == list(winners[0])


def test_short_and_empty_contexts_list_every_position():
    got = indexer.topk_positions([np.zeros(5), np.zeros(0), -np.arange(7.0)], 6)
    assert list(got[0]) == [0, 1, 2, 3, 4, -1]
    assert list(got[1]) == [-1] * 6
    assert list(got[2]) == [0, 1, 2, 3, 4, 5]


def test_equal_scores_take_the_first_positions_and_signed_zeros_tie():
    s = np.zeros(10)
    s[1::2] = -0.0
    assert list(indexer.topk_positions([s], 4)[0]) == [0, 1, 2, 3]
    s = np.array([1.0, 3.0, 3.0, 2.0, 3.0, 3.0])
    assert list(indexer.topk_positions([s], 3)[0]) == [1, 2, 4]


def _codes(shape, scale=1.0, seed=0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=g) * scale
    return x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _torch_scores(q, w, keys, slots):
    K = torch.from_numpy(keys[slots]).view(torch.float8_e4m3fn).to(torch.float64)
    Q = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64)
    S = torch.einsum("pd,hd->ph", K, Q)
    return (torch.relu(S) * torch.from_numpy(w.astype(np.float64))[None, :]).sum(dim=1).numpy(), S.numpy()


def _paged(T, ctx, page, seed):
    # each request owns a random set of pages of a shared key cache
    need = [(c + page - 1) // page for c in ctx]
    perm = np.random.default_rng(seed).permutation(sum(need))
    table = np.full((T, max(need)), -1, dtype=np.int32)
    at = 0
    for t, k in enumerate(need):
        table[t, :k] = perm[at:at + k]
        at += k
    return table, sum(need) * page


def test_scores_equal_torch_decode_and_contraction():
    T, page = 3, 16
    ctx = [50, 17, 200]
    table, n = _paged(T, ctx, page, 1)
    keys = _codes((n, 128), 1.5, 2)
    q = _codes((T, 64, 128), 1.0, 3)
    w = np.random.default_rng(4).normal(size=(T, 64)).astype(np.float32)
    got, mag = indexer.indexer_scores(q, w, keys, table, ctx, page, magnitude=True)
    for t in range(T):
        slots = indexer.context_slots(table[t], ctx[t], page)
        ref, _ = _torch_scores(q[t], w[t], keys, slots)
        np.testing.assert_allclose(got[t], ref, rtol=1e-13, atol=1e-13)
        assert np.all(np.abs(got[t]) <= mag[t] + 1e-12)


def test_one_hot_query_reads_one_key_dim():
    page, ctx = 8, 40
    table, n = _paged(1, [ctx], page, 5)
    keys = _codes((n, 128), 2.0, 6)
    q = np.zeros((1, 64, 128), dtype=np.uint8)
    h0, d0 = 17, 93
    q[0, h0, d0] = 0x38                      # E4M3 1.0
    w = np.zeros((1, 64), dtype=np.float32)
    w[0, h0] = 2.0
    got = indexer.indexer_scores(q, w, keys, table, [ctx], page)[0]
    slots = indexer.context_slots(table[0], ctx, page)
    kd = torch.from_numpy(keys[slots, d0].copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(got, 2.0 * np.maximum(kd, 0.0))


def test_relu_difference_is_linear_in_q():
    # relu(x) - relu(-x) = x: scores(q) - scores(-q) = sum_h w_h (q_h . k)
    page, ctx = 32, 100
    table, n = _paged(1, [ctx], page, 7)
    keys = _codes((n, 128), 1.0, 8)
    q = _codes((1, 64, 128), 1.0, 9)
    w = np.random.default_rng(10).normal(size=(1, 64)).astype(np.float32)
    neg = q ^ np.uint8(0x80)
    a = indexer.indexer_scores(q, w, keys, table, [ctx], page)[0]
    b = indexer.indexer_scores(neg, w, keys, table, [ctx], page)[0]
    slots = indexer.context_slots(table[0], ctx, page)
    _, S = _torch_scores(q[0], w[0], keys, slots)
    np.testing.assert_allclose(a - b, S @ w[0].astype(np.float64), rtol=1e-12, atol=1e-10)


def test_moving_pages_with_the_table_leaves_scores_unchanged():
    page, ctx = 16, 130
    table, n = _paged(1, [ctx], page, 11)
    keys = _codes((n, 128), 1.0, 12)
    q = _codes((1, 64, 128), 1.0, 13)
    w = np.random.default_rng(14).normal(size=(1, 64)).astype(np.float32)
    a = indexer.indexer_scores(q, w, keys, table, [ctx], page)[0]
    perm = np.random.default_rng(15).permutation(n // page)       # new page of old page i: perm[i]
    moved = np.empty_like(keys)
    for i in range(n // page):
        moved[perm[i] * page:(perm[i] + 1) * page] = keys[i * page:(i + 1) * page]
    table2 = np.where(table >= 0, perm[np.maximum(table, 0)], -1).astype(np.int32)
    b = indexer.indexer_scores(q, w, moved, table2, [ctx], page)[0]
    np.testing.assert_array_equal(a, b)


def test_full_indexer_picks_the_planted_rows():
    # keys equal to +q direction for a few planted positions score highest
    page, ctx, k = 64, 3000, 16
    table, n = _paged(1, [ctx], page, 16)
    keys = _codes((n, 128), 0.1, 17)
    q = np.full((1, 64, 128), 0x38, dtype=np.uint8)                 # all ones
    w = np.full((1, 64), 1.0 / 64, dtype=np.float32)
    planted = np.sort(np.random.default_rng(18).choice(ctx, size=k, replace=False))
    slots = indexer.context_slots(table[0], ctx, page)
    keys[slots[planted]] = 0x40                                      # E4M3 2.0
    pos, _ = indexer.sparse_indexer(q, w, keys, table, [ctx], page, k)
    assert list(pos[0]) == list(planted)


def test_context_slots_worked_example():
    # pages of 4: positions 0-3 in page 3, 4-7 in page 0, 8-9 in page 2
    got = indexer.context_slots(np.array([3, 0, 2, -1]), 10, 4)
    assert list(got) == [12, 13, 14, 15, 0, 1, 2, 3, 8, 9]
