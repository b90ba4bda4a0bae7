"""The sparse indexer on the GPU vs the CPU oracle.

Page "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
section "Four-bit caches make room": the indexer picks the rows each token's
attention reads and hands over 2,048 positions (scoring form and tie rule
are the readings stated in oracle/indexer.py).

* selection over given scores: bit-exact against the oracle, ties included;
* scores: the GPU accumulates the 128 exact E4M3 products of a head in FP32
  on the tensor cores and folds the 64 heads with FP32 fused multiply-adds.
  A sum of n terms in FP32 is within n * 2^-24 of the magnitude
  m = sum_h |w_h| * sum_d |q_hd * k_d| of the exact value, whatever the
  order; with n <= 128 + 64 that is below 2^-16 * m, the bound used here
  (plus 1e-6 absolute);
* full indexer: the list must be a valid top-k of the exact scores within
  that bound (every chosen score + its bound >= every unchosen score - its
  bound), in increasing position order, with min(topk, ctx) entries."""
import math

import numpy as np
import pytest
import torch

import nvfp4_sparse_mla_decode_b200 as nv
from nvfp4_sparse_mla_decode_b200 import synth
from oracle import indexer

pytestmark = pytest.mark.gpu

REL = 2.0 ** -16
ABS = 1e-6


def _table(ctx, page, seed, spare_pages=3):
    need = [max(1, math.ceil(c / page)) for c in ctx]
    num_pages = sum(need) + spare_pages
    perm = np.random.default_rng(seed).permutation(num_pages)
    table = np.full((len(ctx), max(need) + 1), -1, dtype=np.int32)
    at = 0
    for t, k in enumerate(need):
        table[t, :k] = perm[at:at + k]
        at += k
    return table, num_pages * page


CASES = ["normal", "ties", "signed_zeros", "neg_inf", "alternating_lines", "rising", "first_part_high",
         "all_neg_inf", "constant", "pos_inf_spikes"]


def _scores(case, T, stride, seed):
    g = torch.Generator().manual_seed(seed)
    s = torch.randn(T, stride, generator=g)
    if case == "ties":                   # far more equal scores at the top than topk
        s = torch.randint(-3, 4, (T, stride), generator=g).float()
    elif case == "signed_zeros":
        s = torch.zeros(T, stride)
        s[:, ::3] = -0.0
        s[:, ::7] = 1.0
    elif case == "neg_inf":
        s[:, ::5] = -math.inf
    elif case == "alternating_lines":    # every other 32-position line constant
        line = torch.arange(stride) // 32
        s = torch.where((line % 2 == 1)[None, :], torch.ones_like(s), s)
    elif case == "rising":               # scores grow with position
        s = s * 0.01 + torch.arange(stride, dtype=torch.float32)[None, :] / 1000
    elif case == "first_part_high":      # one part's own threshold lies above the row's
        s[:, :stride // 8] += 100.0
    elif case == "all_neg_inf":          # every position a candidate: the general path's radix select
        s = torch.full((T, stride), -math.inf)
    elif case == "constant":             # one key everywhere: ties decide by position
        s = torch.full((T, stride), 0.5)
    elif case == "pos_inf_spikes":       # +inf above every finite score
        s[:, 7::997] = math.inf
    return s


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("topk", [2048, 100, 1])
def test_topk_matches_oracle(case, topk):
    ctx = [0, 1, 99, 100, 2047, 2048, 2049, 5000, 33333, 140000]
    T, max_ctx = len(ctx), max(ctx)
    stride = nv.indexer_score_stride(max_ctx)
    s = _scores(case, T, stride, CASES.index(case) * 10007 + topk)
    pos = nv.indexer_topk(s.cuda(), torch.tensor(ctx, dtype=torch.int32, device="cuda"), max_ctx, topk)
    ref = indexer.topk_positions([s[t, :ctx[t]].double().numpy() for t in range(T)], topk)
    got = pos.cpu().numpy()
    bad = [t for t in range(T) if not np.array_equal(got[t], ref[t])]
    assert not bad, "tokens %s differ" % bad


@pytest.mark.parametrize("case", ["normal", "ties", "neg_inf"])
def test_topk_rows_longer_than_eight_ctas_hold(case):
    # more than 8 x 53,248 positions: the row is streamed, not held on chip
    ctx = [450000, 430001]
    T, max_ctx = len(ctx), max(ctx)
    stride = nv.indexer_score_stride(max_ctx)
    s = _scores(case, T, stride, 77 + CASES.index(case))
    pos = nv.indexer_topk(s.cuda(), torch.tensor(ctx, dtype=torch.int32, device="cuda"), max_ctx, 2048)
    ref = indexer.topk_positions([s[t, :ctx[t]].double().numpy() for t in range(T)], 2048)
    got = pos.cpu().numpy()
    assert all(np.array_equal(got[t], ref[t]) for t in range(T))


@pytest.mark.parametrize("T,top_ctx", [(160, 50000), (60, 100000), (200, 140000)])
def test_topk_many_requests(T, top_ctx):
    # one CTA or two per request, and more requests than the device holds
    # at once: clusters run in waves
    ctx = [top_ctx - (977 * t) % (top_ctx // 2) for t in range(T)]
    max_ctx = max(ctx)
    stride = nv.indexer_score_stride(max_ctx)
    s = _scores("normal", T, stride, 9000 + T)
    g = torch.Generator().manual_seed(T)
    s[T // 3, :] = torch.randint(-3, 4, (stride,), generator=g).float()  # one request on the radix path
    pos = nv.indexer_topk(s.cuda(), torch.tensor(ctx, dtype=torch.int32, device="cuda"), max_ctx, 2048)
    ref = indexer.topk_positions([s[t, :ctx[t]].double().numpy() for t in range(T)], 2048)
    got = pos.cpu().numpy()
    bad = [t for t in range(T) if not np.array_equal(got[t], ref[t])]
    assert not bad, "tokens %s differ" % bad


@pytest.mark.parametrize("T", [1, 3, 35])
def test_topk_workspace_reused_across_calls(T):
    # rows split over several CTAs meet on counters in the workspace; every
    # call must leave them ready for the next
    ctx = [140000 - 977 * t for t in range(T)]
    stride = nv.indexer_score_stride(max(ctx))
    ws = torch.zeros(max(256, nv.lib().nvfp4mla_indexer_topk_workspace_size(T)), dtype=torch.uint8, device="cuda")
    lens = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    for call, case in enumerate(["normal", "rising", "ties", "normal"]):
        s = _scores(case, T, stride, 500 + call)
        pos = nv.indexer_topk(s.cuda(), lens, max(ctx), 2048, workspace=ws).cpu().numpy()
        ref = indexer.topk_positions([s[t, :ctx[t]].double().numpy() for t in range(T)], 2048)
        assert np.array_equal(pos, ref), "call %d (%s)" % (call, case)


def _check_scores(sc, ref, mag, ctx):
    worst = 0.0
    for t in range(len(ctx)):
        got = sc[t, :ctx[t]].double().cpu().numpy()
        err = np.abs(got - ref[t])
        bound = REL * mag[t] + ABS
        assert np.all(np.isfinite(got))
        assert np.all(err <= bound), "token %d: worst err/bound %.3g" % (t, float((err / bound).max()))
        if err.size:
            worst = max(worst, float((err / bound).max()))
    return worst


@pytest.mark.parametrize("page", [8, 16, 64, 128, 256])
def test_scores_match_oracle(page):
    ctx = [1, 127, 128, 129, 3000, 10000]
    T = len(ctx)
    table, num_slots = _table(ctx, page, 40 + page)
    keys = synth.indexer_keys(num_slots, 41, "cuda")
    q, w = synth.indexer_queries(T, 42, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sc = nv.indexer_scores(q, w, keys, torch.from_numpy(table).cuda(), page,
                           torch.tensor(ctx, dtype=torch.int32, device="cuda"), max(ctx), dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref, mag = indexer.indexer_scores(q.cpu().numpy(), w.cpu().numpy(), keys.cpu().numpy(), table, ctx, page,
                                      magnitude=True)
    _check_scores(sc, ref, mag, ctx)


def test_missing_pages_score_minus_inf_and_flag():
    page, ctx = 64, [1000, 1000]
    table, num_slots = _table(ctx, page, 50)
    table[0, 3] = -1                     # an empty table entry inside the context
    table[1, 5] = num_slots // page      # a page past the end of the key cache
    keys = synth.indexer_keys(num_slots, 51, "cuda")
    q, w = synth.indexer_queries(2, 52, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    sc = nv.indexer_scores(q, w, keys, torch.from_numpy(table).cuda(), page,
                           torch.tensor(ctx, dtype=torch.int32, device="cuda"), 1000, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & nv.DEV_BAD_INDEX
    sc = sc.cpu()
    assert torch.all(torch.isneginf(sc[0, 192:256])) and torch.all(torch.isneginf(sc[1, 320:384]))
    good = table.copy()
    good[0, 3] = good[0, 4]
    good[1, 5] = good[1, 4]
    ref, mag = indexer.indexer_scores(q.cpu().numpy(), w.cpu().numpy(), keys.cpu().numpy(), good, ctx, page,
                                      magnitude=True)
    keep0 = np.r_[0:192, 256:1000]
    keep1 = np.r_[0:320, 384:1000]
    for t, keep in ((0, keep0), (1, keep1)):
        err = np.abs(sc[t, keep].double().numpy() - ref[t][keep])
        assert np.all(err <= REL * mag[t][keep] + ABS)


def _valid_topk(pos, ref, mag, ctx, topk):
    n = min(topk, ctx)
    assert np.all(pos[n:] == -1)
    sel = pos[:n]
    assert np.all(np.diff(sel) > 0) and sel[0] >= 0 and sel[-1] < ctx
    if ctx <= topk:
        assert np.array_equal(sel, np.arange(ctx))
        return
    e = REL * mag + ABS
    chosen = np.zeros(ctx, dtype=bool)
    chosen[sel] = True
    assert (ref + e)[chosen].min() >= (ref - e)[~chosen].max()


def test_sparse_indexer_long_contexts_sampled_tokens():
    # 35 requests of 140,000 positions in a paged key cache (page 64)
    T, ctx, page = 35, 140_000, 64
    tables = synth.page_tables([ctx] * T, T * math.ceil(ctx / page), 60, "cuda")
    table = torch.stack([tb.to(torch.int32) for tb in tables])
    num_slots = T * math.ceil(ctx / page) * page
    keys = synth.indexer_keys(num_slots, 61, "cuda")
    q, w = synth.indexer_queries(T, 62, "cuda")
    lens = torch.full((T,), ctx, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = nv.sparse_indexer(q, w, keys, table, page, lens, ctx, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    tok = [0, 17, 34]
    rows = lambda s: keys[torch.from_numpy(s).cuda()].cpu().numpy()  # noqa: E731
    ref, mag = indexer.indexer_scores(q.cpu().numpy(), w.cpu().numpy(), rows, table.cpu().numpy(), [ctx] * T,
                                      page, tokens=tok, magnitude=True)
    p = pos.cpu().numpy()
    for i, t in enumerate(tok):
        _valid_topk(p[t], ref[i], mag[i], ctx, 2048)


def test_sparse_indexer_short_and_ragged_contexts():
    ctx = [0, 5, 2048, 2049, 4100, 777]
    page = 16
    table, num_slots = _table(ctx, page, 70)
    keys = synth.indexer_keys(num_slots, 71, "cuda")
    q, w = synth.indexer_queries(len(ctx), 72, "cuda")
    pos = nv.sparse_indexer(q, w, keys, torch.from_numpy(table).cuda(), page,
                            torch.tensor(ctx, dtype=torch.int32, device="cuda"), max(ctx)).cpu().numpy()
    ref, mag = indexer.indexer_scores(q.cpu().numpy(), w.cpu().numpy(), keys.cpu().numpy(), table, ctx, page,
                                      magnitude=True)
    for t in range(len(ctx)):
        if ctx[t] == 0:
            assert np.all(pos[t] == -1)
        else:
            _valid_topk(pos[t], ref[t], mag[t], ctx[t], 2048)


def test_indexer_lists_feed_the_paged_decode():
    # the indexer's positions are the paged decode's input as they stand: the
    # list is a valid top-k of the oracle's scores, and the decode over it
    # matches the oracle's decode over the same positions, translated to
    # slots through the block table by the plain definition
    w = synth.decode35("cuda", T=4, ctx=20000)
    from nvfp4_sparse_mla_decode_b200.cache import build_cache
    from harness import check_close, oracle_decode, translate
    cache = build_cache(w)
    table = synth.block_table(w)
    keys = synth.indexer_keys(w.num_slots, 81, "cuda")
    q, wt = synth.indexer_queries(w.T, 82, "cuda")
    lens = torch.tensor(w.ctx_lens, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos = nv.sparse_indexer(q, wt, keys, table, synth.PAGE_SIZE, lens, max(w.ctx_lens), dev_status=status)
    out, lse = nv.decode_paged(w.q_nope, w.q_rope, cache, pos, table, synth.PAGE_SIZE, w.sm_scale,
                               dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    pos_h = pos.cpu().numpy()
    ref, mag = indexer.indexer_scores(q.cpu().numpy(), wt.cpu().numpy(), keys.cpu().numpy(), table.cpu().numpy(),
                                      list(w.ctx_lens), synth.PAGE_SIZE, magnitude=True)
    for t in range(w.T):
        _valid_topk(pos_h[t], ref[t], mag[t], w.ctx_lens[t], 2048)
    slots = translate(pos_h, table.cpu().numpy(), synth.PAGE_SIZE, w.num_slots)
    w.indices = torch.from_numpy(slots.astype(np.int32)).to("cuda")
    ref_o, ref_l = oracle_decode(w, range(w.T))
    check_close(out, lse, ref_o, ref_l)
