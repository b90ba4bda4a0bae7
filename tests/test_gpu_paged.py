"""Decode over request-local positions with the position -> slot translation
done inside the launch (block table).  The translated launch must equal the
slot-id launch bit for bit (same rows, same order), and the oracle's own
translation of the positions must give the same results within tolerance."""
import numpy as np
import pytest
import torch

import nvfp4_sparse_mla_decode_b200 as nv
from nvfp4_sparse_mla_decode_b200 import synth
from harness import build_cache, check_close, oracle_decode, translate

pytestmark = pytest.mark.gpu
PAGE = synth.PAGE_SIZE


def run_paged(w, cache, positions, table, page):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, lse = nv.decode_paged(w.q_nope, w.q_rope, cache, positions, table, page, w.sm_scale, dev_status=status)
    torch.cuda.synchronize()
    return out, lse, int(status.item())


def test_paged_equals_slot_lists_and_oracle():
    w = synth.per_request("cuda", [20000] * 12, 64, seed=81, name="paged12")   # S = 8
    cache = build_cache(w)
    table = synth.block_table(w)
    pos = w.positions.contiguous()
    slots = translate(pos.cpu().numpy(), table.cpu().numpy(), PAGE, w.num_slots)
    assert np.array_equal(slots, w.indices.cpu().numpy())   # the oracle's translation agrees with the lists
    out_p, lse_p, st = run_paged(w, cache, pos, table, PAGE)
    assert st == 0
    out_s, lse_s = nv.decode(w.q_nope, w.q_rope, cache, w.indices, w.sm_scale)
    torch.cuda.synchronize()
    assert torch.equal(out_p, out_s) and torch.equal(lse_p, lse_s)
    ref_o, ref_l = oracle_decode(w, [0, 5, 11])
    check_close(out_p[[0, 5, 11]], lse_p[[0, 5, 11]], ref_o, ref_l)


def test_paged_empty_and_invalid_entries():
    w = synth.per_request("cuda", [9000] * 4, 64, seed=82, name="paged_bad")
    cache = build_cache(w)
    table = synth.block_table(w)
    pos = w.positions.clone()
    pos[0, 100:200] = -1                              # empty
    pos[1, ::7] = table.shape[1] * PAGE + 5           # beyond the table: empty, flagged
    pos[2, :50] = -3                                  # below -1: empty, flagged
    table[3, 0] = -1                                  # a missing page: entries on it are empty, flagged
    out, lse, st = run_paged(w, cache, pos.contiguous(), table, PAGE)
    assert st & nv.DEV_BAD_INDEX
    slots = translate(pos.cpu().numpy(), table.cpu().numpy(), PAGE, w.num_slots)
    w.indices = torch.from_numpy(slots.astype(np.int32)).to("cuda")
    ref_o, ref_l = oracle_decode(w, range(4))
    check_close(out, lse, ref_o, ref_l)


def test_page_size_16_table_gives_identical_results():
    w = synth.per_request("cuda", [6000] * 6, 128, seed=83, name="paged16")
    cache = build_cache(w)
    t64 = synth.block_table(w)
    # the same slots described with 16-slot pages: page q of 16 = 4 * page64 + q % 4
    t16 = (t64.repeat_interleave(4, dim=1) * 4 + torch.arange(4, device="cuda").repeat(t64.shape[1])).to(torch.int32)
    t16[t64.repeat_interleave(4, dim=1) < 0] = -1
    pos = w.positions.contiguous()
    out64, lse64, st64 = run_paged(w, cache, pos, t64, 64)
    out16, lse16, st16 = run_paged(w, cache, pos, t16.contiguous(), 16)
    assert st64 == 0 and st16 == 0
    assert torch.equal(out64, out16) and torch.equal(lse64, lse16)


def test_paged_zero_tokens_is_noop():
    cache = torch.zeros(16, nv.ROW_BYTES, dtype=torch.uint8, device="cuda")
    qn = torch.empty(0, 64, 512, dtype=torch.float16, device="cuda")
    qr = torch.empty(0, 64, 64, dtype=torch.float16, device="cuda")
    pos = torch.empty(0, 2048, dtype=torch.int32, device="cuda")
    table = torch.empty(0, 4, dtype=torch.int32, device="cuda")
    out, lse = nv.decode_paged(qn, qr, cache, pos, table, 64, 0.1)
    assert out.numel() == 0
