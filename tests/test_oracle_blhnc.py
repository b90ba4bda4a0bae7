"""Pins of the block-major layout oracle (CPU).

Page "Prime Intellect Launches Prime Inference, Serving 600B Tokens Daily",
section "Fewer copies unlock NVLink": the block-major layout keeps every
layer of a block together, with blocks a sixteenth of the earlier size, and
cut a transfer's copy descriptors from 19,559 to about 1,940.  The byte
layout and the descriptor rule are readings (oracle/blhnc.py); the checks
compare them with an independent reshape/transpose formulation, inverses,
closed forms and brute-force counts."""
import numpy as np
import pytest

from oracle import blhnc

RNG = np.random.default_rng(77)


def _caches(L, num_blocks, N, C, seed):
    g = np.random.default_rng(seed)
    return [g.integers(0, 256, size=(num_blocks, N, C), dtype=np.uint8) for _ in range(L)]


@pytest.mark.parametrize("sub", [1, 2, 4, 16])
def test_convert_equals_transpose_formulation(sub):
    L, nb_all, N, C = 3, 20, 16, 32
    caches = _caches(L, nb_all, N, C, sub)
    ids = RNG.choice(nb_all, size=7, replace=False)
    new_ids = np.arange(7 * sub)                      # a packed transfer buffer
    got = blhnc.convert(caches, ids, sub, new_ids, 7 * sub)
    # [L, nb_all, N, C] -> request blocks [L, nb, sub, n, C] -> [nb, sub, L, n, C]
    x = np.stack(caches)[:, ids].reshape(L, 7, sub, N // sub, C).transpose(1, 2, 0, 3, 4)
    assert np.array_equal(got, x.reshape(7 * sub, L, N // sub, C))


def test_convert_scatters_to_given_new_blocks_and_back():
    L, nb_all, N, C, sub = 4, 30, 64, 352, 16
    caches = _caches(L, nb_all, N, C, 5)
    ids = np.array([3, 4, 5, 17, 9])
    new_ids = RNG.permutation(200)[: ids.size * sub]
    out = blhnc.convert(caches, ids, sub, new_ids, 200, fill=0xAB)
    assert np.all(out[np.setdiff1d(np.arange(200), new_ids)] == 0xAB)   # untouched blocks
    # block d = new_ids[i*sub + j] holds positions 4j..4j+3 of block ids[i], every layer
    i, j, l = 3, 11, 2
    assert np.array_equal(out[new_ids[i * sub + j], l], caches[l][ids[i], 4 * j:4 * j + 4])
    zeroed = [c.copy() for c in caches]
    for c in zeroed:
        c[ids] = 0
    back = blhnc.convert_back(out, zeroed, ids, sub, new_ids)
    for c, b in zip(caches, back):
        assert np.array_equal(c, b)


def test_byte_count_is_preserved():
    L, N, C, sub = 5, 32, 48, 8
    caches = _caches(L, 12, N, C, 9)
    ids = np.arange(6)
    out = blhnc.convert(caches, ids, sub, np.arange(6 * sub), 6 * sub)
    assert out.size == ids.size * N * L * C


def test_runs_brute_force():
    for _ in range(200):
        ids = RNG.integers(0, 12, size=int(RNG.integers(0, 10)))
        brute = sum(1 for k in range(ids.size) if k == 0 or ids[k] != ids[k - 1] + 1)
        assert blhnc.runs(ids) == brute


def test_descriptor_closed_forms():
    L = 78
    contiguous = np.arange(100, 400)
    assert blhnc.descriptors_layer_major(contiguous, L) == L
    scattered = np.arange(0, 600, 2)                 # no two consecutive
    assert blhnc.descriptors_layer_major(scattered, L) == L * 300
    # block-major blocks placed at b * 16 + j keep the runs of the old ids
    new = (scattered[:, None] * 16 + np.arange(16)[None, :]).reshape(-1)
    assert blhnc.descriptors_block_major(new) == 300
    assert blhnc.descriptors_block_major(np.arange(4800)) == 1
    assert blhnc.descriptors_block_major(RNG.permutation(4800)[:0]) == 0
