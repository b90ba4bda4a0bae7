"""Block-major multi-layer layout conversion on the GPU vs the CPU oracle:
bit-exact (page "Prime Intellect Launches Prime Inference, Serving 600B
Tokens Daily", section "Fewer copies unlock NVLink"; the byte layout is the
reading stated in oracle/blhnc.py)."""
import numpy as np
import pytest
import torch

import nvfp4_sparse_mla_decode_b200 as nv
from oracle import blhnc

pytestmark = pytest.mark.gpu


def _setup(L, num_blocks, N, C, nb, sub, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    caches = [torch.randint(0, 256, (num_blocks, N, C), generator=g, device="cuda", dtype=torch.int32)
              .to(torch.uint8) for _ in range(L)]
    rng = np.random.default_rng(seed)
    ids = rng.choice(num_blocks, size=nb, replace=False).astype(np.int32)
    num_new = nb * sub + 37
    new_ids = rng.choice(num_new, size=nb * sub, replace=False).astype(np.int32)
    return caches, ids, new_ids, num_new


@pytest.mark.parametrize("L,N,C,sub", [(1, 64, 352, 16), (3, 64, 352, 4), (8, 64, 352, 1), (5, 32, 576, 16),
                                       (2, 16, 16, 16)])
def test_convert_and_back_bit_exact(L, N, C, sub):
    num_blocks, nb = 300, 57
    caches, ids, new_ids, num_new = _setup(L, num_blocks, N, C, nb, sub, L * 1000 + N + C + sub)
    out = torch.full((num_new, L, N // sub, C), 0xAB, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.blhnc_convert(caches, torch.from_numpy(ids).cuda(), torch.from_numpy(new_ids).cuda(), out, sub,
                     to_blhnc=True, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    host = [c.cpu().numpy() for c in caches]
    ref = blhnc.convert(host, ids, sub, new_ids, num_new, fill=0xAB)
    assert np.array_equal(out.cpu().numpy(), ref)
    # back into zeroed copies of the request's blocks
    back = [c.clone() for c in caches]
    for c in back:
        c[torch.from_numpy(ids).long().cuda()] = 0
    nv.blhnc_convert(back, torch.from_numpy(ids).cuda(), torch.from_numpy(new_ids).cuda(), out, sub,
                     to_blhnc=False, dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for c, b in zip(caches, back):
        assert torch.equal(c, b)


def test_bad_ids_are_skipped_and_flagged():
    L, N, C, sub = 2, 64, 352, 16
    caches, ids, new_ids, num_new = _setup(L, 50, N, C, 6, sub, 9)
    ids[2] = 50                      # past the per-layer caches
    new_ids[5] = num_new + 3         # past the block-major cache
    out = torch.full((num_new, L, N // sub, C), 0xAB, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.blhnc_convert(caches, torch.from_numpy(ids).cuda(), torch.from_numpy(new_ids).cuda(), out, sub,
                     dev_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) & nv.DEV_BAD_INDEX
    host = [c.cpu().numpy() for c in caches]
    o = out.cpu().numpy()
    for i in range(6):
        for j in range(sub):
            d = new_ids[i * sub + j]
            if i == 2 or d >= num_new:
                if d < num_new:
                    assert np.all(o[d] == 0xAB)
                continue
            for l in range(L):
                assert np.array_equal(o[d, l], host[l][ids[i], 4 * j:4 * j + 4])
