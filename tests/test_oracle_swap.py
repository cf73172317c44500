"""Oracle of swap_blocks (zwxr.cn 4.3, preemption by swapping): whole blocks
move from one pool to another.  Pinned against numpy fancy indexing, which
states the same definition independently, and by a swap-out / swap-in round
trip that must restore every byte of the moved blocks."""
import numpy as np
import pytest
import torch


def _pools(nb, layers, shape, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda: torch.randint(0, 256, (nb,) + shape, generator=g, dtype=torch.uint8).view(dtype)
    return [mk() for _ in range(layers)], [mk() for _ in range(layers)]


@pytest.mark.parametrize("dtype,shape", [(torch.uint8, (32, 2, 64)), (torch.bfloat16, (16, 8, 128))])
def test_swap_matches_fancy_indexing(orc, dtype, shape):
    sk, sv = _pools(40, 3, shape, dtype, seed=1)
    dk, dv = _pools(25, 3, shape, dtype, seed=2)
    src = torch.randperm(40, generator=torch.Generator().manual_seed(3))[:17]
    dst = torch.randperm(25, generator=torch.Generator().manual_seed(4))[:17]
    mapping = torch.stack([src, dst], 1)
    want_k = [d.view(torch.uint8).numpy().copy() for d in dk]
    want_v = [d.view(torch.uint8).numpy().copy() for d in dv]
    for l in range(3):
        want_k[l][dst.numpy()] = sk[l].view(torch.uint8).numpy()[src.numpy()]
        want_v[l][dst.numpy()] = sv[l].view(torch.uint8).numpy()[src.numpy()]
    orc.swap_blocks(dk, dv, sk, sv, mapping)
    for l in range(3):
        assert np.array_equal(dk[l].view(torch.uint8).numpy(), want_k[l])
        assert np.array_equal(dv[l].view(torch.uint8).numpy(), want_v[l])


def test_swap_round_trip_restores_blocks(orc):
    # device pool -> host pool (swap out), host -> other device blocks (swap in)
    gk, gv = _pools(30, 2, (16, 4, 64), torch.float16, seed=5)
    hk, hv = _pools(12, 2, (16, 4, 64), torch.float16, seed=6)
    out_map = torch.tensor([[3, 0], [17, 5], [29, 11]])
    in_map = torch.tensor([[0, 8], [5, 9], [11, 10]])
    before = [gk[l][[3, 17, 29]].clone() for l in range(2)] + [gv[l][[3, 17, 29]].clone() for l in range(2)]
    orc.swap_blocks(hk, hv, gk, gv, out_map)
    orc.swap_blocks(gk, gv, hk, hv, in_map)
    after = [gk[l][[8, 9, 10]] for l in range(2)] + [gv[l][[8, 9, 10]] for l in range(2)]
    for a, b in zip(before, after):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_swap_rejects_out_of_range_ids(orc):
    sk, sv = _pools(4, 1, (16, 1, 64), torch.uint8, seed=7)
    dk, dv = _pools(4, 1, (16, 1, 64), torch.uint8, seed=8)
    with pytest.raises(ValueError):
        orc.swap_blocks(dk, dv, sk, sv, torch.tensor([[0, 4]]))
