"""swap_blocks on the GPU (zwxr.cn 4.3, preemption by swapping): whole blocks
between device pools and page-locked host pools, bit-exact against the
oracle; a preempted batch swapped out, its device blocks reused, swapped back
into other blocks, decodes to the same bits."""
import ctypes

import pytest
import torch

import oracle as orc
import paged_kv_cache_373_b200 as pkv
from paged_kv_cache_373_b200 import workloads as W
from pkv_testutil import gpu_inputs

pytestmark = pytest.mark.gpu


def _pools(nb, layers, shape, dtype, seed, where):
    g = torch.Generator().manual_seed(seed)
    mk = lambda: torch.randint(0, 256, (nb,) + shape, generator=g, dtype=torch.uint8).view(dtype)
    ks, vs = [mk() for _ in range(layers)], [mk() for _ in range(layers)]
    if where == "cuda":
        return [t.cuda() for t in ks], [t.cuda() for t in vs]
    if where == "pinned":
        return [t.pin_memory() for t in ks], [t.pin_memory() for t in vs]
    return ks, vs


def _mapping(n_src, n_dst, pairs, seed):
    g = torch.Generator().manual_seed(seed)
    src = torch.randperm(n_src, generator=g)[:pairs]
    dst = torch.randperm(n_dst, generator=g)[:pairs]
    return torch.stack([src, dst], 1).to(torch.int64)


@pytest.mark.parametrize("src_where,dst_where,map_where", [
    ("cuda", "pinned", "cuda"),     # swap out
    ("pinned", "cuda", "cuda"),     # swap in
    ("cuda", "cuda", "cuda"),       # between device pools
    ("cuda", "pinned", "pinned"),   # mapping itself in page-locked host memory
])
@pytest.mark.parametrize("dtype,shape,layers", [(torch.bfloat16, (16, 8, 128), 3),
                                                (torch.uint8, (32, 8, 128), 1),
                                                (torch.float32, (16, 2, 64), 2)])
def test_swap_bit_exact(src_where, dst_where, map_where, dtype, shape, layers):
    sk, sv = _pools(70, layers, shape, dtype, 11, src_where)
    dk, dv = _pools(50, layers, shape, dtype, 12, dst_where)
    m = _mapping(70, 50, 37, 13)
    ref_dk, ref_dv = [t.cpu().clone() for t in dk], [t.cpu().clone() for t in dv]
    orc.swap_blocks(ref_dk, ref_dv, [t.cpu() for t in sk], [t.cpu() for t in sv], m)
    mapping = m.cuda() if map_where == "cuda" else m.pin_memory()
    pkv.swap_blocks(dk, dv, sk, sv, mapping)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    for l in range(layers):
        assert torch.equal(dk[l].cpu().view(torch.uint8), ref_dk[l].view(torch.uint8))
        assert torch.equal(dv[l].cpu().view(torch.uint8), ref_dv[l].view(torch.uint8))


def test_swap_bad_ids_are_skipped_and_flagged():
    sk, sv = _pools(8, 1, (16, 2, 64), torch.float16, 21, "cuda")
    dk, dv = _pools(6, 1, (16, 2, 64), torch.float16, 22, "pinned")
    m = torch.tensor([[1, 2], [8, 0], [3, 6], [-1, 1], [4, 5]], dtype=torch.int64)
    before = [dk[0].clone(), dv[0].clone()]
    pkv.swap_blocks(dk, dv, sk, sv, m.cuda())
    torch.cuda.synchronize()
    assert pkv.get_device_error() == pkv.DEVERR_COPY_ID
    ref_k, ref_v = before
    orc.swap_blocks([ref_k], [ref_v], [sk[0].cpu()], [sv[0].cpu()], m[[0, 4]])
    assert torch.equal(dk[0].view(torch.int16), ref_k.view(torch.int16))
    assert torch.equal(dv[0].view(torch.int16), ref_v.view(torch.int16))


def test_swap_rejects_pageable_host_memory():
    sk, sv = _pools(4, 1, (16, 1, 64), torch.float16, 31, "cuda")
    pageable = torch.zeros(4, 16, 1, 64, dtype=torch.float16)
    m = torch.tensor([[0, 1]], dtype=torch.int64).cuda()
    arr = lambda t: (ctypes.c_void_p * 1)(t.data_ptr())
    rc = pkv.lib().pkv_swap_blocks(arr(pageable), arr(pageable), 4, arr(sk[0]), arr(sv[0]), 4, 1,
                                   m.data_ptr(), 1, 16 * 64 * 2, None)
    assert rc == pkv.PKV_EINVAL
    assert b"pageable" in pkv.lib().pkv_last_error_message()
    with pytest.raises(ValueError):
        pkv.swap_blocks([pageable], [pageable], sk, sv, m)


def test_preempt_swap_out_reuse_swap_in_decodes_identically():
    # decode a batch; preempt every other sequence (its blocks go to a pinned
    # host pool), let another tenant overwrite the freed device blocks, then
    # swap the sequences back into different free blocks and decode again
    gen = torch.Generator().manual_seed(41)
    lens = W.loguniform_lengths(24, 64, 4096, gen)
    wl = W.build_decode("preempt", lens, 32, 8, 128, 16, torch.bfloat16, torch.bfloat16, seed=42,
                        slack=1.0)
    g = gpu_inputs(wl)
    pkv.reshape_and_cache(g["nk"], g["nv"], g["kc"], g["vc"], g["slots"], g["ks"], g["vs"])
    out0 = torch.empty_like(g["q"])
    pkv.paged_attention_decode(out0, g["q"], g["kc"], g["vc"], g["tables"], g["lens"], wl.scale)
    tables = g["tables"].cpu()
    lens = g["lens"].cpu()
    bs = wl.block_size
    pre = list(range(0, tables.shape[0], 2))
    moved = []
    for s in pre:
        nb = (int(lens[s]) + bs - 1) // bs
        moved += tables[s, :nb].tolist()
    NB = g["kc"].shape[0]
    hk = torch.empty((len(moved),) + tuple(g["kc"].shape[1:]), dtype=g["kc"].dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_map = torch.tensor([[b, i] for i, b in enumerate(moved)], dtype=torch.int64)
    pkv.swap_blocks([hk], [hv], [g["kc"]], [g["vc"]], out_map.cuda())
    # another tenant writes over the freed blocks
    idx = torch.tensor(moved, device="cuda")
    g["kc"][idx] = torch.randn_like(g["kc"][idx].float()).to(g["kc"].dtype)
    g["vc"][idx] = torch.randn_like(g["vc"][idx].float()).to(g["vc"].dtype)
    # swap back into blocks that were never used (a shifted permutation of the pool)
    used = set(int(b) for b in tables.reshape(-1).tolist() if b >= 0)
    free = [b for b in range(NB) if b not in used]
    assert len(free) >= len(moved), "pool has no room for the swapped-in blocks"
    new_ids = free[:len(moved)]
    in_map = torch.tensor([[i, b] for i, b in enumerate(new_ids)], dtype=torch.int64)
    pkv.swap_blocks([g["kc"]], [g["vc"]], [hk], [hv], in_map.cuda())
    remap = dict(zip(moved, new_ids))
    t2 = tables.clone()
    for s in pre:
        nb = (int(lens[s]) + bs - 1) // bs
        t2[s, :nb] = torch.tensor([remap[int(b)] for b in tables[s, :nb]])
    out1 = torch.empty_like(g["q"])
    pkv.paged_attention_decode(out1, g["q"], g["kc"], g["vc"], t2.cuda(), g["lens"], wl.scale)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0
    assert torch.equal(out0.view(torch.int16), out1.view(torch.int16))
