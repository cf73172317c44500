"""Pins for the oracle's decode attention, indexing, reshape and copy (CPU only).

Checks are chosen so that a plausible slip in the oracle (a wrong GQA head
map, a transposed or off-by-one gather, a dropped scale, a missing mask of
the last block's unused slots, a wrong merge weight) fails at least one:
  * an independent library routine: torch float64 scaled_dot_product_attention
    on K/V gathered with plain tensor indexing (not the oracle's gather);
  * the worked block-table example of zwxr.cn section 3.2;
  * closed forms: seq_len 1 -> v_0, q = 0 -> mean(V), equal keys -> mean(V);
  * the block-wise softmax merge equals the global softmax (zwxr.cn 3.3);
  * invariance under any permutation of physical block ids (ttlab section 2);
  * shared (copy-on-write) reads equal private copies (zwxr.cn 3.4).
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from paged_kv_cache_373_b200 import workloads as W
from paged_kv_cache_373_b200.block_manager import BlockManager

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLD, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def _fp8_cache(wl, orc):
    """Quantise the FP8 pool sources with the oracle's reshape (all slots)."""
    NB, bs, Hkv, D = wl.key_src.shape
    kc = torch.zeros((NB, bs, Hkv, D), dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    slots = torch.arange(NB * bs, dtype=torch.int64)
    orc.reshape_and_cache(wl.key_src.reshape(NB * bs, Hkv, D), wl.value_src.reshape(NB * bs, Hkv, D),
                          kc, vc, slots, wl.k_scale, wl.v_scale)
    return kc, vc


def _caches_after_step(wl, orc):
    """Oracle decode step inputs: CoW copies, then the new tokens' writes."""
    if wl.is_fp8:
        kc, vc = _fp8_cache(wl, orc)
    else:
        kc, vc = wl.key_cache.clone(), wl.value_cache.clone()
    if wl.cow_pairs.numel():
        orc.copy_blocks([kc], [vc], wl.cow_pairs)
    orc.reshape_and_cache(wl.new_key, wl.new_value, kc, vc, wl.slot_mapping, wl.k_scale, wl.v_scale)
    return kc, vc


def _sdpa_reference(wl, kc, vc):
    """torch float64 SDPA over K/V gathered by plain tensor indexing."""
    S, Hq, D = wl.query.shape
    g = wl.num_heads // wl.num_kv_heads
    out = np.zeros((S, Hq, D))
    if wl.is_fp8:
        kf = kc.view(torch.float8_e4m3fn).to(torch.float64) * wl.k_scale
        vf = vc.view(torch.float8_e4m3fn).to(torch.float64) * wl.v_scale
    else:
        kf, vf = kc.to(torch.float64), vc.to(torch.float64)
    for s in range(S):
        L = int(wl.seq_lens[s])
        if L == 0:
            continue
        t = torch.arange(L)
        phys = wl.block_tables[s].to(torch.int64)[t // wl.block_size]
        K = kf[phys, t % wl.block_size]              # [L, Hkv, D]
        V = vf[phys, t % wl.block_size]
        K = K.permute(1, 0, 2).repeat_interleave(g, dim=0)   # [Hq, L, D]
        V = V.permute(1, 0, 2).repeat_interleave(g, dim=0)
        q = wl.query[s].to(torch.float64).unsqueeze(1)       # [Hq, 1, D]
        o = F.scaled_dot_product_attention(q, K, V, scale=wl.scale)
        out[s] = o.squeeze(1).numpy()
    return out


@pytest.mark.parametrize("make", [
    lambda: W.config1(),
    lambda: W.build_decode("mha_f16", [1, 5, 16, 17, 33, 64, 100], 4, 4, 128, 16,
                           torch.float16, torch.float16, seed=5),
    lambda: W.build_decode("gqa_bf16", [3, 31, 32, 47, 90], 8, 2, 64, 32,
                           torch.bfloat16, torch.bfloat16, seed=6),
    lambda: W.build_decode("gqa8_fp8", [2, 40, 77], 16, 2, 128, 32, W.FP8,
                           torch.bfloat16, seed=7),
    lambda: W.config5(num_prompts=2, samples=3, prefix=40, tail_lo=3, tail_hi=20),
])
def test_oracle_matches_torch_sdpa(orc, make):
    wl = make()
    kc, vc = _caches_after_step(wl, orc)
    got = orc.paged_attention_decode(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.scale,
                                     wl.k_scale, wl.v_scale)
    ref = _sdpa_reference(wl, kc, vc)
    assert np.abs(got - ref).max() < 1e-12


def test_worked_block_table_example(orc):
    # zwxr.cn section 3.2: logical 0 -> 3, 1 -> 11, 2 -> 7, 16-token blocks.
    rows = [tuple(int(x) for x in r) for r in _rows("block_table_example.txt")]
    NB, bs, Hkv, D = 16, 16, 2, 8
    # provenance cache: element value encodes (block, slot, head, dim) exactly
    idx = torch.arange(NB * bs * Hkv * D, dtype=torch.float64).reshape(NB, bs, Hkv, D)
    kc = idx.to(torch.float32)
    vc = (-idx).to(torch.float32)
    table = torch.tensor([3, 11, 7], dtype=torch.int32)
    for kvh in range(Hkv):
        K, V = orc.gather_kv(kc, vc, table, 48, kvh)
        for t, phys, off, slot in rows:
            assert slot == phys * bs + off
            want = ((phys * bs + off) * Hkv + kvh) * D + np.arange(D)
            assert np.array_equal(K[t], want) and np.array_equal(V[t], -want)
    # the host block manager reproduces the same table and slots
    order = [3, 11, 7] + [b for b in range(NB) if b not in (3, 11, 7)]
    bm = BlockManager(NB, bs, order)
    sid = bm.add_sequence(48)
    assert bm.block_table(sid) == [3, 11, 7]
    for t, phys, off, slot in rows:
        assert bm.slot_of(sid, t) == slot


def test_closed_forms(orc):
    rng = np.random.default_rng(1)
    D, L = 64, 37
    K = rng.normal(size=(L, D))
    V = rng.normal(size=(L, D))
    q = rng.normal(size=D)
    # seq_len 1: softmax of one score is 1 -> exactly v_0
    assert np.array_equal(orc.contiguous_attend(q, K[:1], V[:1], 0.125), V[0])
    # q = 0: uniform weights -> mean of V
    assert np.allclose(orc.contiguous_attend(np.zeros(D), K, V, 0.125), V.mean(0), rtol=0, atol=1e-13)
    # identical keys: uniform weights -> mean of V
    Ks = np.tile(K[:1], (L, 1))
    assert np.allclose(orc.contiguous_attend(q, Ks, V, 0.125), V.mean(0), rtol=0, atol=1e-13)
    # a key far above the rest takes all the weight
    Kd = K.copy()
    Kd[5] = q * 50.0
    assert np.allclose(orc.contiguous_attend(q, Kd, V, 1.0), V[5], atol=1e-12)
    # scale enters as exp(scale * q.k): doubling q equals doubling the scale
    assert np.allclose(orc.contiguous_attend(2 * q, K, V, 0.1), orc.contiguous_attend(q, K, V, 0.2),
                       atol=1e-14)


@pytest.mark.parametrize("part", [1, 3, 16, 64, 500, 10000])
def test_blockwise_merge_equals_global(orc, part):
    # zwxr.cn 3.3: per-block (m, l) plus the rescale merge is exactly the global softmax
    rng = np.random.default_rng(part)
    D, L = 128, 1000
    K = rng.normal(size=(L, D)) * 2
    V = rng.normal(size=(L, D))
    q = rng.normal(size=D)
    a = orc.blockwise_attend(q, K, V, 1 / math.sqrt(D), part)
    b = orc.contiguous_attend(q, K, V, 1 / math.sqrt(D))
    assert np.abs(a - b).max() <= 1e-12 * max(1.0, np.abs(b).max())


def test_empty_sequence_gives_zero(orc):
    wl = W.build_decode("empty", [0, 5], 2, 2, 64, 16, torch.float32, torch.float32, seed=3)
    kc, vc = _caches_after_step(wl, orc)
    out = orc.paged_attention_decode(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.scale)
    assert np.all(out[0] == 0.0)
    assert np.abs(out[1] - _sdpa_reference(wl, kc, vc)[1]).max() < 1e-12


def test_permutation_of_physical_blocks_is_invisible(orc):
    wl = W.build_decode("perm", [7, 16, 33, 64, 129], 8, 2, 64, 16, torch.bfloat16,
                        torch.bfloat16, seed=9)
    kc, vc = _caches_after_step(wl, orc)
    base = orc.paged_attention_decode(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.scale)
    perm = torch.randperm(wl.num_blocks, generator=torch.Generator().manual_seed(4))
    kp, vp = torch.empty_like(kc), torch.empty_like(vc)
    kp[perm] = kc                                      # block b moves to perm[b]
    vp[perm] = vc
    tables = wl.block_tables.clone()
    m = tables >= 0
    tables[m] = perm[tables[m].long()].to(torch.int32)
    moved = orc.paged_attention_decode(wl.query, kp, vp, tables, wl.seq_lens, wl.scale)
    assert np.array_equal(base, moved)


def test_new_token_is_attended_at_its_slot(orc):
    # a token takes its slot when produced (zwxr.cn 3.1): after the write, the
    # paged result equals contiguous attention over the old rows plus the new one
    wl = W.build_decode("append", [9, 16, 17, 40], 4, 2, 64, 16, torch.float32, torch.float32,
                        seed=12)
    kc, vc = wl.key_cache.clone(), wl.value_cache.clone()
    orc.reshape_and_cache(wl.new_key, wl.new_value, kc, vc, wl.slot_mapping)
    out = orc.paged_attention_decode(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.scale)
    g = wl.num_heads // wl.num_kv_heads
    for s in range(wl.num_seqs):
        L = int(wl.seq_lens[s])
        t = torch.arange(L - 1)
        phys = wl.block_tables[s].long()[t // 16]
        for h in range(wl.num_heads):
            kvh = h // g
            K = torch.cat([wl.key_cache[phys, t % 16, kvh], wl.new_key[s, kvh][None]]).double()
            V = torch.cat([wl.value_cache[phys, t % 16, kvh], wl.new_value[s, kvh][None]]).double()
            ref = orc.contiguous_attend(wl.query[s, h].double().numpy(), K.numpy(), V.numpy(),
                                        wl.scale)
            assert np.abs(out[s, h] - ref).max() < 1e-13


def test_reshape_skips_padding_and_encodes_fp8(orc):
    NB, bs, Hkv, D = 4, 16, 2, 128
    kc = torch.zeros((NB, bs, Hkv, D), dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    g = torch.Generator().manual_seed(2)
    k = torch.randn((3, Hkv, D), generator=g).to(torch.bfloat16)
    v = torch.randn((3, Hkv, D), generator=g).to(torch.bfloat16)
    slots = torch.tensor([5, -1, 63], dtype=torch.int64)
    ks, vs = 0.01, 0.02
    orc.reshape_and_cache(k, v, kc, vc, slots, ks, vs)
    assert int(kc.sum()) > 0
    ref_k = (k.float() / torch.tensor(ks, dtype=torch.float32)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    ref_v = (v.float() / torch.tensor(vs, dtype=torch.float32)).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(kc[0, 5], ref_k[0]) and torch.equal(vc[0, 5], ref_v[0])
    assert torch.equal(kc[3, 15], ref_k[2]) and torch.equal(vc[3, 15], ref_v[2])
    written = torch.zeros(NB * bs, dtype=torch.bool)
    written[[5, 63]] = True
    assert int(kc.reshape(NB * bs, -1)[~written].sum()) == 0   # slot -1 skipped, rest untouched


def test_copy_blocks_and_cow_invariance(orc):
    wl = W.config5(num_prompts=3, samples=4, prefix=40, tail_lo=3, tail_hi=30)
    assert wl.cow_pairs.shape[0] == 3 * 3          # samples-1 copies per prompt
    kc, vc = wl.key_cache.clone(), wl.value_cache.clone()
    k0 = kc.clone()
    orc.copy_blocks([kc], [vc], wl.cow_pairs)
    for src, dst in wl.cow_pairs.tolist():
        assert torch.equal(kc[dst], k0[src]) and torch.equal(kc[src], k0[src])
    touched = set(wl.cow_pairs[:, 1].tolist())
    others = [b for b in range(wl.num_blocks) if b not in touched]
    assert torch.equal(kc[others], k0[others])
    # shared reads equal private copies (zwxr.cn 3.4): every sample copies instead
    a = orc.paged_attention_decode(wl.query, *_caches_after_step(wl, orc), wl.block_tables,
                                   wl.seq_lens, wl.scale)
    wl2 = W.with_all_copies(wl)
    b = orc.paged_attention_decode(wl2.query, *_caches_after_step(wl2, orc), wl2.block_tables,
                                   wl2.seq_lens, wl2.scale)
    assert np.array_equal(a, b)
    # and equal a layout with no sharing at all: every sequence on private blocks
    kc1, vc1 = _caches_after_step(wl, orc)
    total = sum((int(L) + 15) // 16 for L in wl.seq_lens)
    kp = torch.empty((total,) + kc1.shape[1:], dtype=kc1.dtype)
    vp = torch.empty_like(kp)
    tables = torch.full_like(wl.block_tables, -1)
    nxt = 0
    for s in range(wl.num_seqs):
        for i in range((int(wl.seq_lens[s]) + 15) // 16):
            b = int(wl.block_tables[s, i])
            kp[nxt], vp[nxt] = kc1[b], vc1[b]
            tables[s, i] = nxt
            nxt += 1
    c = orc.paged_attention_decode(wl.query, kp, vp, tables, wl.seq_lens, wl.scale)
    assert np.array_equal(a, c)


def test_oracle_rejects_bad_block_ids(orc):
    wl = W.build_decode("bad", [20], 2, 2, 64, 16, torch.float32, torch.float32, seed=1)
    t = wl.block_tables.clone()
    t[0, 1] = wl.num_blocks          # out of range
    with pytest.raises(ValueError):
        orc.paged_attention_decode(wl.query, wl.key_cache, wl.value_cache, t, wl.seq_lens, wl.scale)
