"""GPU parity of the decode step (copy_blocks -> reshape_and_cache ->
paged_attention_decode) against the fp64 oracle, through the C ABI.

Tolerances (max-abs vs the oracle): 2e-3 for f32/f16/bf16 caches, 2e-2 for
FP8 caches (the oracle uses the same dequantised values), each plus half an
ulp of the output dtype for the final store."""
import math

import numpy as np
import pytest
import torch

import paged_kv_cache_373_b200 as pkv
from paged_kv_cache_373_b200 import workloads as W
from pkv_testutil import compare, gpu_inputs, gpu_step, oracle_step

pytestmark = pytest.mark.gpu

SMALL = {
    "cfg1": lambda: W.config1(),
    "f16_mha_d128": lambda: W.build_decode("f16_mha_d128", [1, 5, 16, 17, 33, 64, 100, 250, 513],
                                           8, 8, 128, 16, torch.float16, torch.float16, seed=31),
    "f16_gqa_d64_bs32": lambda: W.build_decode("f16_gqa_d64_bs32", [2, 31, 32, 33, 95, 300],
                                               8, 2, 64, 32, torch.float16, torch.float16, seed=32),
    "bf16_gqa4_d128": lambda: W.build_decode("bf16_gqa4_d128", [1, 15, 16, 47, 64, 200, 777],
                                             32, 8, 128, 16, torch.bfloat16, torch.bfloat16, seed=33),
    "bf16_g1_d64": lambda: W.build_decode("bf16_g1_d64", [3, 16, 18, 129], 4, 4, 64, 16,
                                          torch.bfloat16, torch.bfloat16, seed=34),
    "bf16_g3_ragged": lambda: W.build_decode("bf16_g3_ragged", [7, 40, 100], 6, 2, 128, 16,
                                             torch.bfloat16, torch.bfloat16, seed=35),
    "bf16_g16_two_chunks": lambda: W.build_decode("bf16_g16", [9, 80, 160], 32, 2, 128, 32,
                                                  torch.bfloat16, torch.bfloat16, seed=36),
    "f32_d128": lambda: W.build_decode("f32_d128", [1, 17, 64, 90], 4, 2, 128, 16, torch.float32,
                                       torch.float32, seed=37),
    "fp8_g8_bs32_qbf16": lambda: W.build_decode("fp8_g8", [1, 33, 64, 500, 1025], 64, 8, 128, 32,
                                                W.FP8, torch.bfloat16, seed=38),
    "fp8_g1_bs16_qf16": lambda: W.build_decode("fp8_g1", [2, 16, 17, 260], 4, 4, 128, 16, W.FP8,
                                               torch.float16, seed=39),
    "cfg5_mini": lambda: W.config5(num_prompts=2, samples=4, prefix=200, tail_lo=3, tail_hi=40),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_parity(name):
    wl = SMALL[name]()
    out, err, _ = gpu_step(wl)
    assert err == 0
    compare(out, oracle_step(wl), wl)


@pytest.mark.parametrize("num_ctas", [1, 3, 17, 148, 1000])
def test_split_count_changes_stay_within_tolerance(num_ctas):
    wl = SMALL["bf16_gqa4_d128"]()
    out, err, _ = gpu_step(wl, num_ctas=num_ctas)
    assert err == 0
    compare(out, oracle_step(wl), wl)


def test_physical_permutation_is_bit_identical():
    wl = SMALL["f16_mha_d128"]()
    out1, _, g = gpu_step(wl, num_ctas=40)
    # relabel every physical block b -> perm[b] and move its data accordingly
    perm = torch.randperm(wl.num_blocks, generator=torch.Generator().manual_seed(9))
    wl2 = W.build_decode("f16_mha_d128", [1, 5, 16, 17, 33, 64, 100, 250, 513], 8, 8, 128, 16,
                         torch.float16, torch.float16, seed=31)
    kc, vc = torch.empty_like(wl2.key_cache), torch.empty_like(wl2.value_cache)
    kc[perm], vc[perm] = wl2.key_cache, wl2.value_cache
    wl2.key_cache, wl2.value_cache = kc, vc
    t = wl2.block_tables.clone()
    m = t >= 0
    t[m] = perm[t[m].long()].to(torch.int32)
    wl2.block_tables = t
    s = wl2.slot_mapping.clone()
    s = perm[s // 16] * 16 + s % 16
    wl2.slot_mapping = s
    out2, err, _ = gpu_step(wl2, num_ctas=40)
    assert err == 0
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_shared_prefix_equals_private_copies_bit_identical():
    wl = W.config5(num_prompts=3, samples=8, prefix=3000, tail_lo=32, tail_hi=512)
    out1, err1, _ = gpu_step(wl, num_ctas=148)
    out2, err2, _ = gpu_step(W.with_all_copies(wl), num_ctas=148)
    assert err1 == 0 and err2 == 0
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_empty_and_single_token_sequences():
    wl = W.build_decode("edge", [0, 1, 0, 16, 1, 0], 4, 2, 128, 16, torch.bfloat16,
                        torch.bfloat16, seed=40)
    out, err, g = gpu_step(wl)
    assert err == 0
    ref = oracle_step(wl)
    compare(out, ref, wl)
    assert float(out[0].abs().max()) == 0.0 and float(out[2].abs().max()) == 0.0
    # seq_len 1: the output is the new token's value row (softmax of one score)
    v1 = wl.new_value[1].float()                 # [Hkv, D]
    for h in range(4):
        assert torch.equal(out[1, h].float().cpu(), v1[h // 2])


def test_all_sequences_empty():
    wl = W.build_decode("allempty", [0, 0, 0], 4, 4, 64, 16, torch.float16, torch.float16, seed=41)
    out, err, _ = gpu_step(wl)
    assert err == 0 and float(out.abs().max()) == 0.0


def test_indexing_probe_exact():
    """One dominant key per (sequence, head) picks out one logical token; the
    output must equal that token's value row exactly, which pins the
    logical -> physical translation (zwxr.cn 3.2) bit for bit."""
    S, H, D, bs = 6, 8, 128, 16
    lens = [5, 16, 17, 64, 130, 400]
    wl = W.build_decode("probe", lens, H, H, D, bs, torch.float16, torch.float16, seed=42)
    NB = wl.num_blocks
    # value rows encode (physical block, slot, head) as small exact integers
    b = torch.arange(NB).view(NB, 1, 1, 1)
    sl = torch.arange(bs).view(1, bs, 1, 1)
    hh = torch.arange(H).view(1, 1, H, 1)
    d = torch.arange(D).view(1, 1, 1, D)
    wl.value_cache = (((b * bs + sl) * 7 + hh * 3 + d) % 2000).to(torch.float16)
    wl.key_cache = torch.zeros((NB, bs, H, D), dtype=torch.float16)
    wl.new_key = torch.zeros_like(wl.new_key)
    wl.new_value = torch.full_like(wl.new_value, -1.0)
    q = torch.zeros((S, H, D), dtype=torch.float16)
    q[:, :, 0] = 1.0
    g = torch.Generator().manual_seed(3)
    target = {}
    for s in range(S):
        for h in range(H):
            t = int(torch.randint(0, lens[s] - 1, (1,), generator=g))   # an existing token
            phys = int(wl.block_tables[s, t // bs])
            wl.key_cache[phys, t % bs, h, 0] = 1000.0
            target[(s, h)] = (phys, t % bs)
    wl.query = q
    out, err, _ = gpu_step(wl)
    assert err == 0
    for (s, h), (phys, off) in target.items():
        assert torch.equal(out[s, h].cpu(), wl.value_cache[phys, off, h]), (s, h)


def test_bad_block_id_is_flagged_not_fatal():
    wl = W.build_decode("badid", [40, 20], 4, 4, 64, 16, torch.float16, torch.float16, seed=43)
    wl.block_tables[0, 1] = wl.num_blocks + 5
    out, err, _ = gpu_step(wl)
    assert err & pkv.DEVERR_BLOCK_ID
    torch.cuda.synchronize()                       # the context is still usable
    wl2 = SMALL["cfg1"]()
    out2, err2, _ = gpu_step(wl2)
    assert err2 == 0
    compare(out2, oracle_step(wl2), wl2)


def test_seq_len_beyond_table_is_flagged():
    wl = W.build_decode("badlen", [40], 4, 4, 64, 16, torch.float16, torch.float16, seed=44)
    g = gpu_inputs(wl)
    g["lens"][0] = 1000                              # table row holds 3 blocks
    out = torch.empty_like(g["q"])
    pkv.paged_attention_decode(out, g["q"], g["kc"], g["vc"], g["tables"], g["lens"], wl.scale)
    assert pkv.get_device_error() & pkv.DEVERR_SEQ_LEN


def test_host_validation_rejects_before_launch():
    wl = SMALL["cfg1"]()
    g = gpu_inputs(wl)
    out = torch.empty_like(g["q"])
    with pytest.raises(pkv.PkvError) as e:
        pkv.paged_attention_decode(out, g["q"], g["kc"], g["vc"], g["tables"], g["lens"], wl.scale,
                                   workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert e.value.status == pkv.PKV_EINVAL
    with pytest.raises(pkv.PkvError) as e:                       # q dtype != cache dtype
        pkv.paged_attention_decode(out.half(), g["q"].half(), g["kc"], g["vc"], g["tables"],
                                   g["lens"], wl.scale)
    assert e.value.status == pkv.PKV_EUNSUPPORTED


# ---- full-size configurations, sampled sequences ----------------------------
def _sample(wl, k, seed):
    g = torch.Generator().manual_seed(seed)
    idx = torch.randperm(wl.num_seqs, generator=g)[:k].tolist()
    # always include the longest and the shortest sequence
    idx += [int(wl.seq_lens.argmax()), int(wl.seq_lens.argmin())]
    return sorted(set(idx))


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_full_config_sampled_parity(cfg):
    wl = W.make_config(cfg)
    out, err, _ = gpu_step(wl)
    assert err == 0
    seqs = _sample(wl, 6, cfg)
    compare(out, oracle_step(wl, seqs=seqs), wl, seqs=seqs)
    assert torch.isfinite(out.float()).all()


def _step_args(wl, g, ws, num_ctas):
    a = pkv.DecodeStepArgs()
    a.num_seqs, a.num_heads, a.num_kv_heads = wl.num_seqs, wl.num_heads, wl.num_kv_heads
    a.head_dim, a.block_size, a.max_blocks_per_seq = wl.head_dim, wl.block_size, wl.max_blocks_per_seq
    a.num_blocks = wl.num_blocks
    a.q_dtype = pkv.dtype_code(wl.query)
    a.cache_dtype = pkv.PKV_FP8_E4M3 if wl.is_fp8 else a.q_dtype
    a.scale, a.num_ctas = wl.scale, num_ctas
    a.num_cow_pairs = int(wl.cow_pairs.shape[0])
    a.key_cache, a.value_cache = g["kc"].data_ptr(), g["vc"].data_ptr()
    a.k_scale = g["ks"].data_ptr() if g["ks"] is not None else None
    a.v_scale = g["vs"].data_ptr() if g["vs"] is not None else None
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    return a


STEP_CASES = {
    # larger steps: 70 sequences with copy-on-write pairs, 96 GQA sequences
    "prefix_cow_70": lambda: W.config5(num_prompts=10, samples=7, prefix=100, tail_lo=1, tail_hi=60),
    "bf16_gqa4_96": lambda: W.build_decode("bf16_gqa4_96", [(i * 37) % 301 for i in range(96)],
                                           32, 8, 128, 16, torch.bfloat16, torch.bfloat16, seed=36),
}


@pytest.mark.parametrize("name", ["cfg5_mini", "fp8_g8_bs32_qbf16", "bf16_gqa4_d128",
                                  "prefix_cow_70", "bf16_gqa4_96"])
def test_decode_step_host_packed_and_unpacked(name):
    """pkv_decode_step_host from host buffers, one copy per input and packed
    (one copy for all inputs), gives the device path's bits."""
    wl = STEP_CASES[name]() if name in STEP_CASES else SMALL[name]()
    ref, err, _ = gpu_step(wl, num_ctas=37)
    assert err == 0
    # each step starts from fresh caches: replaying a step's copy-on-write
    # copies on caches it already advanced would copy source blocks that now
    # hold other sequences' new tokens
    g = gpu_inputs(wl)
    ws = pkv.alloc_workspace(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim, 37)
    src = dict(q=wl.query, nk=wl.new_key.to(wl.q_dtype), nv=wl.new_value.to(wl.q_dtype),
               slots=wl.slot_mapping, tables=wl.block_tables, lens=wl.seq_lens, pairs=wl.cow_pairs)
    # one copy per input
    h = {k: v.contiguous().pin_memory() for k, v in src.items()}
    d = {k: torch.empty_like(v, device="cuda") for k, v in src.items()}
    h_out = torch.full_like(wl.query, float("nan")).pin_memory()
    d_out = torch.empty_like(ref)
    a = _step_args(wl, g, ws, 37)
    a.h_query, a.h_new_key, a.h_new_value = h["q"].data_ptr(), h["nk"].data_ptr(), h["nv"].data_ptr()
    a.h_slot_mapping, a.h_block_tables = h["slots"].data_ptr(), h["tables"].data_ptr()
    a.h_seq_lens, a.h_cow_pairs = h["lens"].data_ptr(), h["pairs"].data_ptr()
    a.d_query, a.d_new_key, a.d_new_value = d["q"].data_ptr(), d["nk"].data_ptr(), d["nv"].data_ptr()
    a.d_slot_mapping, a.d_block_tables = d["slots"].data_ptr(), d["tables"].data_ptr()
    a.d_seq_lens, a.d_cow_pairs = d["lens"].data_ptr(), d["pairs"].data_ptr()
    a.h_out, a.d_out = h_out.data_ptr(), d_out.data_ptr()
    pkv.decode_step_host(a)
    assert pkv.get_device_error() == 0
    assert torch.equal(h_out.view(-1).view(torch.uint8), ref.cpu().view(-1).view(torch.uint8))
    # packed: every input in one pinned buffer at the layout's offsets
    lay = pkv.decode_step_layout(wl.num_seqs, wl.num_heads, wl.num_kv_heads, wl.head_dim,
                                 a.q_dtype, wl.max_blocks_per_seq, a.num_cow_pairs)
    hb = torch.zeros(lay.total, dtype=torch.uint8).pin_memory()
    for key, off in (("q", lay.query), ("nk", lay.new_key), ("nv", lay.new_value),
                     ("slots", lay.slot_mapping), ("tables", lay.block_tables),
                     ("lens", lay.seq_lens), ("pairs", lay.cow_pairs)):
        b = src[key].contiguous().view(-1).view(torch.uint8)
        hb[off:off + b.numel()] = b
    db = torch.empty(lay.total, dtype=torch.uint8, device="cuda")
    h_out2 = torch.full_like(wl.query, float("nan")).pin_memory()
    g2 = gpu_inputs(wl)  # kept alive: the args hold raw pointers
    p = _step_args(wl, g2, ws, 37)
    p.h_packed, p.d_packed = hb.data_ptr(), db.data_ptr()
    d_out2 = torch.empty_like(ref)
    p.h_out, p.d_out = h_out2.data_ptr(), d_out2.data_ptr()
    pkv.decode_step_host(p)
    assert pkv.get_device_error() == 0
    assert torch.equal(h_out2.view(-1).view(torch.uint8), ref.cpu().view(-1).view(torch.uint8))
    compare(h_out2, oracle_step(wl), wl)


def test_many_short_sequences():
    """2048 sequences of 1..64 tokens (plus empty ones): every warp's length
    scans cover the whole batch and the merge grid sees many unit boundaries."""
    wl = W.short_batch()
    lens = wl.seq_lens.clone()
    out, err, _ = gpu_step(wl)
    assert err == 0
    compare(out, oracle_step(wl), wl)
    for num_ctas in (1, 7, 300):
        out2, err2, _ = gpu_step(wl, num_ctas=num_ctas)
        assert err2 == 0
        compare(out2, oracle_step(wl), wl)
    # a sprinkle of empty sequences in a large batch
    wl0 = W.build_decode("short_with_empty", [0 if i % 97 == 3 else int(L) for i, L in enumerate(lens)],
                         32, 8, 128, 16, torch.bfloat16, torch.bfloat16, seed=62)
    out3, err3, _ = gpu_step(wl0)
    assert err3 == 0
    compare(out3, oracle_step(wl0), wl0)
    assert float(out3[3].abs().max()) == 0.0


@pytest.mark.parametrize("heads,d,dtype,n", [((32, 32), 128, torch.float16, 700),
                                             ((64, 8), 64, torch.bfloat16, 1000),
                                             ((24, 2), 128, torch.bfloat16, 600)])
def test_large_batches_merge_eight_boundaries_per_cta(heads, d, dtype, n):
    """Batches above 512 sequences: the merge grid locates 8 worker boundaries
    per CTA with one CTA-wide length scan (MHA, g = 8 with D = 64, and g = 12,
    whose units are split into two head chunks), and the decode prologue scans
    the lengths once per CTA."""
    gen = torch.Generator().manual_seed(70 + n)
    lens = torch.randint(0, 120, (n,), generator=gen).tolist()
    wl = W.build_decode(f"large_batch_{n}", lens, heads[0], heads[1], d, 16, dtype, dtype, seed=71 + n)
    ref = oracle_step(wl)
    for num_ctas in (0, 5, 149):
        out, err, _ = gpu_step(wl, num_ctas=num_ctas)
        assert err == 0
        compare(out, ref, wl)


@pytest.mark.parametrize("name,num_ctas", [("bf16_gqa4_d128", 17), ("fp8_g8_bs32_qbf16", 3),
                                           ("f32_d128", 5), ("bf16_g16_two_chunks", 1000),
                                           ("f16_mha_d128", 1)])
def test_split_units_over_a_garbage_workspace_are_repeatable(name, num_ctas):
    """The workspace needs no initialisation: filled with 0xFF bytes before
    every call it changes nothing, and repeated calls give the same bits (the
    split units' partials are merged in worker order).  Grids of 1000 CTAs
    split most units many ways; one CTA splits the units its 8 warps share."""
    wl = SMALL[name]()
    _, err, g = gpu_step(wl)
    assert err == 0
    S, Hq, D = g["q"].shape
    ws = pkv.alloc_workspace(S, Hq, g["kc"].shape[2], D, num_ctas)
    outs = []
    for _ in range(3):
        ws.fill_(0xFF)
        out = torch.empty_like(g["q"])
        pkv.paged_attention_decode(out, g["q"], g["kc"], g["vc"], g["tables"], g["lens"], wl.scale,
                                   g["ks"], g["vs"], workspace=ws, num_ctas=num_ctas)
        outs.append(out)
    assert pkv.get_device_error() == 0
    compare(outs[0], oracle_step(wl), wl)
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


def _grow_keys(wl, rate):
    """Scale each sequence's key at position t by (1 + t * rate): the scores'
    running maximum keeps growing, past the 2^8 rescale threshold many times."""
    bs = wl.block_size
    for s in range(wl.num_seqs):
        for t in range(int(wl.seq_lens[s]) - 1):      # the cached tokens
            b = int(wl.block_tables[s, t // bs])
            wl.key_cache[b, t % bs] = (wl.key_cache[b, t % bs].float() * (1.0 + t * rate)).to(wl.key_cache.dtype)
    wl.query = (wl.query.float() * 3.0).to(wl.query.dtype)


@pytest.mark.parametrize("dtype,heads", [(torch.bfloat16, (32, 8)), (torch.float16, (8, 8))])
def test_growing_scores_exercise_the_lazy_rescale(dtype, heads):
    """Scores that grow along each sequence move every head's reference
    maximum on many tiles (a rescale whenever a tile's maximum passes it by
    2^8) and leave P just below 2^8 between them; split units merge partials
    taken against different references."""
    wl = W.build_decode("grow", [37, 300, 1000, 1500], heads[0], heads[1], 128, 16, dtype, dtype, seed=81)
    _grow_keys(wl, 1.0 / 64.0)
    ref = oracle_step(wl)
    for num_ctas in (0, 3):
        out, err, _ = gpu_step(wl, num_ctas=num_ctas)
        assert err == 0
        compare(out, ref, wl)
