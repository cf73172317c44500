"""Cascade (shared-prefix) decode: the shared prefix blocks of a group are read
once for all members (zwxr.cn 3.4 sharing turned into bandwidth); the result
must equal ordinary decode attention, so it is checked against the fp64
oracle with the same tolerances, and against the plain decode path."""
import pytest
import torch

import paged_kv_cache_373_b200 as pkv
from paged_kv_cache_373_b200 import workloads as W
from pkv_testutil import compare, gpu_inputs, oracle_step

pytestmark = pytest.mark.gpu


def _cascade_step(wl, groups=None, num_ctas=0):
    g = gpu_inputs(wl)
    if g["pairs"].numel():
        pkv.copy_blocks([g["kc"]], [g["vc"]], g["pairs"])
    pkv.reshape_and_cache(g["nk"], g["nv"], g["kc"], g["vc"], g["slots"], g["ks"], g["vs"])
    off, mem, pre, mgs = groups or W.cascade_groups(wl)
    out = torch.empty_like(g["q"])
    pkv.paged_attention_decode_cascade(out, g["q"], g["kc"], g["vc"], g["tables"], g["lens"],
                                       off.cuda(), mem.cuda(), pre.cuda(), mgs, wl.scale,
                                       g["ks"], g["vs"], num_ctas=num_ctas)
    plain = torch.empty_like(g["q"])
    pkv.paged_attention_decode(plain, g["q"], g["kc"], g["vc"], g["tables"], g["lens"], wl.scale,
                               g["ks"], g["vs"], num_ctas=num_ctas)
    return out, plain, pkv.get_device_error()


@pytest.mark.parametrize("shape", [(2, 4, 200, 3, 40), (3, 8, 3000, 32, 512), (1, 3, 40, 1, 20)])
def test_cascade_matches_oracle(shape):
    prompts, samples, prefix, lo, hi = shape
    wl = W.config5(num_prompts=prompts, samples=samples, prefix=prefix, tail_lo=lo, tail_hi=hi)
    out, plain, err = _cascade_step(wl)
    assert err == 0
    ref = oracle_step(wl)
    compare(out, ref, wl)
    compare(plain, ref, wl)


@pytest.mark.parametrize("dtype,heads,d", [(torch.float16, (16, 4), 64), (torch.bfloat16, (24, 2), 128),
                                           (torch.float16, (8, 8), 128), (torch.float32, (8, 2), 64),
                                           (torch.float16, (32, 8), 128)])
def test_cascade_dtypes_and_head_groupings(dtype, heads, d):
    # f16 / bf16 with g = 4, 12 (two head chunks) and 1; fp32 takes the plain
    # path; f16 with head_dim 128 and 20 rows per kv head takes the
    # tensor-core prefix pass (f16 operands)
    wl = W.config5(num_prompts=3, samples=5, prefix=333, tail_lo=1, tail_hi=70, dtype=dtype,
                   num_heads=heads[0], num_kv_heads=heads[1], head_dim=d)
    out, _, err = _cascade_step(wl)
    assert err == 0
    compare(out, oracle_step(wl), wl)


def test_cascade_with_many_groups():
    # 640 sequences: the suffix pass's merge takes its 8-boundaries-per-CTA form
    wl = W.config5(num_prompts=80, samples=8, prefix=40, tail_lo=1, tail_hi=30)
    for num_ctas in (0, 9):
        out, plain, err = _cascade_step(wl, num_ctas=num_ctas)
        assert err == 0
        ref = oracle_step(wl)
        compare(out, ref, wl)
        compare(plain, ref, wl)


@pytest.mark.parametrize("prefix", [700, 1000])
def test_cascade_block_sizes(prefix):
    # 32-token blocks: a 128-token K/V tile of the prefix pass spans 4 blocks
    # (2 per copy warp); the shared run (672 or 992 tokens) ends 32 or 96
    # tokens into its last tile
    wl = W.config5(num_prompts=3, samples=4, prefix=prefix, tail_lo=5, tail_hi=200, block_size=32)
    for num_ctas in (0, 4):
        out, plain, err = _cascade_step(wl, num_ctas=num_ctas)
        assert err == 0
        ref = oracle_step(wl)
        compare(out, ref, wl)
        compare(plain, ref, wl)


def test_cascade_full_config5_sampled():
    wl = W.config5()
    out, plain, err = _cascade_step(wl)
    assert err == 0
    seqs = [0, 7, 8, 63, 64, 100, 127]
    compare(out, oracle_step(wl, seqs=seqs), wl, seqs=seqs)
    d = (out.float() - plain.float()).abs().max().item()
    assert d < 4e-3, d


@pytest.mark.parametrize("num_ctas", [1, 7, 148])
def test_cascade_split_counts(num_ctas):
    wl = W.config5(num_prompts=2, samples=5, prefix=700, tail_lo=1, tail_hi=90)
    out, _, err = _cascade_step(wl, num_ctas=num_ctas)
    assert err == 0
    compare(out, oracle_step(wl), wl)


def test_cascade_groups_that_share_less_than_declared():
    # requested prefix longer than what the tables share, a member shorter than
    # the request, a single-member group and an empty group: still exact
    wl = W.config5(num_prompts=3, samples=4, prefix=100, tail_lo=1, tail_hi=60)
    off = torch.tensor([0, 4, 5, 5, 12], dtype=torch.int32)     # groups: 4, 1, 0, 7 members
    mem = torch.tensor([0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11], dtype=torch.int32)
    pre = torch.tensor([4096, 96, 0, 64], dtype=torch.int32)
    out, _, err = _cascade_step(wl, groups=(off, mem, pre, 7))
    assert err == pkv.DEVERR_SEQ_LEN        # 4096 exceeds the members' lengths: flagged, clamped
    compare(out, oracle_step(wl), wl)


def test_cascade_invalid_member_and_oversize_group_are_flagged_and_unshared():
    # a member id outside [0, num_seqs) and a group larger than max_group_size:
    # both flagged, neither group shared, every output still exact
    wl = W.config5(num_prompts=2, samples=4, prefix=160, tail_lo=1, tail_hi=40)
    off = torch.tensor([0, 4, 8], dtype=torch.int32)
    mem = torch.tensor([0, 1, 2, 999, 4, 5, 6, 7], dtype=torch.int32)
    pre = torch.tensor([160, 160], dtype=torch.int32)
    out, plain, err = _cascade_step(wl, groups=(off, mem, pre, 3))
    assert err == pkv.DEVERR_SEQ_LEN
    compare(out, oracle_step(wl), wl)
    assert (out.float() - plain.float()).abs().max().item() < 4e-3


def test_cascade_without_groups_is_plain_decode():
    wl = W.build_decode("nogroups", [5, 40, 300], 8, 2, 128, 16, torch.bfloat16, torch.bfloat16, seed=61)
    wl.meta.update(prompts=0, samples=1, prefix=0)
    groups = (torch.zeros(1, dtype=torch.int32), torch.zeros(0, dtype=torch.int32),
              torch.zeros(0, dtype=torch.int32), 1)
    out, plain, err = _cascade_step(wl, groups=groups)
    assert err == 0
    assert torch.equal(out.view(torch.int16), plain.view(torch.int16))


@pytest.mark.parametrize("num_ctas", [0, 3, 11])
def test_cascade_finish_pass_merges_unshared_and_zeroes_empty_sequences(num_ctas):
    # groups whose members share no blocks (and request no prefix): every
    # sequence takes the suffix pass from token 0, and the finish pass must
    # merge its split units and zero the empty ones -- the same partials, in
    # the same order, as plain decode's merge, so the bits match it
    wl = W.build_decode("unshared", [0, 300, 17, 0, 900, 64, 5, 1200], 32, 8, 128, 16, torch.bfloat16,
                        torch.bfloat16, seed=92)
    wl.meta.update(prompts=0, samples=1, prefix=0)
    groups = (torch.tensor([0, 3, 8], dtype=torch.int32), torch.arange(8, dtype=torch.int32),
              torch.zeros(2, dtype=torch.int32), 5)
    out, plain, err = _cascade_step(wl, groups=groups, num_ctas=num_ctas)
    assert err == 0
    compare(out, oracle_step(wl), wl)
    assert torch.equal(out, plain)
    assert float(out[0].abs().max()) == 0.0 and float(out[3].abs().max()) == 0.0


@pytest.mark.parametrize("num_ctas", [8, 20, 300])
def test_cascade_side_by_side_split_edges(num_ctas):
    # the prefix and suffix passes split the grid between them (8 CTAs: the
    # smallest grid that splits; 300: more CTAs than SMs, so the suffix
    # pass's arrival tickets outnumber the free SMs); two groups share a
    # prefix, a third shares nothing
    wl = W.config5(num_prompts=3, samples=6, prefix=900, tail_lo=10, tail_hi=260)
    off, mem, pre, mgs = W.cascade_groups(wl)
    pre = pre.clone()
    pre[1] = 0  # the second prompt's members: unshared
    out, plain, err = _cascade_step(wl, groups=(off, mem, pre, mgs), num_ctas=num_ctas)
    assert err == 0
    ref = oracle_step(wl)
    compare(out, ref, wl)
    compare(plain, ref, wl)


def test_cascade_replays_in_a_cuda_graph():
    # the whole call (zeroing, setup, the side-by-side prefix and suffix
    # passes with their arrival tickets, finish) captured once and replayed:
    # every replay gives the eager call's bits
    wl = W.config5(num_prompts=4, samples=8, prefix=1200, tail_lo=10, tail_hi=300)
    g = gpu_inputs(wl)
    if g["pairs"].numel():
        pkv.copy_blocks([g["kc"]], [g["vc"]], g["pairs"])
    pkv.reshape_and_cache(g["nk"], g["nv"], g["kc"], g["vc"], g["slots"], g["ks"], g["vs"])
    off, mem, pre, mgs = W.cascade_groups(wl)
    off, mem, pre = off.cuda(), mem.cuda(), pre.cuda()
    n = pkv.paged_attention_cascade_workspace_bytes(wl.num_seqs, wl.num_heads, wl.num_kv_heads,
                                                    wl.head_dim, pre.shape[0], mgs, 0)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    eager = torch.empty_like(g["q"])
    pkv.paged_attention_decode_cascade(eager, g["q"], g["kc"], g["vc"], g["tables"], g["lens"], off, mem, pre,
                                       mgs, wl.scale, workspace=ws)
    torch.cuda.synchronize()
    out = torch.zeros_like(g["q"])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        pkv.paged_attention_decode_cascade(out, g["q"], g["kc"], g["vc"], g["tables"], g["lens"], off, mem, pre,
                                           mgs, wl.scale, workspace=ws)
    for _ in range(2):
        out.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    assert pkv.get_device_error() == 0
    compare(eager, oracle_step(wl), wl)


def test_cascade_growing_scores_exercise_the_lazy_rescale():
    # keys grow along the shared prefix and the tails: the prefix pass's rows
    # and the suffix pass rescale on many tiles
    wl = W.config5(num_prompts=2, samples=4, prefix=700, tail_lo=20, tail_hi=300)
    bs = wl.block_size
    for s in range(wl.num_seqs):
        for t in range(int(wl.seq_lens[s]) - 1):
            b = int(wl.block_tables[s, t // bs])
            if t < 700 and s % 4 != 0:
                continue  # shared prefix blocks: scaled once, through the group's first member
            wl.key_cache[b, t % bs] = (wl.key_cache[b, t % bs].float() * (1.0 + t / 64.0)).to(torch.bfloat16)
    wl.query = (wl.query.float() * 3.0).to(torch.bfloat16)
    for num_ctas in (0, 5):
        out, plain, err = _cascade_step(wl, num_ctas=num_ctas)
        assert err == 0
        ref = oracle_step(wl)
        compare(out, ref, wl)
        compare(plain, ref, wl)
