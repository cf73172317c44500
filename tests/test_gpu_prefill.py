"""Chunked-prefill attention on the GPU (ttlab.hopto.org "LLM KV cache 02",
section 3) against the fp64 oracle: the chunk's K/V go to the cache with
reshape_and_cache, then every chunk row attends causally through the block
table.  Tolerance as for decode: 2e-3 max-abs plus half an ulp of the output
dtype."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_373_b200 as pkv
from paged_kv_cache_373_b200 import workloads as W
from pkv_testutil import TOL_16, half_ulp

pytestmark = pytest.mark.gpu


def gpu_prefill(wl, kc=None, vc=None):
    kc = wl.key_cache.cuda() if kc is None else kc
    vc = wl.value_cache.cuda() if vc is None else vc
    pkv.reshape_and_cache(wl.new_key.cuda(), wl.new_value.cuda(), kc, vc, wl.slot_mapping.cuda())
    out = torch.full_like(wl.query, float("nan")).cuda()
    pkv.paged_prefill(out, wl.query.cuda(), kc, vc, wl.block_tables.cuda(), wl.seq_lens.cuda(),
                      wl.query_start.cuda(), wl.scale)
    err = pkv.get_device_error()
    return out, err, kc, vc


def oracle_caches(wl):
    kc, vc = wl.key_cache.clone(), wl.value_cache.clone()
    oracle.reshape_and_cache(wl.new_key, wl.new_value, kc, vc, wl.slot_mapping)
    return kc, vc


def check(out, ref, dtype, rows=None):
    g = out.float().cpu().double().numpy()
    if rows is not None:
        g = g[rows]
    assert np.isfinite(g).all(), "non-finite output"
    err = np.abs(g - ref)
    worst = float((err - (TOL_16 + half_ulp(ref, dtype))).max())
    assert worst <= 0.0, f"max|err| {err.max():.3e} exceeds the bound by {worst:.3e}"
    return float(err.max())


CASES = [
    # name, ctx, chunks, Hq, Hkv, D, bs, dtype
    ("g2_bf16_d128", [0, 37, 5, 0], [100, 21, 1, 64], 16, 8, 128, 16, torch.bfloat16),
    ("g1_f16_d128_bs32", [3, 100, 0], [29, 64, 130], 4, 4, 128, 32, torch.float16),
    ("g4_bf16_d64", [17, 0, 250], [1, 33, 70], 8, 2, 64, 16, torch.bfloat16),
    ("g8_f16_d64", [0, 64, 1], [65, 63, 16], 16, 2, 64, 16, torch.float16),
    ("g16_bf16_d128", [5, 0], [9, 40], 16, 1, 128, 32, torch.bfloat16),
    ("empty_chunks", [10, 20, 0, 30], [0, 5, 0, 1], 8, 4, 128, 16, torch.bfloat16),
    # units without a partner split their tiles over both groups (odd and even tile counts)
    ("lone_long", [3000, 2047, 0], [1, 1, 70], 16, 8, 128, 16, torch.bfloat16),
    ("lone_f16_d64", [1000, 63, 64], [2, 3, 40], 8, 8, 64, 32, torch.float16),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_prefill_matches_oracle(case):
    name, ctx, ch, hq, hkv, d, bs, dt = case
    wl = W.build_prefill(name, ctx, ch, hq, hkv, d, bs, dt, seed=21)
    out, err, _, _ = gpu_prefill(wl)
    assert err == 0
    kc, vc = oracle_caches(wl)
    ref = oracle.paged_prefill(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.query_start, wl.scale)
    check(out, ref, dt)


def oracle_rows(wl, kc, vc, rows):
    """The oracle one row at a time: row r of sequence s is a one-token chunk at its position."""
    qs = wl.query_start.tolist()
    res = []
    for r in rows:
        s = max(i for i in range(wl.num_seqs) if qs[i] <= r)
        pos = int(wl.seq_lens[s]) - (qs[s + 1] - qs[s]) + (r - qs[s])
        res.append(oracle.paged_prefill(wl.query[r:r + 1], kc, vc, wl.block_tables[s:s + 1],
                                        torch.tensor([pos + 1], dtype=torch.int32),
                                        torch.tensor([0, 1], dtype=torch.int32), wl.scale)[0])
    return np.stack(res)


@pytest.mark.parametrize("budget", [2048, 8192])
def test_prefill_full_step_sampled(budget):
    wl = W.prefill_config(budget)
    out, err, _, _ = gpu_prefill(wl)
    assert err == 0
    assert torch.isfinite(out.float()).all()
    kc, vc = oracle_caches(wl)
    qs = wl.query_start.tolist()
    rows = sorted({0, 1, 2, 63, 64, 65, qs[-2], qs[-1] - 1, qs[-2] + 200, qs[1] + 3499 if budget == 8192 else 5,
                   qs[2] + 1000, qs[-1] // 2})
    rows = [r for r in rows if 0 <= r < wl.num_tokens]
    check(out, oracle_rows(wl, kc, vc, rows), wl.kv_dtype, rows)


def test_growing_scores_exercise_the_rescale():
    # keys of later positions scaled up so each 64-token tile's maximum score
    # exceeds the running reference by far more than 2^8: the accumulator
    # rescale path runs on every tile
    wl = W.build_prefill("rescale", [0, 70], [200, 90], 8, 2, 128, 16, torch.bfloat16, seed=25)
    bs = wl.block_size
    for s_ in range(wl.num_seqs):
        L = int(wl.seq_lens[s_])
        C = int(wl.query_start[s_ + 1] - wl.query_start[s_])
        for t in range(L - C):                      # cached context tokens
            b = int(wl.block_tables[s_, t // bs])
            wl.key_cache[b, t % bs] = (wl.key_cache[b, t % bs].float() * (1.0 + t / 8.0)).to(torch.bfloat16)
    wl.new_key = (wl.new_key.float() * torch.linspace(1.0, 30.0, wl.num_tokens)[:, None, None]).to(torch.bfloat16)
    wl.query = (wl.query.float() * 3.0).to(torch.bfloat16)
    out, err, _, _ = gpu_prefill(wl)
    assert err == 0
    kc, vc = oracle_caches(wl)
    ref = oracle.paged_prefill(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.query_start, wl.scale)
    check(out, ref, torch.bfloat16)


def test_splitting_a_chunk_matches_and_calls_are_deterministic():
    # the same 150 tokens as one chunk, or as chunks of 70 and 80 in two calls:
    # both within the oracle bound.  The rows may be summed in another order
    # (a unit without a partner splits its tiles over two groups), so the two
    # need not be bit-identical; repeating a call is.
    wl = W.build_prefill("whole", [40], [150], 8, 4, 128, 16, torch.bfloat16, seed=22)
    whole, err, kc, vc = gpu_prefill(wl)
    assert err == 0
    q = wl.query.cuda()
    t = wl.block_tables.cuda()
    again = torch.empty_like(q)
    pkv.paged_prefill(again, q, kc, vc, t, wl.seq_lens.cuda(), wl.query_start.cuda(), wl.scale)
    assert torch.equal(whole.view(torch.int16), again.view(torch.int16))
    part = torch.empty_like(q)
    for lo, hi in ((0, 70), (70, 150)):
        pkv.paged_prefill(part[lo:hi], q[lo:hi].contiguous(), kc, vc, t,
                          torch.tensor([40 + hi], dtype=torch.int32, device="cuda"),
                          torch.tensor([0, hi - lo], dtype=torch.int32, device="cuda"), wl.scale)
    assert pkv.get_device_error() == 0
    okc, ovc = oracle_caches(wl)
    ref = oracle.paged_prefill(wl.query, okc, ovc, wl.block_tables, wl.seq_lens, wl.query_start, wl.scale)
    check(whole, ref, torch.bfloat16)
    check(part, ref, torch.bfloat16)


def test_one_token_chunks_match_decode():
    lens = [1, 17, 300, 2049]
    wl = W.build_prefill("decode_rows", [L - 1 for L in lens], [1] * 4, 32, 8, 128, 16, torch.bfloat16, seed=23)
    out, err, kc, vc = gpu_prefill(wl)
    assert err == 0
    dec = torch.empty_like(out)
    pkv.paged_attention_decode(dec, wl.query.cuda(), kc, vc, wl.block_tables.cuda(), wl.seq_lens.cuda(),
                               wl.scale)
    assert (out.float() - dec.float()).abs().max().item() < 4e-3


def test_bad_lengths_and_block_ids_are_flagged():
    wl = W.build_prefill("bad", [10, 20], [5, 5], 8, 4, 64, 16, torch.float16, seed=24)
    kc, vc = wl.key_cache.cuda(), wl.value_cache.cuda()
    q = wl.query.cuda()
    out = torch.zeros_like(q)
    short = torch.tensor([3, 25], dtype=torch.int32, device="cuda")          # 3 < chunk of 5
    pkv.paged_prefill(out, q, kc, vc, wl.block_tables.cuda(), short, wl.query_start.cuda(), wl.scale)
    assert pkv.get_device_error() == pkv.DEVERR_SEQ_LEN
    tables = wl.block_tables.clone()
    tables[1, 0] = wl.num_blocks + 7
    pkv.paged_prefill(out, q, kc, vc, tables.cuda(), wl.seq_lens.cuda(), wl.query_start.cuda(), wl.scale)
    assert pkv.get_device_error() == pkv.DEVERR_BLOCK_ID
    with pytest.raises(pkv.PkvError):   # g = 3 is not supported
        pkv.paged_prefill(torch.zeros(10, 6, 64, dtype=torch.float16, device="cuda"),
                          torch.zeros(10, 6, 64, dtype=torch.float16, device="cuda"),
                          torch.zeros(4, 16, 2, 64, dtype=torch.float16, device="cuda"),
                          torch.zeros(4, 16, 2, 64, dtype=torch.float16, device="cuda"),
                          wl.block_tables.cuda(), wl.seq_lens.cuda(), wl.query_start.cuda(), 0.125)


@pytest.mark.parametrize("stop_tile", [0, 2])
def test_bounded_waits_run_out_then_the_context_recovers(stop_tile):
    """A test hook makes every CTA's copy lane stop before K/V tile `stop_tile`
    (after the q rows), so the other roles' bounded waits (1 ms here) run out:
    the call sets PKV_DEVERR_TIMEOUT and each CTA drains what it issued and
    frees its tensor memory.  The next, normal call on the same context -- its
    CTAs allocate the same tensor-memory columns on the same SMs -- completes
    and matches the oracle."""
    wl = W.build_prefill("timeout", [0, 300, 1000], [200, 64, 1], 16, 8, 128, 16, torch.bfloat16, seed=23)
    L = pkv.lib()
    assert L.pkv_testing_prefill_timeout(stop_tile, 1_000_000) == pkv.PKV_OK
    out, err, kc, vc = gpu_prefill(wl)
    assert err & pkv.DEVERR_TIMEOUT, f"device error word {err:#x}"
    assert err & ~pkv.DEVERR_TIMEOUT == 0
    out2, err2, _, _ = gpu_prefill(wl, kc, vc)       # disarmed after one call
    assert err2 == 0
    kh, vh = oracle_caches(wl)
    ref = oracle.paged_prefill(wl.query, kh, vh, wl.block_tables, wl.seq_lens, wl.query_start, wl.scale)
    check(out2, ref, torch.bfloat16)
