"""Pins of the chunked-prefill oracle (ttlab.hopto.org "LLM KV cache 02",
section 3): against torch float64 scaled_dot_product_attention with an
explicit causal mask on K/V gathered by plain indexing (an independent
library routine), the decode oracle for one-token chunks, splitting a chunk
in two (chunked prefill must not change any row), and causality (tokens after
a row's position do not affect it)."""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_373_b200 import workloads as W


def caches_after_chunk(wl):
    kc, vc = wl.key_cache.clone(), wl.value_cache.clone()
    oracle.reshape_and_cache(wl.new_key, wl.new_value, kc, vc, wl.slot_mapping)
    return kc, vc


def sdpa_reference(wl, kc, vc):
    out = np.zeros(tuple(wl.query.shape), dtype=np.float64)
    g = wl.num_heads // wl.num_kv_heads
    bs = wl.block_size
    for s in range(wl.num_seqs):
        L = int(wl.seq_lens[s])
        q0, q1 = int(wl.query_start[s]), int(wl.query_start[s + 1])
        C = q1 - q0
        t = torch.arange(L)
        phys = wl.block_tables[s, t // bs].long()
        K = kc[phys, t % bs].double()                     # [L, Hkv, D]
        V = vc[phys, t % bs].double()
        K = K.repeat_interleave(g, dim=1).transpose(0, 1)  # [Hq, L, D]
        V = V.repeat_interleave(g, dim=1).transpose(0, 1)
        q = wl.query[q0:q1].double().transpose(0, 1)       # [Hq, C, D]
        pos = torch.arange(L - C, L)
        mask = t[None, :] <= pos[:, None]                  # [C, L]
        o = torch.nn.functional.scaled_dot_product_attention(q, K, V, attn_mask=mask, scale=wl.scale)
        out[q0:q1] = o.transpose(0, 1).numpy()
    return out


CASES = [
    ("g2_bf16", [0, 37, 5], [40, 21, 1], 8, 4, 64, 16, torch.bfloat16),
    ("g1_f16_bs32", [3, 100], [29, 64], 4, 4, 128, 32, torch.float16),
    ("g4_f32", [17, 0], [1, 33], 8, 2, 64, 16, torch.float32),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_prefill_oracle_matches_torch_sdpa(case):
    name, ctx, ch, hq, hkv, d, bs, dt = case
    wl = W.build_prefill(name, ctx, ch, hq, hkv, d, bs, dt, seed=11)
    kc, vc = caches_after_chunk(wl)
    got = oracle.paged_prefill(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.query_start, wl.scale)
    ref = sdpa_reference(wl, kc, vc)
    assert np.abs(got - ref).max() < 1e-10


def test_one_token_chunks_equal_decode():
    wl = W.build_prefill("decode_like", [0, 15, 16, 200], [1, 1, 1, 1], 8, 2, 64, 16, torch.bfloat16, seed=12)
    kc, vc = caches_after_chunk(wl)
    got = oracle.paged_prefill(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.query_start, wl.scale)
    dec = oracle.paged_attention_decode(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.scale)
    assert np.array_equal(got, dec)


def test_splitting_a_chunk_changes_nothing():
    wl = W.build_prefill("split", [30], [50], 4, 2, 64, 16, torch.float16, seed=13)
    kc, vc = caches_after_chunk(wl)
    whole = oracle.paged_prefill(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.query_start, wl.scale)
    # the same tokens as two chunks: positions 30..49 (seq_len 50), then 50..79
    tables = wl.block_tables.repeat(2, 1)
    lens = torch.tensor([50, 80], dtype=torch.int32)
    qs = torch.tensor([0, 20, 50], dtype=torch.int32)
    parts = oracle.paged_prefill(wl.query, kc, vc, tables, lens, qs, wl.scale)
    assert np.array_equal(whole, parts)


def test_causality():
    wl = W.build_prefill("causal", [8], [24], 4, 4, 64, 16, torch.float32, seed=14)
    kc, vc = caches_after_chunk(wl)
    a = oracle.paged_prefill(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.query_start, wl.scale)
    # overwrite the K/V of positions 20.. (rows for tokens at positions < 20 must not move)
    bs = wl.block_size
    for t in range(20, 32):
        b = int(wl.block_tables[0, t // bs])
        kc[b, t % bs] = 100.0
        vc[b, t % bs] = -100.0
    b_ = oracle.paged_prefill(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.query_start, wl.scale)
    first_changed = 20 - 8                                # chunk row of position 20
    assert np.array_equal(a[:first_changed], b_[:first_changed])
    assert not np.allclose(a[first_changed:], b_[first_changed:])
