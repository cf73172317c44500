"""Seeded synthetic inputs for the decode step (no attention arithmetic here).

The pages measure on model workloads (Llama-2-7B / Llama-3-8B / Qwen3 serving
ShareGPT or Alpaca requests); none of those models or datasets is used.  These
generators draw tensors with the same shapes, dtypes, value distributions and
length mixes instead:

  cfg1  tiny fp32 decode: 4 seqs, lengths {1,15,16,37}, 4/4 heads, D=64, bs=16,
        U[-1,1] values, a 16-block pool, scale 1/sqrt(64)
  cfg2  Llama-2-7B-shaped MHA layer: 64 seqs, lengths U[128,2048], 32/32 heads,
        D=128, bs=16, fp16 N(0,1), pool max(4096, needed) blocks, shuffled
  cfg3  Llama-3-8B-shaped GQA layer: 256 seqs, lengths log-uniform [64,8192],
        32/8 heads, D=128, bs=16, bf16 N(0,1), pool = needed + 10 %, shuffled
  cfg4  long-context FP8 KV: 32 seqs, lengths U[16384,32768], 64/8 heads, D=128,
        bs=32, K/V quantised to FP8 E4M3 from N(0,1) bf16 sources with
        per-tensor scales amax/448, bf16 q, pool = needed + 10 %, shuffled
  cfg5  prefix sharing with copy-on-write: 16 prompts x 8 samples, a
        3000-token shared prefix (187 full blocks + one 8-token block, reference
        count 8), per-sample tails U[32,512], 32/8 heads, D=128, bs=16, bf16
  short 2048 seqs of U[1,64] tokens, cfg3's shapes (a large-batch test case,
        not one of the five configurations)

Every sequence's newest token (position seq_len-1) is the decode step's new
token: its K/V are in ``new_key``/``new_value`` and its slot in
``slot_mapping``; ``reshape_and_cache`` must run before the attention call.

Block tables come from :class:`BlockManager` over a shuffled free list (the
physical blocks of a sequence are scattered across the pool); unused table
entries hold -1.  FP8 pools are given as bf16 sources (``key_src`` /
``value_src``) plus scales: the caller quantises them with reshape_and_cache.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import torch

from .block_manager import BlockManager

FP8 = torch.uint8          # storage dtype used for FP8 E4M3 codes
FP8_E4M3_MAX = 448.0       # largest finite E4M3 value (scale calibration only)


@dataclass
class DecodeWorkload:
    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    kv_dtype: torch.dtype            # float32 / float16 / bfloat16, or FP8 (uint8 codes)
    q_dtype: torch.dtype
    scale: float
    query: torch.Tensor              # [S, Hq, D]
    key_cache: Optional[torch.Tensor]    # [NB, bs, Hkv, D]; None for FP8 pools
    value_cache: Optional[torch.Tensor]
    block_tables: torch.Tensor       # int32 [S, max_blocks_per_seq], -1 = unused
    seq_lens: torch.Tensor           # int32 [S]
    new_key: torch.Tensor            # [T, Hkv, D] source dtype
    new_value: torch.Tensor
    slot_mapping: torch.Tensor       # int64 [T], -1 = padding
    key_src: Optional[torch.Tensor] = None    # bf16 [NB, bs, Hkv, D] (FP8 pools)
    value_src: Optional[torch.Tensor] = None
    k_scale: float = 1.0
    v_scale: float = 1.0
    cow_pairs: torch.Tensor = field(default_factory=lambda: torch.zeros((0, 2), dtype=torch.int64))
    meta: dict = field(default_factory=dict)

    @property
    def is_fp8(self) -> bool:
        return self.kv_dtype == FP8

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max().item()) if self.num_seqs else 0

    def kv_elem_bytes(self) -> int:
        return 1 if self.is_fp8 else torch.tensor([], dtype=self.kv_dtype).element_size()

    def algorithmic_bytes(self) -> int:
        """Bytes one decode attention call must move: every K and V row of every
        (sequence, kv head) once, q, the output, the used table entries and
        seq_lens."""
        L = self.seq_lens.to(torch.int64)
        b_kv = self.kv_elem_bytes()
        b_q = torch.tensor([], dtype=self.q_dtype).element_size()
        kv = int(L.sum()) * 2 * self.num_kv_heads * self.head_dim * b_kv
        qo = self.num_seqs * self.num_heads * self.head_dim * 2 * b_q
        tbl = int(((L + self.block_size - 1) // self.block_size).sum()) * 4
        return kv + qo + tbl + 4 * self.num_seqs

    def unique_kv_bytes(self) -> int:
        """KV bytes counting each physical block once (shared prefixes)."""
        seen = set()
        total = 0
        row = self.num_kv_heads * self.head_dim * self.kv_elem_bytes()
        for s in range(self.num_seqs):
            L = int(self.seq_lens[s])
            for i in range((L + self.block_size - 1) // self.block_size):
                b = int(self.block_tables[s, i])
                if b in seen:
                    continue
                seen.add(b)
                total += min(self.block_size, L - i * self.block_size) * row * 2
        return total


# ----------------------------------------------------------------------------
def _fill(shape, dtype, gen: torch.Generator, dist: str, chunk: int = 1 << 24) -> torch.Tensor:
    """Chunked seeded fill (bounded host memory for multi-GB pools)."""
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(-1)
    n = flat.numel()
    for i in range(0, n, chunk):
        m = min(chunk, n - i)
        if dist == "normal":
            x = torch.randn(m, generator=gen, dtype=torch.float32)
        elif dist == "uniform":
            x = torch.rand(m, generator=gen, dtype=torch.float32) * 2.0 - 1.0
        else:
            raise ValueError(dist)
        flat[i:i + m] = x.to(dtype)
    return out


def _amax(*ts: torch.Tensor, chunk: int = 1 << 24) -> float:
    m = 0.0
    for t in ts:
        f = t.reshape(-1)
        for i in range(0, f.numel(), chunk):
            m = max(m, float(f[i:i + chunk].float().abs().max()))
    return m


def build_decode(name: str, seq_lens: Sequence[int], num_heads: int, num_kv_heads: int,
                 head_dim: int, block_size: int, kv_dtype: torch.dtype, q_dtype: torch.dtype,
                 seed: int, dist: str = "normal", num_blocks: Optional[int] = None,
                 min_blocks: int = 0, slack: float = 0.10,
                 scale: Optional[float] = None) -> DecodeWorkload:
    """Generic decode-step workload: one new token per sequence (at seq_len-1)."""
    gen = torch.Generator().manual_seed(seed)
    lens = [int(x) for x in seq_lens]
    S = len(lens)
    need = sum((L + block_size - 1) // block_size for L in lens)
    if num_blocks is None:
        num_blocks = max(min_blocks, need + int(math.ceil(need * slack)), 1)
    if num_blocks < need:
        raise ValueError(f"pool of {num_blocks} blocks < {need} needed")
    free_order = torch.randperm(num_blocks, generator=gen).tolist()
    bm = BlockManager(num_blocks, block_size, free_order)
    slots: List[int] = []
    sids = []
    for L in lens:
        sid = bm.add_sequence(max(L - 1, 0))
        if L > 0:
            slot, cow = bm.append_slot(sid)      # the decode step's new token
            assert cow is None
        else:
            slot = -1
        slots.append(slot)
        sids.append(sid)
    mb = max(1, max(((L + block_size - 1) // block_size for L in lens), default=1))
    tables = torch.full((S, mb), -1, dtype=torch.int32)
    for i, sid in enumerate(sids):
        t = bm.block_table(sid)
        if t:
            tables[i, :len(t)] = torch.tensor(t, dtype=torch.int32)

    fp8 = kv_dtype == FP8
    src_dtype = torch.bfloat16 if fp8 else kv_dtype
    pool_shape = (num_blocks, block_size, num_kv_heads, head_dim)
    kpool = _fill(pool_shape, src_dtype, gen, dist)
    vpool = _fill(pool_shape, src_dtype, gen, dist)
    query = _fill((S, num_heads, head_dim), q_dtype, gen, dist)
    new_k = _fill((S, num_kv_heads, head_dim), src_dtype, gen, dist)
    new_v = _fill((S, num_kv_heads, head_dim), src_dtype, gen, dist)
    wl = DecodeWorkload(
        name=name, num_seqs=S, num_heads=num_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=block_size, num_blocks=num_blocks, kv_dtype=kv_dtype,
        q_dtype=q_dtype, scale=(1.0 / math.sqrt(head_dim)) if scale is None else scale,
        query=query, key_cache=None if fp8 else kpool, value_cache=None if fp8 else vpool,
        block_tables=tables, seq_lens=torch.tensor(lens, dtype=torch.int32),
        new_key=new_k, new_value=new_v, slot_mapping=torch.tensor(slots, dtype=torch.int64),
        meta={"blocks_needed": need, "seed": seed, "dist": dist})
    if fp8:
        wl.key_src, wl.value_src = kpool, vpool
        # per-tensor scales are fp32 device scalars: keep them fp32-representable
        wl.k_scale = float(torch.tensor(_amax(kpool, new_k) / FP8_E4M3_MAX, dtype=torch.float32))
        wl.v_scale = float(torch.tensor(_amax(vpool, new_v) / FP8_E4M3_MAX, dtype=torch.float32))
    return wl


def _seed(cfg: int) -> int:
    return 373 + cfg


def config1() -> DecodeWorkload:
    return build_decode("cfg1_tiny_fp32", [1, 15, 16, 37], 4, 4, 64, 16, torch.float32,
                        torch.float32, _seed(1), dist="uniform", num_blocks=16,
                        scale=1.0 / math.sqrt(64))


def config2(num_seqs: int = 64) -> DecodeWorkload:
    gen = torch.Generator().manual_seed(_seed(2) * 1000)
    lens = torch.randint(128, 2049, (num_seqs,), generator=gen).tolist()
    return build_decode(f"cfg2_llama2_7b_mha_fp16_b{num_seqs}", lens, 32, 32, 128, 16,
                        torch.float16, torch.float16, _seed(2), min_blocks=4096, slack=0.0)


def loguniform_lengths(n: int, lo: int, hi: int, gen: torch.Generator) -> List[int]:
    u = torch.rand(n, generator=gen, dtype=torch.float64)
    L = torch.floor(torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))))
    return L.clamp(lo, hi).to(torch.int64).tolist()


def config3(num_seqs: int = 256) -> DecodeWorkload:
    gen = torch.Generator().manual_seed(_seed(3) * 1000)
    lens = loguniform_lengths(num_seqs, 64, 8192, gen)
    return build_decode(f"cfg3_llama3_8b_gqa_bf16_b{num_seqs}", lens, 32, 8, 128, 16,
                        torch.bfloat16, torch.bfloat16, _seed(3))


def config4(num_seqs: int = 32, lo: int = 16384, hi: int = 32768) -> DecodeWorkload:
    gen = torch.Generator().manual_seed(_seed(4) * 1000)
    lens = torch.randint(lo, hi + 1, (num_seqs,), generator=gen).tolist()
    return build_decode(f"cfg4_longctx_fp8_b{num_seqs}", lens, 64, 8, 128, 32, FP8,
                        torch.bfloat16, _seed(4))


def config5(num_prompts: int = 16, samples: int = 8, prefix: int = 3000,
            tail_lo: int = 32, tail_hi: int = 512, dtype: torch.dtype = torch.bfloat16,
            num_heads: int = 32, num_kv_heads: int = 8, head_dim: int = 128,
            block_size: int = 16) -> DecodeWorkload:
    """Shared prompt prefix + copy-on-write of its partially filled last block.

    Each prompt's prefix is prefilled once and forked ``samples`` times
    (reference count = samples).  Every sample then appends its tail; the first
    tail token lands in the shared partial block, so samples 0..samples-2 copy
    it (copy-on-write) and the last sample writes in place (its reference count
    has dropped to 1).  :func:`with_all_copies` derives the variant in which
    every sample copies.

    Tail tokens before the newest one are synthetic pool contents; the tokens
    that share the copied block take the values the copy brings.  The step
    replays: copy_blocks(cow_pairs) -> reshape_and_cache(new tokens) -> decode.
    """
    bs, Hq, Hkv, D = block_size, num_heads, num_kv_heads, head_dim
    gen = torch.Generator().manual_seed(_seed(5))
    tails = torch.randint(tail_lo, tail_hi + 1, (num_prompts, samples), generator=gen)
    pblocks = (prefix + bs - 1) // bs
    need = num_prompts * pblocks
    for p in range(num_prompts):
        for j in range(samples):
            L = prefix + int(tails[p, j])
            need += (L + bs - 1) // bs - pblocks + 1
    num_blocks = need + int(math.ceil(need * 0.10))
    free_order = torch.randperm(num_blocks, generator=gen).tolist()
    bm = BlockManager(num_blocks, bs, free_order)
    pairs, slots, sids = [], [], []
    for p in range(num_prompts):
        parent = bm.add_sequence(prefix)
        kids = [bm.fork(parent) for _ in range(samples)]
        bm.free(parent)
        for j, sid in enumerate(kids):
            L = prefix + int(tails[p, j])
            for pos in range(prefix, L):
                slot, cow = bm.append_slot(sid)
                if cow is not None:
                    pairs.append(cow)
            slots.append(slot)
            sids.append(sid)
    S = len(sids)
    mb = max(len(bm.block_table(s)) for s in sids)
    tables = torch.full((S, mb), -1, dtype=torch.int32)
    lens = []
    for i, sid in enumerate(sids):
        t = bm.block_table(sid)
        tables[i, :len(t)] = torch.tensor(t, dtype=torch.int32)
        lens.append(bm.seq_len(sid))
    pool_shape = (num_blocks, bs, Hkv, D)
    kpool = _fill(pool_shape, dtype, gen, "normal")
    vpool = _fill(pool_shape, dtype, gen, "normal")
    query = _fill((S, Hq, D), dtype, gen, "normal")
    new_k = _fill((S, Hkv, D), dtype, gen, "normal")
    new_v = _fill((S, Hkv, D), dtype, gen, "normal")
    dname = {torch.bfloat16: "bf16", torch.float16: "fp16", torch.float32: "fp32"}[dtype]
    return DecodeWorkload(
        name=f"cfg5_prefix_cow_{dname}_{num_prompts}x{samples}", num_seqs=S, num_heads=Hq,
        num_kv_heads=Hkv, head_dim=D, block_size=bs, num_blocks=num_blocks,
        kv_dtype=dtype, q_dtype=dtype, scale=1.0 / math.sqrt(D),
        query=query, key_cache=kpool, value_cache=vpool, block_tables=tables,
        seq_lens=torch.tensor(lens, dtype=torch.int32), new_key=new_k, new_value=new_v,
        slot_mapping=torch.tensor(slots, dtype=torch.int64),
        cow_pairs=torch.tensor(pairs, dtype=torch.int64).reshape(-1, 2),
        meta={"prefix": prefix, "samples": samples, "prompts": num_prompts,
              "blocks_needed": need})


def with_all_copies(wl: DecodeWorkload) -> DecodeWorkload:
    """Variant of a prefix-sharing workload in which the last sample of every
    prompt also copies the shared partial block (into a spare pool block)
    instead of writing in place.  Every logical token keeps its value, so the
    decode result must not change."""
    import copy
    bs, prefix, samples = wl.block_size, wl.meta["prefix"], wl.meta["samples"]
    lb = prefix // bs
    used = set(int(b) for b in wl.block_tables.reshape(-1).tolist() if b >= 0)
    used |= set(int(b) for b in wl.cow_pairs.reshape(-1).tolist())
    spare = (b for b in range(wl.num_blocks) if b not in used)
    tables = wl.block_tables.clone()
    slots = wl.slot_mapping.clone()
    pairs = wl.cow_pairs.tolist()
    for p in range(wl.meta["prompts"]):
        s = p * samples + samples - 1
        src = int(tables[s, lb])
        dst = next(spare)
        pairs.append((src, dst))
        tables[s, lb] = dst
        pos = int(wl.seq_lens[s]) - 1              # the new token may sit in that block
        if pos // bs == lb:
            slots[s] = dst * bs + pos % bs
    out = copy.copy(wl)
    out.block_tables = tables
    out.slot_mapping = slots
    out.cow_pairs = torch.tensor(pairs, dtype=torch.int64).reshape(-1, 2)
    out.name = wl.name + "_allcopy"
    out.meta = dict(wl.meta, all_copy=True)
    return out


def cascade_groups(wl: DecodeWorkload):
    """Sharing groups of a prefix-sharing workload (one group per prompt, its
    samples as members, the prompt length as the requested shared prefix):
    (group_offsets int32 [G+1], group_members int32, prefix_lens int32 [G],
    max_group_size)."""
    prompts, samples, prefix = wl.meta["prompts"], wl.meta["samples"], wl.meta["prefix"]
    offsets = torch.arange(0, prompts * samples + 1, samples, dtype=torch.int32)
    members = torch.arange(prompts * samples, dtype=torch.int32)
    prefix_lens = torch.full((prompts,), prefix, dtype=torch.int32)
    return offsets, members, prefix_lens, samples


# ----------------------------------------------------------------------------
# Chunked prefill (ttlab.hopto.org "LLM KV cache 02", section 3: a long prompt
# is cut into chunks that share each step's token budget with decode tokens).
@dataclass
class PrefillWorkload:
    name: str
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    kv_dtype: torch.dtype
    scale: float
    query: torch.Tensor              # [T, Hq, D] the chunks' query rows, sequence after sequence
    query_start: torch.Tensor        # int32 [S+1]
    key_cache: torch.Tensor          # [NB, bs, Hkv, D] context tokens filled, chunk slots not yet
    value_cache: torch.Tensor
    block_tables: torch.Tensor       # int32 [S, max_blocks]
    seq_lens: torch.Tensor           # int32 [S] context + chunk
    new_key: torch.Tensor            # [T, Hkv, D] the chunks' K/V
    new_value: torch.Tensor
    slot_mapping: torch.Tensor       # int64 [T]
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def num_tokens(self) -> int:
        return int(self.query.shape[0])

    @property
    def max_query_len(self) -> int:
        qs = self.query_start
        return int((qs[1:] - qs[:-1]).max()) if self.num_seqs else 0

    def causal_pairs(self) -> int:
        """(query token, attended token) pairs per head: sum over chunk tokens of position + 1."""
        tot = 0
        for s in range(self.num_seqs):
            L = int(self.seq_lens[s])
            C = int(self.query_start[s + 1] - self.query_start[s])
            tot += C * (L - C) + C * (C + 1) // 2
        return tot

    def flops(self) -> int:
        """4 flops per (pair, q head, dim): q.k and p.v, multiply + add."""
        return 4 * self.causal_pairs() * self.num_heads * self.head_dim


def build_prefill(name: str, ctx_lens: Sequence[int], chunk_lens: Sequence[int], num_heads: int,
                  num_kv_heads: int, head_dim: int, block_size: int, dtype: torch.dtype, seed: int,
                  slack: float = 0.10) -> PrefillWorkload:
    """Sequence s has ctx_lens[s] tokens cached and a chunk of chunk_lens[s]
    new tokens: their K/V go to the cache through slot_mapping, then the
    chunk's query rows attend causally over all ctx + chunk tokens."""
    gen = torch.Generator().manual_seed(seed)
    ctx = [int(c) for c in ctx_lens]
    ch = [int(c) for c in chunk_lens]
    lens = [a + b for a, b in zip(ctx, ch)]
    need = sum((L + block_size - 1) // block_size for L in lens)
    num_blocks = max(need + int(math.ceil(need * slack)), 1)
    bm = BlockManager(num_blocks, block_size, torch.randperm(num_blocks, generator=gen).tolist())
    slots: List[int] = []
    tables = []
    for c, n in zip(ctx, ch):
        sid = bm.add_sequence(c)
        for _ in range(n):
            slots.append(bm.append_slot(sid)[0])
        tables.append(bm.block_table(sid))
    mb = max([len(t) for t in tables] + [1])
    bt = torch.full((len(lens), mb), -1, dtype=torch.int32)
    for i, t in enumerate(tables):
        bt[i, :len(t)] = torch.tensor(t, dtype=torch.int32)
    T = sum(ch)
    shape = (num_blocks, block_size, num_kv_heads, head_dim)
    kc = _fill(shape, dtype, gen, "normal")
    vc = _fill(shape, dtype, gen, "normal")
    q = _fill((T, num_heads, head_dim), dtype, gen, "normal")
    nk = _fill((T, num_kv_heads, head_dim), dtype, gen, "normal")
    nv = _fill((T, num_kv_heads, head_dim), dtype, gen, "normal")
    qs = torch.tensor([0] + list(torch.tensor(ch).cumsum(0).tolist()), dtype=torch.int32)
    return PrefillWorkload(
        name=name, num_heads=num_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
        block_size=block_size, num_blocks=num_blocks, kv_dtype=dtype, scale=1.0 / math.sqrt(head_dim),
        query=q, query_start=qs, key_cache=kc, value_cache=vc, block_tables=bt,
        seq_lens=torch.tensor(lens, dtype=torch.int32), new_key=nk, new_value=nv,
        slot_mapping=torch.tensor(slots, dtype=torch.int64), meta={"ctx": ctx, "chunks": ch})


def prefill_config(budget: int = 8192) -> PrefillWorkload:
    """A chunked-prefill step of the ttlab.hopto.org experiment (Qwen3-1.7B
    layer shape: 16 q / 8 kv heads, D=128, bf16, bs=16): three 3,500-token
    inputs arrive while one request decodes; the step's token budget goes to
    the decode token first, then to the inputs' chunks in arrival order.
      budget 8192: two whole inputs (ctx 0, 3500 tokens each), the first 1191
                   tokens of the third, one decode row at length 4500
      budget 2048: the first input's second chunk (ctx 2047, 1453 tokens), the
                   second input's first 594 tokens, one decode row"""
    if budget == 8192:
        ctx, ch = [4499, 0, 0, 0], [1, 3500, 3500, 1191]
    elif budget == 2048:
        ctx, ch = [4499, 2047, 0], [1, 1453, 594]
    else:
        raise ValueError("budget must be 2048 or 8192")
    return build_prefill(f"prefill_qwen3_1p7b_bf16_budget{budget}", ctx, ch, 16, 8, 128, 16,
                         torch.bfloat16, _seed(6) + budget)


def short_batch(num_seqs: int = 2048, lo: int = 1, hi: int = 64) -> DecodeWorkload:
    """A large batch of short sequences (Llama-3-8B GQA layer shapes, bf16):
    lengths U[lo, hi], so the per-sequence work (length scans, unit starts,
    merges) weighs more than in the five configurations."""
    gen = torch.Generator().manual_seed(_seed(7) * 1000)
    lens = torch.randint(lo, hi + 1, (num_seqs,), generator=gen).tolist()
    return build_decode(f"short_llama3_8b_gqa_bf16_b{num_seqs}", lens, 32, 8, 128, 16,
                        torch.bfloat16, torch.bfloat16, _seed(7))


CONFIGS = {1: config1, 2: config2, 3: config3, 4: config4, 5: config5, 7: short_batch}


def make_config(cfg: int, **kw) -> DecodeWorkload:
    return CONFIGS[cfg](**kw)
