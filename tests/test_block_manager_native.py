"""The native host block manager (libpkv.so, include/pkv_block_manager.h)
against the oracle: the same random operation sequences -- prompts with
shared prefixes and salts, forks, single and batched appends, frees, pools
small enough to force evictions and exhaustion -- must give identical block
ids, slots, copy-on-write pairs, cached-token counts, keys and statistics.
Host code only: runs without a GPU."""
import hashlib
import random

import pytest
import torch

import paged_kv_cache_373_b200 as pkv
from oracle.block_manager import OracleBlockManager, OutOfBlocks


def test_sha256_matches_hashlib():
    rng = random.Random(0)
    for n in list(range(0, 130)) + [1000, 4096 + 3]:
        data = bytes(rng.randrange(256) for _ in range(n))
        assert pkv.sha256(data) == hashlib.sha256(data).digest(), n


def _compare_state(nat, orc, live):
    st = nat.stats()
    reserved, tokens = orc.waste()
    assert st["free_blocks"] == len(orc.free)
    assert st["parked_blocks"] == len(orc.parked)
    assert st["cached_blocks"] == len(orc.block_of)
    assert st["reserved_slots"] == reserved and st["token_slots"] == tokens
    assert st["hit_blocks"] == orc.hits and st["evicted_blocks"] == orc.evictions
    assert st["num_seqs"] == len(orc.tables)
    for sid in live:
        assert nat.block_table(sid) == orc.block_table(sid)
        assert nat.seq_len(sid) == orc.seq_len(sid)


def _run(seed, num_blocks, bs, prefix_cache, steps=600):
    rng = random.Random(seed)
    order = rng.sample(range(num_blocks), num_blocks)
    nat = pkv.HostBlockManager(num_blocks, bs, order, prefix_cache)
    orc = OracleBlockManager(num_blocks, bs, order, prefix_cache)
    prompts = [[rng.randrange(1000) for _ in range(rng.randrange(1, 6 * bs))] for _ in range(5)]
    salts = [b"", b"", b"lora:7"]
    live, n_enospc, n_cow = [], 0, 0
    for _ in range(steps):
        op = rng.random()
        if op < 0.2 or not live:
            p = rng.choice(prompts)
            toks = p[:rng.randrange(1, len(p) + 1)] + [rng.randrange(1000) for _ in range(rng.randrange(4))]
            salt = rng.choice(salts)
            try:
                want = orc.add_sequence(toks, salt)
            except OutOfBlocks:
                with pytest.raises(pkv.PkvError) as e:
                    nat.add_sequence(toks, salt)
                assert e.value.status == pkv.PKV_ENOBLOCKS
                n_enospc += 1
            else:
                assert nat.add_sequence(toks, salt) == want
                live.append(want[0])
        elif op < 0.3:
            p = rng.choice(live)
            c = orc.fork(p)
            assert nat.fork(p) == c
            live.append(c)
        elif op < 0.6:
            sid, tok = rng.choice(live), rng.randrange(1000)
            try:
                want = orc.append_token(sid, tok)
            except OutOfBlocks:
                with pytest.raises(pkv.PkvError) as e:
                    nat.append_token(sid, tok)
                assert e.value.status == pkv.PKV_ENOBLOCKS
                n_enospc += 1
            else:
                assert nat.append_token(sid, tok) == want
                n_cow += want[1] is not None
        elif op < 0.85:
            batch = rng.sample(live, rng.randrange(1, len(live) + 1))
            toks = [rng.randrange(1000) for _ in batch]
            # the oracle takes the batch as single appends, all or nothing
            snap = (list(orc.free), list(orc.parked), list(orc.ref), dict(orc.block_of), dict(orc.key_of),
                    {s: list(t) for s, t in orc.tables.items()}, {s: list(t) for s, t in orc.tokens.items()},
                    orc.hits, orc.evictions)
            try:
                want = [orc.append_token(s, t) for s, t in zip(batch, toks)]
            except OutOfBlocks:
                (orc.free, parked, orc.ref, orc.block_of, orc.key_of, orc.tables, orc.tokens,
                 orc.hits, orc.evictions) = snap
                orc.parked.clear()
                orc.parked.update((b, None) for b in parked)
                with pytest.raises(pkv.PkvError) as e:
                    nat.append_batch(batch, toks)
                assert e.value.status == pkv.PKV_ENOBLOCKS
                n_enospc += 1
            else:
                slots, pairs = nat.append_batch(batch, toks)
                assert slots.tolist() == [w[0] for w in want]
                assert [tuple(p) for p in pairs.tolist()] == [w[1] for w in want if w[1] is not None]
        else:
            sid = live.pop(rng.randrange(len(live)))
            orc.free_sequence(sid)
            nat.free_sequence(sid)
        _compare_state(nat, orc, live)
    if prefix_cache:
        for sid in live:
            for i, k in enumerate(orc._keys(sid, orc.seq_len(sid) // bs)):
                assert nat.block_key(sid, i) == k
    nat.close()
    return n_enospc, n_cow, orc.hits, orc.evictions


@pytest.mark.parametrize("seed", range(5))
@pytest.mark.parametrize("num_blocks,bs,prefix_cache", [(48, 4, True), (300, 16, True), (48, 4, False)])
def test_native_matches_oracle(seed, num_blocks, bs, prefix_cache):
    n_enospc, n_cow, hits, evictions = _run(seed, num_blocks, bs, prefix_cache)
    if prefix_cache and num_blocks == 48:
        assert hits > 0 and evictions > 0     # the cache and the LRU were exercised


def test_exercises_exhaustion_and_copy_on_write():
    tot = [0, 0]
    for seed in range(5):
        e, c, _, _ = _run(seed, 32, 4, True)
        tot[0] += e
        tot[1] += c
    assert tot[0] > 0 and tot[1] > 0


def test_batch_tables_and_errors():
    bm = pkv.HostBlockManager(16, 4, prefix_cache=False)
    a, _ = bm.add_sequence(list(range(9)))
    b, _ = bm.add_sequence(list(range(3)))
    t, lens = bm.batch_tables([b, a], 4)
    assert t.tolist() == [[3, -1, -1, -1], [0, 1, 2, -1]] and lens.tolist() == [3, 9]
    with pytest.raises(pkv.PkvError):
        bm.batch_tables([a], 2)                     # row too short
    with pytest.raises(pkv.PkvError):
        bm.free_sequence(77)                        # unknown id
    with pytest.raises(pkv.PkvError):
        bm.append_batch([a, a], [1, 2])             # same sequence twice
    with pytest.raises(pkv.PkvError):
        pkv.HostBlockManager(4, 4, free_order=[0, 1, 1, 2])
    with pytest.raises(pkv.PkvError):
        bm.block_key(a, 0)                          # caching off: no keys
