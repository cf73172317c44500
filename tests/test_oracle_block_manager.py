"""Pins of the block-manager oracle against facts fixed by the pages and by
arithmetic: the waste of paging in closed form, the prefix-cache key chain
(sha256 as the pages name it, checked against hashlib's published digests),
hits only under the same prefix and extras, tail-first LRU eviction, the
copy-on-write count of parallel sampling, and the bookkeeping invariants
after random operation sequences."""
import hashlib
import random

import pytest

from oracle.block_manager import ROOT_KEY, OracleBlockManager, OutOfBlocks, block_key


def _check_invariants(bm: OracleBlockManager):
    refs = [0] * bm.num_blocks
    for t in bm.tables.values():
        for b in t:
            refs[b] += 1
    assert refs == bm.ref
    used = {b for b in range(bm.num_blocks) if refs[b] > 0}
    free, parked = set(bm.free), set(bm.parked)
    assert len(free) == len(bm.free)
    assert not (used & free) and not (used & parked) and not (free & parked)
    assert used | free | parked == set(range(bm.num_blocks))
    assert parked <= set(bm.key_of)            # parked blocks keep their keys
    assert all(bm.block_of[k] == b for b, k in bm.key_of.items())
    for sid, t in bm.tables.items():
        assert len(t) == (len(bm.tokens[sid]) + bm.bs - 1) // bm.bs


def test_sha256_known_digests():
    # FIPS 180-4 example messages
    assert hashlib.sha256(b"abc").hexdigest() == \
        "ba7816bf8f01cfea414140de5dae2223b00361a396177a9cb410ff61f20015ad"
    assert hashlib.sha256(b"").hexdigest() == \
        "e3b0c44298fc1c149afbf4c8996fb92427ae41e4649b934ca495991b7852b855"
    k = block_key(ROOT_KEY, [1, 2], b"x")
    assert k == hashlib.sha256(bytes(32) + b"\x01\x00\x00\x00\x02\x00\x00\x00x").digest()


def test_waste_is_the_tail_of_each_last_block():
    # paging wastes only the unused slots of each sequence's last block
    bs = 16
    lens = [1, 15, 16, 17, 100, 2048, 33]
    bm = OracleBlockManager(1000, bs, prefix_cache=False)
    for i, L in enumerate(lens):
        bm.add_sequence([i] * L)
    reserved, tokens = bm.waste()
    assert tokens == sum(lens)
    assert reserved == sum(-(-L // bs) * bs for L in lens)
    assert reserved - tokens == sum((-L) % bs for L in lens)


def test_key_chain_depends_on_the_whole_prefix():
    # the same 16 tokens give different keys after different prefixes
    bs = 16
    a = list(range(100, 132))
    b = list(range(200, 216)) + list(range(116, 132))
    assert a[16:] == b[16:]
    bm = OracleBlockManager(64, bs)
    sa, _ = bm.add_sequence(a)
    sb, cached = bm.add_sequence(b)
    assert cached == 0
    ka, kb = bm._keys(sa, 2), bm._keys(sb, 2)
    assert ka[1] != kb[1]
    assert ka[1] == block_key(block_key(ROOT_KEY, a[:16]), a[16:])


def test_prefix_hits_need_same_tokens_and_extras():
    bs = 16
    prompt = list(range(3000 % 97, 3000 % 97 + 70))     # 4 full blocks + 6 tokens
    bm = OracleBlockManager(64, bs)
    s0, c0 = bm.add_sequence(prompt)
    assert c0 == 0
    s1, c1 = bm.add_sequence(prompt[:64] + [7] * 10)
    assert c1 == 64 and bm.tables[s1][:4] == bm.tables[s0][:4]
    s2, c2 = bm.add_sequence(prompt, extras=b"salt")
    assert c2 == 0
    s3, c3 = bm.add_sequence(prompt[:40])
    assert c3 == 32                                        # two full blocks
    assert bm.hits == 6
    _check_invariants(bm)


def test_finished_request_parks_tail_first_and_lru_evicts_it_first():
    bs = 4
    bm = OracleBlockManager(6, bs)
    s, _ = bm.add_sequence(list(range(12)))               # 3 full cached blocks
    t = bm.tables[s]
    bm.free_sequence(s)
    assert list(bm.parked) == [t[2], t[1], t[0]]          # tail enters first
    other, _ = bm.add_sequence([99] * 16)                  # 3 free + 1 evicted
    assert bm.evictions == 1 and t[2] not in bm.parked
    # the head of the prompt is still cached and found again
    again, cached = bm.add_sequence(list(range(8)))
    assert cached == 8 and bm.tables[again] == [t[0], t[1]]
    _check_invariants(bm)


def test_parallel_sampling_copy_on_write_count():
    # prompt 3000 tokens (187 full + 1 partial block), 8 samples: the first
    # token of samples 0..6 copies the shared partial block, the 8th writes
    # in place (its reference count has dropped to 1)
    bs, samples = 16, 8
    bm = OracleBlockManager(200 + 16, bs, prefix_cache=False)
    parent, _ = bm.add_sequence([1] * 3000)
    kids = [bm.fork(parent) for _ in range(samples)]
    bm.free_sequence(parent)
    cows = [bm.append_token(k, 5)[1] for k in kids]
    assert sum(c is not None for c in cows) == samples - 1
    assert cows[-1] is None
    _check_invariants(bm)


def test_out_of_blocks_changes_nothing():
    bm = OracleBlockManager(4, 4)
    s, _ = bm.add_sequence(list(range(12)))
    before = (list(bm.free), list(bm.parked), list(bm.ref), dict(bm.block_of))
    with pytest.raises(OutOfBlocks):
        bm.add_sequence(list(range(50, 58)))
    assert before == (list(bm.free), list(bm.parked), list(bm.ref), dict(bm.block_of))


@pytest.mark.parametrize("seed", range(6))
def test_invariants_after_random_operations(seed):
    rng = random.Random(seed)
    bm = OracleBlockManager(40, 4, free_order=rng.sample(range(40), 40))
    prefixes = [[rng.randrange(50) for _ in range(rng.randrange(1, 20))] for _ in range(4)]
    live = []
    for _ in range(400):
        op = rng.random()
        try:
            if op < 0.25 or not live:
                p = rng.choice(prefixes)
                live.append(bm.add_sequence(p + [rng.randrange(50) for _ in range(rng.randrange(6))])[0])
            elif op < 0.35:
                live.append(bm.fork(rng.choice(live)))
            elif op < 0.85:
                bm.append_token(rng.choice(live), rng.randrange(50))
            else:
                bm.free_sequence(live.pop(rng.randrange(len(live))))
        except OutOfBlocks:
            pass
        _check_invariants(bm)
