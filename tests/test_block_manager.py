"""Host block manager: allocation on demand, reference counts, copy-on-write.

Behaviour follows zwxr.cn sections 3.1 / 3.2 / 3.4 and ttlab.hopto.org
section 2 (only the last block of a sequence holds unused slots).
"""
import pytest

from paged_kv_cache_373_b200.block_manager import BlockManager, OutOfBlocks


def test_blocks_allocated_on_demand_and_returned_whole():
    bm = BlockManager(8, 16)
    sid = bm.add_sequence(0)
    assert bm.block_table(sid) == []
    slot, cow = bm.append_slot(sid)
    assert slot == 0 and cow is None and bm.num_free == 7
    for _ in range(15):
        bm.append_slot(sid)
    assert len(bm.block_table(sid)) == 1          # 16 tokens fill exactly one block
    bm.append_slot(sid)
    assert len(bm.block_table(sid)) == 2 and bm.num_free == 6
    bm.free(sid)
    assert bm.num_free == 8


def test_only_last_block_has_unused_slots():
    bm = BlockManager(64, 16)
    sids = [bm.add_sequence(n) for n in (1, 16, 17, 100, 37)]
    reserved, tokens = bm.used_slots_waste()
    assert reserved - tokens == sum((-n) % 16 for n in (1, 16, 17, 100, 37))
    for sid, n in zip(sids, (1, 16, 17, 100, 37)):
        assert len(bm.block_table(sid)) == (n + 15) // 16


def test_fork_shares_and_copy_on_write():
    bm = BlockManager(32, 16)
    parent = bm.add_sequence(40)            # blocks: 2 full + 1 partial (8 tokens)
    kids = [bm.fork(parent) for _ in range(3)]
    bm.free(parent)
    shared = bm.block_table(kids[0])
    assert all(bm.refcount[b] == 3 for b in shared)
    pairs = []
    for k in kids:
        slot, cow = bm.append_slot(k)
        if cow:
            pairs.append(cow)
    # the first two writers copy the shared partial block, the last writes in place
    assert len(pairs) == 2 and all(src == shared[2] for src, _ in pairs)
    assert bm.block_table(kids[2])[2] == shared[2]
    assert bm.refcount[shared[2]] == 1
    assert all(bm.refcount[b] == 3 for b in shared[:2])   # full blocks stay shared
    # slots point into each writer's own last block, offset 8
    for k in kids:
        assert bm.slot_of(k, 40) == bm.block_table(k)[2] * 16 + 8


def test_out_of_blocks_and_bad_order():
    bm = BlockManager(2, 4)
    bm.add_sequence(8)
    with pytest.raises(OutOfBlocks):
        bm.add_sequence(1)
    with pytest.raises(ValueError):
        BlockManager(3, 4, [0, 0, 1])


def test_shuffled_free_order_scatters_blocks():
    order = [5, 2, 7, 0, 1, 3, 4, 6]
    bm = BlockManager(8, 16, order)
    sid = bm.add_sequence(50)
    assert bm.block_table(sid) == [5, 2, 7, 0]
