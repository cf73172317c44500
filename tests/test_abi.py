"""The C-ABI library loads, exports every entry point include/pkv.h declares,
and rejects bad arguments on the host before touching a GPU (CPU only)."""
import ctypes
import os
import re

import pytest

import paged_kv_cache_373_b200 as pkv
from paged_kv_cache_373_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    _build.build()
    return pkv.lib()


def declared_symbols():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(pkv_[a-z0-9_]+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(L):
    names = declared_symbols()
    assert {"pkv_reshape_and_cache", "pkv_copy_blocks", "pkv_paged_attention_decode"} <= names
    for n in sorted(names):
        assert hasattr(L, n), n
    assert set(pkv.EXPORTED) <= names


def test_status_strings(L):
    for s in range(6):
        assert pkv.status_string(s)
    assert pkv.status_string(99) == "unknown status"


def test_workspace_size_formula(L):
    # (12 workers per CTA x G + S*Hkv*ceil(g/8)) segments x min(g,8) heads
    # x (D floats + one float2), 256-aligned split
    G, S, Hq, Hkv, D = 148, 64, 32, 32, 128
    segs = 12 * G + S * Hkv * 1
    o = segs * 1 * D * 4
    want = ((o + 255) // 256) * 256 + segs * 1 * 8
    assert pkv.paged_attention_workspace_bytes(S, Hq, Hkv, D, G) == want
    # g = 16 -> two head chunks of 8
    segs = 12 * G + 4 * 2 * 2
    o = segs * 8 * 128 * 4
    assert pkv.paged_attention_workspace_bytes(4, 32, 2, 128, G) == ((o + 255) // 256) * 256 + segs * 8 * 8
    assert pkv.paged_attention_workspace_bytes(4, 30, 8, 128, G) == 0     # 30 % 8 != 0


def _decode(L, **kw):
    a = dict(out=None, query=None, q_dtype=pkv.PKV_F16, key_cache=None, value_cache=None,
             cache_dtype=pkv.PKV_F16, block_tables=None, max_blocks_per_seq=4, seq_lens=None,
             num_seqs=2, num_heads=8, num_kv_heads=2, head_dim=128, block_size=16, num_blocks=64,
             scale=0.1, k_scale=None, v_scale=None, workspace=None, workspace_bytes=0, num_ctas=4,
             stream=None)
    a.update(kw)
    return L.pkv_paged_attention_decode(*a.values())


def test_host_validation_without_gpu(L):
    assert _decode(L, head_dim=96) == pkv.PKV_EUNSUPPORTED
    assert _decode(L, block_size=8) == pkv.PKV_EUNSUPPORTED
    assert _decode(L, num_heads=6, num_kv_heads=4) == pkv.PKV_EINVAL
    assert _decode(L, num_seqs=-1) == pkv.PKV_EINVAL
    assert _decode(L, scale=float("nan")) == pkv.PKV_EINVAL
    assert _decode(L, cache_dtype=pkv.PKV_FP8_E4M3, q_dtype=pkv.PKV_F32) == pkv.PKV_EUNSUPPORTED
    assert _decode(L, cache_dtype=pkv.PKV_FP8_E4M3, q_dtype=pkv.PKV_BF16) == pkv.PKV_EINVAL  # no scales
    assert _decode(L, num_seqs=0) == pkv.PKV_OK                      # nothing to do
    assert _decode(L) == pkv.PKV_EINVAL                                # null pointers
    assert b"null" in L.pkv_last_error_message()
    # reshape / copy
    assert L.pkv_reshape_and_cache(None, None, pkv.PKV_F16, None, None, pkv.PKV_BF16, None, 4, 8, 16,
                                   2, 128, None, None, None) == pkv.PKV_EUNSUPPORTED
    assert L.pkv_reshape_and_cache(None, None, pkv.PKV_F16, None, None, pkv.PKV_F16, None, 4, 8, 16,
                                   2, 100, None, None, None) == pkv.PKV_EUNSUPPORTED
    assert L.pkv_reshape_and_cache(None, None, pkv.PKV_F16, None, None, pkv.PKV_F16, None, 0, 8, 16,
                                   2, 128, None, None, None) == pkv.PKV_OK
    assert L.pkv_copy_blocks(None, None, 0, None, 1, 8, 4096, None) == pkv.PKV_EINVAL
    assert L.pkv_copy_blocks(None, None, 1, None, 1, 8, 4095, None) == pkv.PKV_EINVAL
    assert L.pkv_copy_blocks(None, None, 1, None, 0, 8, 4096, None) == pkv.PKV_OK


def test_decode_step_struct_layout():
    # pkv_decode_step_args: 6 ints, int64, 2 enums, float, int, 7 pointers, int64,
    # 9 pointers, 5 pointers, size_t, 2 pointers (packed inputs)
    assert ctypes.sizeof(pkv.DecodeStepArgs) == 248
    assert pkv.DecodeStepArgs.num_blocks.offset == 24
    assert pkv.DecodeStepArgs.h_query.offset == 48
    assert pkv.DecodeStepArgs.workspace_bytes.offset == 224
    assert pkv.DecodeStepArgs.h_packed.offset == 232 and pkv.DecodeStepArgs.d_packed.offset == 240


def test_decode_step_layout_offsets(L):
    # cfg3 shapes: S 256, Hq 32, Hkv 8, D 128, bf16, 512 table entries per sequence
    lay = pkv.decode_step_layout(256, 32, 8, 128, pkv.PKV_BF16, 512, 0)
    sizes = [256 * 32 * 128 * 2, 256 * 8 * 128 * 2, 256 * 8 * 128 * 2, 256 * 8, 256 * 512 * 4, 256 * 4, 0]
    offs = [lay.query, lay.new_key, lay.new_value, lay.slot_mapping, lay.block_tables, lay.seq_lens,
            lay.cow_pairs]
    at = 0
    for off, n in zip(offs, sizes):
        assert off == at and off % 256 == 0
        at = (at + n + 255) // 256 * 256
    assert lay.total == at
    # copy-on-write pairs and odd sizes stay 256-byte aligned and disjoint
    lay = pkv.decode_step_layout(3, 6, 2, 64, pkv.PKV_F32, 5, 7)
    offs = [lay.query, lay.new_key, lay.new_value, lay.slot_mapping, lay.block_tables, lay.seq_lens,
            lay.cow_pairs, lay.total]
    assert all(o % 256 == 0 for o in offs) and offs == sorted(offs)
    assert lay.total - lay.cow_pairs >= 7 * 16
    with pytest.raises(pkv.PkvError):
        pkv.decode_step_layout(-1, 6, 2, 64, pkv.PKV_F32, 5, 0)
    with pytest.raises(pkv.PkvError):
        pkv.decode_step_layout(3, 6, 2, 64, 9, 5, 0)


def test_num_ctas_bound(L):
    assert pkv.paged_attention_workspace_bytes(4, 8, 2, 128, 1 << 20) > 0
    assert pkv.paged_attention_workspace_bytes(4, 8, 2, 128, (1 << 20) + 1) == 0
    assert _decode(L, num_ctas=(1 << 20) + 1) == pkv.PKV_EINVAL
    assert b"num_ctas" in L.pkv_last_error_message()


def _prefill(L, **kw):
    a = dict(out=None, query=None, q_dtype=pkv.PKV_BF16, key_cache=None, value_cache=None,
             cache_dtype=pkv.PKV_BF16, block_tables=None, max_blocks_per_seq=4, seq_lens=None,
             query_start=None, num_seqs=2, num_query_tokens=10, num_heads=8, num_kv_heads=4, head_dim=128,
             block_size=16, num_blocks=64, scale=0.1, stream=None)
    a.update(kw)
    return L.pkv_paged_prefill(*a.values())


def test_prefill_host_validation_without_gpu(L):
    assert _prefill(L, head_dim=96) == pkv.PKV_EUNSUPPORTED
    assert _prefill(L, block_size=8) == pkv.PKV_EUNSUPPORTED
    assert _prefill(L, num_heads=12, num_kv_heads=4) == pkv.PKV_EUNSUPPORTED   # g = 3
    assert _prefill(L, num_heads=6, num_kv_heads=4) == pkv.PKV_EINVAL
    assert _prefill(L, cache_dtype=pkv.PKV_FP8_E4M3) == pkv.PKV_EUNSUPPORTED
    assert _prefill(L, q_dtype=pkv.PKV_F16) == pkv.PKV_EUNSUPPORTED            # q dtype != cache dtype
    assert _prefill(L, q_dtype=pkv.PKV_F32, cache_dtype=pkv.PKV_F32) == pkv.PKV_EUNSUPPORTED
    assert _prefill(L, scale=0.0) == pkv.PKV_EINVAL
    assert _prefill(L, num_query_tokens=-1) == pkv.PKV_EINVAL
    assert _prefill(L, num_blocks=0) == pkv.PKV_EINVAL
    assert _prefill(L, num_seqs=0) == pkv.PKV_OK                               # nothing to do
    assert _prefill(L, num_query_tokens=0) == pkv.PKV_OK
    assert _prefill(L) == pkv.PKV_EINVAL                                        # null pointers
    assert b"null" in L.pkv_last_error_message()


def test_swap_host_validation_without_gpu(L):
    def swap(**kw):
        a = dict(dk=None, dv=None, dnb=64, sk=None, sv=None, snb=64, layers=2, mapping=None, pairs=3,
                 block_bytes=4096, stream=None)
        a.update(kw)
        return L.pkv_swap_blocks(*a.values())
    assert swap(pairs=-1) == pkv.PKV_EINVAL
    assert swap(layers=0) == pkv.PKV_EINVAL
    assert swap(dnb=0) == pkv.PKV_EINVAL
    assert swap(block_bytes=4095) == pkv.PKV_EINVAL
    assert swap(block_bytes=0) == pkv.PKV_EINVAL
    assert swap(pairs=0) == pkv.PKV_OK                                     # nothing to do
    assert swap() == pkv.PKV_EINVAL                                        # null pointers


def test_prefill_timeout_hook_validation(L):
    assert L.pkv_testing_prefill_timeout(-1, 1_000_000) == pkv.PKV_EINVAL
    assert L.pkv_testing_prefill_timeout(0, 10) == pkv.PKV_EINVAL            # below 0.1 ms
    assert L.pkv_testing_prefill_timeout(0, 10**9) == pkv.PKV_EINVAL         # above the normal 0.2 s
    assert L.pkv_testing_prefill_timeout(0, 1_000_000) == pkv.PKV_OK
    assert _prefill(L, num_seqs=0) == pkv.PKV_OK                              # consumes (disarms) it
