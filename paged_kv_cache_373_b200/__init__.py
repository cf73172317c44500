"""paged_kv_cache_373_b200 -- B200 (sm_100a) paged KV-cache decode library.

Thin ctypes binding over ``libpkv.so`` (C ABI in include/pkv.h).  Every
function here only marshals arguments: all work runs in the library's CUDA
kernels.  There is no CPU fallback; if the library is missing or the tensors
are not on a CUDA device, the call raises.

Names follow the C entry points without their ``pkv_`` prefix:
  reshape_and_cache, copy_blocks, swap_blocks, paged_attention_decode, paged_prefill,
  paged_attention_decode_noalloc, paged_attention_decode_cascade,
  paged_attention_workspace_bytes, default_num_ctas, decode_step_host, decode_step_layout,
  get_device_error, status_string
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpkv.so")

PKV_F32, PKV_F16, PKV_BF16, PKV_FP8_E4M3 = 0, 1, 2, 3
PKV_OK, PKV_EINVAL, PKV_EUNSUPPORTED, PKV_ECUDA, PKV_EDEVICE, PKV_ENOBLOCKS = 0, 1, 2, 3, 4, 5
DEVERR_BLOCK_ID, DEVERR_SLOT, DEVERR_SEQ_LEN, DEVERR_COPY_ID, DEVERR_TIMEOUT = 1, 2, 4, 8, 16

_DTYPES = {torch.float32: PKV_F32, torch.float16: PKV_F16, torch.bfloat16: PKV_BF16,
           torch.uint8: PKV_FP8_E4M3, torch.float8_e4m3fn: PKV_FP8_E4M3}

EXPORTED = ("pkv_reshape_and_cache", "pkv_copy_blocks", "pkv_swap_blocks", "pkv_paged_attention_workspace_bytes",
            "pkv_default_num_ctas", "pkv_paged_attention_decode",
            "pkv_paged_attention_decode_noalloc", "pkv_paged_attention_cascade_workspace_bytes",
            "pkv_paged_attention_decode_cascade", "pkv_paged_prefill", "pkv_decode_step_host",
            "pkv_decode_step_layout", "pkv_testing_prefill_timeout",
            "pkv_get_device_error", "pkv_status_string", "pkv_last_error_message")


class PkvError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"pkv status {status}: {message}")
        self.status = status


class DecodeStepArgs(ctypes.Structure):
    """Mirror of ``pkv_decode_step_args``."""
    _fields_ = [
        ("num_seqs", ctypes.c_int), ("num_heads", ctypes.c_int), ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("block_size", ctypes.c_int),
        ("max_blocks_per_seq", ctypes.c_int), ("num_blocks", ctypes.c_int64),
        ("q_dtype", ctypes.c_int), ("cache_dtype", ctypes.c_int), ("scale", ctypes.c_float),
        ("num_ctas", ctypes.c_int),
        ("h_query", ctypes.c_void_p), ("h_new_key", ctypes.c_void_p),
        ("h_new_value", ctypes.c_void_p), ("h_slot_mapping", ctypes.c_void_p),
        ("h_block_tables", ctypes.c_void_p), ("h_seq_lens", ctypes.c_void_p),
        ("h_cow_pairs", ctypes.c_void_p), ("num_cow_pairs", ctypes.c_int64),
        ("h_out", ctypes.c_void_p),
        ("d_query", ctypes.c_void_p), ("d_new_key", ctypes.c_void_p),
        ("d_new_value", ctypes.c_void_p), ("d_slot_mapping", ctypes.c_void_p),
        ("d_block_tables", ctypes.c_void_p), ("d_seq_lens", ctypes.c_void_p),
        ("d_cow_pairs", ctypes.c_void_p), ("d_out", ctypes.c_void_p),
        ("key_cache", ctypes.c_void_p), ("value_cache", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("h_packed", ctypes.c_void_p), ("d_packed", ctypes.c_void_p),
    ]


class StepLayout(ctypes.Structure):
    """Mirror of ``pkv_step_layout`` (byte offsets inside one packed input buffer)."""
    _fields_ = [(n, ctypes.c_size_t) for n in ("query", "new_key", "new_value", "slot_mapping",
                                               "block_tables", "seq_lens", "cow_pairs", "total")]


_lib_handle = None


def lib() -> ctypes.CDLL:
    """Load libpkv.so (raises if it has not been built)."""
    global _lib_handle
    if _lib_handle is not None:
        return _lib_handle
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m paged_kv_cache_373_b200._build` (no CPU fallback exists)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
    L.pkv_reshape_and_cache.restype = c_int
    L.pkv_reshape_and_cache.argtypes = [vp, vp, c_int, vp, vp, c_int, vp, i64, i64, c_int, c_int,
                                        c_int, vp, vp, vp]
    L.pkv_copy_blocks.restype = c_int
    L.pkv_copy_blocks.argtypes = [vp, vp, c_int, vp, i64, i64, ctypes.c_size_t, vp]
    L.pkv_swap_blocks.restype = c_int
    L.pkv_swap_blocks.argtypes = [vp, vp, i64, vp, vp, i64, c_int, vp, i64, ctypes.c_size_t, vp]
    L.pkv_paged_attention_workspace_bytes.restype = ctypes.c_size_t
    L.pkv_paged_attention_workspace_bytes.argtypes = [c_int, c_int, c_int, c_int, c_int]
    L.pkv_default_num_ctas.restype = c_int
    L.pkv_default_num_ctas.argtypes = []
    L.pkv_paged_attention_decode.restype = c_int
    L.pkv_paged_attention_decode.argtypes = [vp, vp, c_int, vp, vp, c_int, vp, c_int, vp, c_int,
                                             c_int, c_int, c_int, c_int, i64, ctypes.c_float, vp,
                                             vp, vp, ctypes.c_size_t, c_int, vp]
    L.pkv_paged_attention_decode_noalloc.restype = c_int
    L.pkv_paged_attention_decode_noalloc.argtypes = [vp, vp, c_int, vp, vp, c_int, vp, c_int, vp,
                                                     c_int, c_int, c_int, c_int, c_int, i64,
                                                     ctypes.c_float, vp, vp, c_int, vp]
    L.pkv_paged_attention_cascade_workspace_bytes.restype = ctypes.c_size_t
    L.pkv_paged_attention_cascade_workspace_bytes.argtypes = [c_int] * 7
    L.pkv_paged_attention_decode_cascade.restype = c_int
    L.pkv_paged_attention_decode_cascade.argtypes = [vp, vp, c_int, vp, vp, c_int, vp, c_int, vp, c_int,
                                                     vp, vp, vp, c_int, c_int, c_int, c_int, c_int,
                                                     c_int, i64, ctypes.c_float, vp, vp, vp,
                                                     ctypes.c_size_t, c_int, vp]
    L.pkv_paged_prefill.restype = c_int
    L.pkv_paged_prefill.argtypes = [vp, vp, c_int, vp, vp, c_int, vp, c_int, vp, vp, c_int, i64, c_int,
                                    c_int, c_int, c_int, i64, ctypes.c_float, vp]
    L.pkv_decode_step_host.restype = c_int
    L.pkv_decode_step_host.argtypes = [ctypes.POINTER(DecodeStepArgs), vp]
    L.pkv_decode_step_layout.restype = c_int
    L.pkv_decode_step_layout.argtypes = [c_int, c_int, c_int, c_int, c_int, c_int, i64,
                                         ctypes.POINTER(StepLayout)]
    L.pkv_testing_prefill_timeout.restype = c_int
    L.pkv_testing_prefill_timeout.argtypes = [c_int, ctypes.c_uint64]
    L.pkv_get_device_error.restype = c_int
    L.pkv_get_device_error.argtypes = [ctypes.POINTER(i32), vp]
    L.pkv_status_string.restype = ctypes.c_char_p
    L.pkv_status_string.argtypes = [c_int]
    L.pkv_last_error_message.restype = ctypes.c_char_p
    L.pkv_last_error_message.argtypes = []
    _lib_handle = L
    return L


def _check(status: int) -> None:
    if status != PKV_OK:
        L = lib()
        raise PkvError(status, f"{L.pkv_status_string(status).decode()}: "
                               f"{L.pkv_last_error_message().decode()}")


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dev(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def dtype_code(t: torch.Tensor) -> int:
    return _DTYPES[t.dtype]


def status_string(status: int) -> str:
    return lib().pkv_status_string(status).decode()


def reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, k_scale=None,
                      v_scale=None, stream=None) -> None:
    """key/value [T, Hkv, D] -> caches [NB, bs, Hkv, D] at slot_mapping (int64 [T])."""
    T, Hkv, D = key.shape
    NB, bs = key_cache.shape[0], key_cache.shape[1]
    _check(lib().pkv_reshape_and_cache(
        _dev(key), _dev(value), dtype_code(key), _dev(key_cache), _dev(value_cache),
        dtype_code(key_cache), _dev(slot_mapping), T, NB, bs, Hkv, D, _dev(k_scale), _dev(v_scale),
        _stream(stream)))


def copy_blocks(key_caches: Sequence[torch.Tensor], value_caches: Sequence[torch.Tensor],
                block_mapping: torch.Tensor, stream=None) -> None:
    """Copy whole blocks block_mapping[p,0] -> block_mapping[p,1] in every layer."""
    n = len(key_caches)
    kp = (ctypes.c_void_p * n)(*[_dev(t) for t in key_caches])
    vp = (ctypes.c_void_p * n)(*[_dev(t) for t in value_caches])
    kc = key_caches[0]
    block_bytes = kc[0].numel() * kc.element_size()
    _check(lib().pkv_copy_blocks(kp, vp, n, _dev(block_mapping), block_mapping.shape[0],
                                 kc.shape[0], block_bytes, _stream(stream)))


def paged_prefill(out, query, key_cache, value_cache, block_tables, seq_lens, query_start, scale,
                  stream=None) -> None:
    """Chunked-prefill attention: query/out [T, Hq, D]; sequence s owns rows
    query_start[s]..query_start[s+1]-1, the last of them at position seq_lens[s]-1."""
    T, Hq, D = query.shape
    NB, bs, Hkv, _ = key_cache.shape
    S = seq_lens.shape[0]
    if query_start.shape[0] != S + 1:
        raise ValueError("query_start needs num_seqs + 1 entries")
    _check(lib().pkv_paged_prefill(
        _dev(out), _dev(query), dtype_code(query), _dev(key_cache), _dev(value_cache),
        dtype_code(key_cache), _dev(block_tables), block_tables.shape[1], _dev(seq_lens),
        _dev(query_start), S, T, Hq, Hkv, D, bs, NB, float(scale), _stream(stream)))


def _pool(t: torch.Tensor) -> int:
    """A pool on a CUDA device or in page-locked host memory."""
    if not (t.is_cuda or t.is_pinned()):
        raise ValueError("pool must be on a CUDA device or in pinned host memory")
    if not t.is_contiguous():
        raise ValueError("pool must be contiguous")
    return t.data_ptr()


def swap_blocks(dst_key_caches: Sequence[torch.Tensor], dst_value_caches: Sequence[torch.Tensor],
                src_key_caches: Sequence[torch.Tensor], src_value_caches: Sequence[torch.Tensor],
                block_mapping: torch.Tensor, stream=None) -> None:
    """Copy whole blocks src[block_mapping[p,0]] -> dst[block_mapping[p,1]] in every layer,
    between pools on the device or in pinned host memory (swap out / swap in)."""
    n = len(dst_key_caches)
    if not (len(dst_value_caches) == len(src_key_caches) == len(src_value_caches) == n):
        raise ValueError("every pool list needs one entry per layer")
    dk = (ctypes.c_void_p * n)(*[_pool(t) for t in dst_key_caches])
    dv = (ctypes.c_void_p * n)(*[_pool(t) for t in dst_value_caches])
    sk = (ctypes.c_void_p * n)(*[_pool(t) for t in src_key_caches])
    sv = (ctypes.c_void_p * n)(*[_pool(t) for t in src_value_caches])
    src0, dst0 = src_key_caches[0], dst_key_caches[0]
    block_bytes = src0[0].numel() * src0.element_size()
    if dst0[0].numel() * dst0.element_size() != block_bytes:
        raise ValueError("source and destination blocks differ in size")
    _check(lib().pkv_swap_blocks(dk, dv, dst0.shape[0], sk, sv, src0.shape[0], n,
                                 _pool(block_mapping), block_mapping.shape[0], block_bytes,
                                 _stream(stream)))


def paged_attention_workspace_bytes(num_seqs: int, num_heads: int, num_kv_heads: int,
                                    head_dim: int, num_ctas: int = 0) -> int:
    return int(lib().pkv_paged_attention_workspace_bytes(num_seqs, num_heads, num_kv_heads,
                                                         head_dim, num_ctas))


def default_num_ctas() -> int:
    return int(lib().pkv_default_num_ctas())


def alloc_workspace(num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int,
                    num_ctas: int = 0, device=None) -> torch.Tensor:
    n = paged_attention_workspace_bytes(num_seqs, num_heads, num_kv_heads, head_dim, num_ctas)
    if n == 0:
        raise PkvError(PKV_EINVAL, "invalid workspace shape")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def paged_attention_decode(out, query, key_cache, value_cache, block_tables, seq_lens, scale,
                           k_scale=None, v_scale=None, workspace=None, num_ctas: int = 0,
                           stream=None) -> torch.Tensor:
    """out[S, Hq, D] = decode attention of query over the paged caches."""
    S, Hq, D = query.shape
    NB, bs, Hkv, _ = key_cache.shape
    if workspace is None:
        workspace = alloc_workspace(S, Hq, Hkv, D, num_ctas, device=query.device)
    _check(lib().pkv_paged_attention_decode(
        _dev(out), _dev(query), dtype_code(query), _dev(key_cache), _dev(value_cache),
        dtype_code(key_cache), _dev(block_tables), block_tables.shape[1], _dev(seq_lens), S, Hq,
        Hkv, D, bs, NB, float(scale), _dev(k_scale), _dev(v_scale), _dev(workspace),
        workspace.numel() * workspace.element_size(), int(num_ctas), _stream(stream)))
    return out


STATIC_WORKSPACE_BYTES = 16 * 1024 * 1024   # PKV_STATIC_WORKSPACE_BYTES


def paged_attention_decode_noalloc(out, query, key_cache, value_cache, block_tables, seq_lens,
                                   scale, k_scale=None, v_scale=None, num_ctas: int = 0,
                                   stream=None) -> torch.Tensor:
    """Like paged_attention_decode, with the library's static scratch instead of
    a workspace (see pkv_paged_attention_decode_noalloc)."""
    S, Hq, D = query.shape
    NB, bs, Hkv, _ = key_cache.shape
    _check(lib().pkv_paged_attention_decode_noalloc(
        _dev(out), _dev(query), dtype_code(query), _dev(key_cache), _dev(value_cache),
        dtype_code(key_cache), _dev(block_tables), block_tables.shape[1], _dev(seq_lens), S, Hq,
        Hkv, D, bs, NB, float(scale), _dev(k_scale), _dev(v_scale), int(num_ctas), _stream(stream)))
    return out


def paged_attention_cascade_workspace_bytes(num_seqs: int, num_heads: int, num_kv_heads: int,
                                            head_dim: int, num_groups: int, max_group_size: int,
                                            num_ctas: int = 0) -> int:
    return int(lib().pkv_paged_attention_cascade_workspace_bytes(
        num_seqs, num_heads, num_kv_heads, head_dim, num_groups, max_group_size, num_ctas))


def paged_attention_decode_cascade(out, query, key_cache, value_cache, block_tables, seq_lens,
                                   group_offsets, group_members, group_prefix_lens,
                                   max_group_size: int, scale, k_scale=None, v_scale=None,
                                   workspace=None, num_ctas: int = 0, stream=None) -> torch.Tensor:
    """Decode attention that reads each group's shared prefix blocks once for
    all its members (see pkv_paged_attention_decode_cascade)."""
    S, Hq, D = query.shape
    NB, bs, Hkv, _ = key_cache.shape
    G = group_prefix_lens.shape[0]
    if workspace is None:
        n = paged_attention_cascade_workspace_bytes(S, Hq, Hkv, D, G, max_group_size, num_ctas)
        workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=query.device)
    _check(lib().pkv_paged_attention_decode_cascade(
        _dev(out), _dev(query), dtype_code(query), _dev(key_cache), _dev(value_cache),
        dtype_code(key_cache), _dev(block_tables), block_tables.shape[1], _dev(seq_lens), S,
        _dev(group_offsets), _dev(group_members), _dev(group_prefix_lens), G, int(max_group_size),
        Hq, Hkv, D, bs, NB, float(scale), _dev(k_scale), _dev(v_scale), _dev(workspace),
        workspace.numel() * workspace.element_size(), int(num_ctas), _stream(stream)))
    return out


def decode_step_host(args: DecodeStepArgs, stream=None) -> None:
    """One host-driven decode step (see pkv_decode_step_host); synchronises."""
    _check(lib().pkv_decode_step_host(ctypes.byref(args), _stream(stream)))


def decode_step_layout(num_seqs: int, num_heads: int, num_kv_heads: int, head_dim: int,
                       q_dtype: int, max_blocks_per_seq: int, num_cow_pairs: int = 0) -> StepLayout:
    """Offsets of a decode step's inputs in one packed buffer (pkv_decode_step_layout)."""
    lay = StepLayout()
    _check(lib().pkv_decode_step_layout(num_seqs, num_heads, num_kv_heads, head_dim, q_dtype,
                                        max_blocks_per_seq, num_cow_pairs, ctypes.byref(lay)))
    return lay


def get_device_error(stream=None) -> int:
    """Synchronise, return and clear the device error word (PKV_DEVERR_* bits)."""
    v = ctypes.c_int32(0)
    st = lib().pkv_get_device_error(ctypes.byref(v), _stream(stream))
    if st not in (PKV_OK, PKV_EDEVICE):
        _check(st)
    return int(v.value)


# ---------------------------------------------------------------------------
# Host block manager (include/pkv_block_manager.h): host memory only.
# ---------------------------------------------------------------------------
class BmStats(ctypes.Structure):
    """Mirror of ``pkv_bm_stats``."""
    _fields_ = [(n, ctypes.c_int64) for n in (
        "num_blocks", "block_size", "free_blocks", "parked_blocks", "used_blocks", "cached_blocks",
        "reserved_slots", "token_slots", "hit_blocks", "evicted_blocks", "cow_copies", "num_seqs")]

    def as_dict(self) -> dict:
        return {n: int(getattr(self, n)) for n, _ in self._fields_}


BM_EXPORTED = ("pkv_bm_create", "pkv_bm_destroy", "pkv_bm_add_sequence", "pkv_bm_fork",
               "pkv_bm_append_token", "pkv_bm_append_batch", "pkv_bm_free_sequence",
               "pkv_bm_seq_len", "pkv_bm_block_table", "pkv_bm_batch_tables", "pkv_bm_block_key",
               "pkv_bm_get_stats", "pkv_sha256")


def _bm_lib() -> ctypes.CDLL:
    L = lib()
    if getattr(L, "_bm_ready", False):
        return L
    vp, i64, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    P64 = ctypes.POINTER(i64)
    for name, res, args in (
            ("pkv_bm_create", c_int, [i64, c_int, vp, c_int, ctypes.POINTER(vp)]),
            ("pkv_bm_destroy", None, [vp]),
            ("pkv_bm_add_sequence", c_int, [vp, vp, i64, vp, ctypes.c_size_t, P64, P64]),
            ("pkv_bm_fork", c_int, [vp, i64, P64]),
            ("pkv_bm_append_token", c_int, [vp, i64, ctypes.c_int32, P64, P64, P64]),
            ("pkv_bm_append_batch", c_int, [vp, vp, vp, i64, vp, vp, P64]),
            ("pkv_bm_free_sequence", c_int, [vp, i64]),
            ("pkv_bm_seq_len", c_int, [vp, i64, P64]),
            ("pkv_bm_block_table", c_int, [vp, i64, vp, i64, P64]),
            ("pkv_bm_batch_tables", c_int, [vp, vp, i64, vp, i64, vp]),
            ("pkv_bm_block_key", c_int, [vp, i64, i64, vp]),
            ("pkv_bm_get_stats", c_int, [vp, ctypes.POINTER(BmStats)]),
            ("pkv_sha256", None, [vp, ctypes.c_size_t, vp])):
        f = getattr(L, name)
        f.restype, f.argtypes = res, args
    L._bm_ready = True
    return L


def sha256(data: bytes) -> bytes:
    """The library's SHA-256 (the hash of the block key chain)."""
    out = (ctypes.c_uint8 * 32)()
    _bm_lib().pkv_sha256(data, len(data), out)
    return bytes(out)


class HostBlockManager:
    """Native host block manager: free list, reference counts, copy-on-write
    and the prefix cache (key chain, parked LRU queue).  Raises PkvError with
    status PKV_ENOBLOCKS when the pool is exhausted (nothing changed then)."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None, prefix_cache: bool = True):
        L = _bm_lib()
        self._L = L
        self.block_size = block_size
        fo = None
        if free_order is not None:
            fo = (ctypes.c_int32 * num_blocks)(*[int(b) for b in free_order])
        h = ctypes.c_void_p()
        _check(L.pkv_bm_create(num_blocks, block_size, fo, int(prefix_cache), ctypes.byref(h)))
        self._h = h

    def close(self) -> None:
        if self._h:
            self._L.pkv_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_sequence(self, tokens, extras: bytes = b""):
        toks = (ctypes.c_int32 * len(tokens))(*[int(t) for t in tokens])
        sid, cached = ctypes.c_int64(), ctypes.c_int64()
        _check(self._L.pkv_bm_add_sequence(self._h, toks, len(tokens), extras or None, len(extras),
                                           ctypes.byref(sid), ctypes.byref(cached)))
        return sid.value, cached.value

    def fork(self, parent: int) -> int:
        c = ctypes.c_int64()
        _check(self._L.pkv_bm_fork(self._h, parent, ctypes.byref(c)))
        return c.value

    def append_token(self, sid: int, token: int):
        slot, src, dst = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        _check(self._L.pkv_bm_append_token(self._h, sid, int(token), ctypes.byref(slot),
                                           ctypes.byref(src), ctypes.byref(dst)))
        return slot.value, (None if src.value < 0 else (src.value, dst.value))

    def append_batch(self, sids, tokens):
        """One token per sequence: (slot_mapping int64 tensor, cow pairs int64 [k, 2] tensor)."""
        n = len(sids)
        ids = torch.tensor(list(sids), dtype=torch.int64)
        tok = torch.tensor(list(tokens), dtype=torch.int32)
        slots = torch.empty(n, dtype=torch.int64)
        pairs = torch.empty((n, 2), dtype=torch.int64)
        k = ctypes.c_int64()
        _check(self._L.pkv_bm_append_batch(self._h, ids.data_ptr(), tok.data_ptr(), n, slots.data_ptr(),
                                           pairs.data_ptr(), ctypes.byref(k)))
        return slots, pairs[:k.value].clone()

    def free_sequence(self, sid: int) -> None:
        _check(self._L.pkv_bm_free_sequence(self._h, sid))

    def seq_len(self, sid: int) -> int:
        n = ctypes.c_int64()
        _check(self._L.pkv_bm_seq_len(self._h, sid, ctypes.byref(n)))
        return n.value

    def block_table(self, sid: int):
        n = self.seq_len(sid)
        cap = (n + self.block_size - 1) // self.block_size + 1
        buf = (ctypes.c_int32 * cap)()
        nb = ctypes.c_int64()
        _check(self._L.pkv_bm_block_table(self._h, sid, buf, cap, ctypes.byref(nb)))
        return list(buf[:nb.value])

    def batch_tables(self, sids, max_blocks_per_seq: int):
        """(block_tables int32 [n, max_blocks_per_seq] padded with -1, seq_lens int32 [n])."""
        ids = torch.tensor(list(sids), dtype=torch.int64)
        t = torch.empty((len(sids), max_blocks_per_seq), dtype=torch.int32)
        lens = torch.empty(len(sids), dtype=torch.int32)
        _check(self._L.pkv_bm_batch_tables(self._h, ids.data_ptr(), len(sids), t.data_ptr(),
                                           max_blocks_per_seq, lens.data_ptr()))
        return t, lens

    def block_key(self, sid: int, block_index: int) -> bytes:
        out = (ctypes.c_uint8 * 32)()
        _check(self._L.pkv_bm_block_key(self._h, sid, block_index, out))
        return bytes(out)

    def stats(self) -> dict:
        st = BmStats()
        _check(self._L.pkv_bm_get_stats(self._h, ctypes.byref(st)))
        return st.as_dict()
