"""fp64 CPU oracle for the paged KV-cache decode hot path -- TEST INFRASTRUCTURE.

Only tests/, ``__graft_entry__.smoke()`` and bench.py's CPU-baseline leg may
import this module.  The product package (paged_kv_cache_373_b200) never
imports it and shares no code with it; the C source lives in pkv_oracle.c.

All inputs are torch CPU tensors (or numpy arrays) holding the stored bytes;
the oracle widens them itself with its own decoders and computes in fp64.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import build as _build

DT_F32, DT_F16, DT_BF16, DT_FP8 = 0, 1, 2, 3
_TORCH_DT = {torch.float32: DT_F32, torch.float16: DT_F16, torch.bfloat16: DT_BF16,
             torch.uint8: DT_FP8, torch.float8_e4m3fn: DT_FP8}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        c_void, c_i64, c_i32, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
        L.oracle_f16_decode.restype = ctypes.c_double
        L.oracle_f16_decode.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_decode.restype = ctypes.c_double
        L.oracle_bf16_decode.argtypes = [ctypes.c_uint16]
        L.oracle_f16_encode.restype = ctypes.c_uint16
        L.oracle_f16_encode.argtypes = [ctypes.c_double]
        L.oracle_bf16_encode.restype = ctypes.c_uint16
        L.oracle_bf16_encode.argtypes = [ctypes.c_double]
        L.oracle_fp8_e4m3_decode.restype = ctypes.c_double
        L.oracle_fp8_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_fp8_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_fp8_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_kv_bytes_per_token.restype = c_i64
        L.oracle_kv_bytes_per_token.argtypes = [c_int, c_int, c_int, c_int]
        L.oracle_reshape_and_cache.restype = c_int
        L.oracle_reshape_and_cache.argtypes = [c_void, c_void, c_int, c_void, c_void, c_int,
                                               c_void, c_i64, c_i64, c_int, c_int, c_int,
                                               ctypes.c_float, ctypes.c_float]
        L.oracle_copy_blocks.restype = c_int
        L.oracle_copy_blocks.argtypes = [c_void, c_void, c_int, c_void, c_i64, c_i64, c_i64]
        L.oracle_paged_prefill.restype = c_int
        L.oracle_paged_prefill.argtypes = [c_void, c_void, c_int, c_void, c_void, c_int, c_void, c_int,
                                           c_void, c_void, c_int, c_int, c_int, c_int, c_int, c_i64,
                                           ctypes.c_double, ctypes.c_float, ctypes.c_float, c_int]
        L.oracle_swap_blocks.restype = c_int
        L.oracle_swap_blocks.argtypes = [c_void, c_void, c_i64, c_void, c_void, c_i64, c_int, c_void,
                                         c_i64, c_i64]
        L.oracle_paged_attention_decode.restype = c_int
        L.oracle_paged_attention_decode.argtypes = [
            c_void, c_void, c_int, c_void, c_void, c_int, c_void, c_int, c_void, c_int, c_int,
            c_int, c_int, c_int, c_i64, ctypes.c_double, ctypes.c_float, ctypes.c_float,
            c_void, c_int, c_int]
        L.oracle_blockwise_attend.restype = c_int
        L.oracle_blockwise_attend.argtypes = [c_void, c_void, c_void, c_void, c_int, c_int,
                                              ctypes.c_double, c_int]
        L.oracle_contiguous_attend.restype = c_int
        L.oracle_contiguous_attend.argtypes = [c_void, c_void, c_void, c_void, c_int, c_int,
                                               ctypes.c_double]
        L.oracle_gather_kv.restype = c_int
        L.oracle_gather_kv.argtypes = [c_void, c_void, c_void, c_void, c_int, c_void, c_int,
                                       c_int, c_i64, c_int, c_int, c_int, ctypes.c_float,
                                       ctypes.c_float]
        L.oracle_num_threads_available.restype = c_int
        L.oracle_num_threads_available.argtypes = []
        _lib = L
    return _lib


def _ptr(t):
    if isinstance(t, np.ndarray):
        assert t.flags["C_CONTIGUOUS"]
        return t.ctypes.data
    assert t.device.type == "cpu" and t.is_contiguous()
    return t.data_ptr()


def dtype_code(t) -> int:
    return _TORCH_DT[t.dtype]


# -- scalar format helpers --------------------------------------------------
def f16_decode(bits: int) -> float: return lib().oracle_f16_decode(bits)
def bf16_decode(bits: int) -> float: return lib().oracle_bf16_decode(bits)
def f16_encode(x: float) -> int: return lib().oracle_f16_encode(x)
def bf16_encode(x: float) -> int: return lib().oracle_bf16_encode(x)
def fp8_decode(code: int) -> float: return lib().oracle_fp8_e4m3_decode(code)
def fp8_encode(x: float) -> int: return lib().oracle_fp8_e4m3_encode(x)


def kv_bytes_per_token(layers: int, kv_heads: int, head_dim: int, nbytes: int) -> int:
    return lib().oracle_kv_bytes_per_token(layers, kv_heads, head_dim, nbytes)


def round_to_dtype(x: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """fp64 -> stored dtype (RNE) -> fp64, with the oracle's own encoders."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    flat, of = x.reshape(-1), out.reshape(-1)
    L = lib()
    if dtype == torch.float32:
        return x.astype(np.float32).astype(np.float64)
    enc, dec = ((L.oracle_f16_encode, L.oracle_f16_decode) if dtype == torch.float16
                else (L.oracle_bf16_encode, L.oracle_bf16_decode))
    for i in range(flat.size):
        of[i] = dec(enc(float(flat[i])))
    return out


# -- hot-path reference functions --------------------------------------------
def reshape_and_cache(key, value, key_cache, value_cache, slot_mapping,
                      k_scale: float = 1.0, v_scale: float = 1.0) -> None:
    """In place on the CPU caches. key/value [T, Hkv, D]; caches [NB, bs, Hkv, D]."""
    T, Hkv, D = key.shape
    NB, bs = key_cache.shape[0], key_cache.shape[1]
    sm = slot_mapping.to(torch.int64).contiguous()
    rc = lib().oracle_reshape_and_cache(
        _ptr(key), _ptr(value), dtype_code(key), _ptr(key_cache), _ptr(value_cache),
        dtype_code(key_cache), _ptr(sm), T, NB, bs, Hkv, D, float(k_scale), float(v_scale))
    if rc != 0:
        raise ValueError(f"oracle_reshape_and_cache failed: {rc}")


def copy_blocks(key_caches, value_caches, block_mapping) -> None:
    """In place. key_caches/value_caches: lists of CPU tensors [NB, ...]."""
    n = len(key_caches)
    kp = (ctypes.c_void_p * n)(*[_ptr(t) for t in key_caches])
    vp = (ctypes.c_void_p * n)(*[_ptr(t) for t in value_caches])
    bm = block_mapping.to(torch.int64).contiguous()
    NB = key_caches[0].shape[0]
    block_bytes = key_caches[0][0].numel() * key_caches[0].element_size()
    rc = lib().oracle_copy_blocks(ctypes.addressof(kp), ctypes.addressof(vp), n, _ptr(bm),
                                  bm.shape[0], block_bytes, NB)
    if rc != 0:
        raise ValueError(f"oracle_copy_blocks failed: {rc}")


def swap_blocks(dst_key_caches, dst_value_caches, src_key_caches, src_value_caches,
                block_mapping) -> None:
    """dst pools modified in place; every pool a list (per layer) of CPU tensors [NB, ...]."""
    n = len(dst_key_caches)
    arr = lambda ts: (ctypes.c_void_p * n)(*[_ptr(t) for t in ts])
    dk, dv, sk, sv = arr(dst_key_caches), arr(dst_value_caches), arr(src_key_caches), arr(src_value_caches)
    bm = block_mapping.to(torch.int64).contiguous()
    block_bytes = src_key_caches[0][0].numel() * src_key_caches[0].element_size()
    rc = lib().oracle_swap_blocks(ctypes.addressof(dk), ctypes.addressof(dv), dst_key_caches[0].shape[0],
                                  ctypes.addressof(sk), ctypes.addressof(sv), src_key_caches[0].shape[0],
                                  n, _ptr(bm), bm.shape[0], block_bytes)
    if rc != 0:
        raise ValueError(f"oracle_swap_blocks failed: {rc}")


def paged_attention_decode(query, key_cache, value_cache, block_tables, seq_lens, scale,
                           k_scale: float = 1.0, v_scale: float = 1.0, seq_subset=None,
                           num_threads: int = 0) -> np.ndarray:
    """fp64 [S, Hq, D] output (rows outside seq_subset are left as NaN)."""
    S, Hq, D = query.shape
    NB, bs, Hkv, D2 = key_cache.shape
    assert D == D2
    bt = block_tables.to(torch.int32).contiguous()
    sl = seq_lens.to(torch.int32).contiguous()
    out = np.full((S, Hq, D), np.nan, dtype=np.float64)
    if seq_subset is None:
        sub_ptr, nsub = None, -1
    else:
        sub = np.ascontiguousarray(np.asarray(seq_subset, dtype=np.int32))
        sub_ptr, nsub = sub.ctypes.data, sub.size
    rc = lib().oracle_paged_attention_decode(
        out.ctypes.data, _ptr(query), dtype_code(query), _ptr(key_cache), _ptr(value_cache),
        dtype_code(key_cache), _ptr(bt), bt.shape[1], _ptr(sl), S, Hq, Hkv, D, bs, NB,
        float(scale), float(k_scale), float(v_scale), sub_ptr, nsub, int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle_paged_attention_decode failed: {rc}")
    return out


def paged_prefill(query, key_cache, value_cache, block_tables, seq_lens, query_start, scale,
                  k_scale: float = 1.0, v_scale: float = 1.0, num_threads: int = 0) -> np.ndarray:
    """Chunked-prefill attention, fp64 [T, Hq, D]: the chunk of sequence s is
    query rows query_start[s]..query_start[s+1]-1, ending at position seq_lens[s]-1."""
    T, Hq, D = query.shape
    NB, bs, Hkv, D2 = key_cache.shape
    assert D == D2
    bt = block_tables.to(torch.int32).contiguous()
    sl = seq_lens.to(torch.int32).contiguous()
    qs = query_start.to(torch.int32).contiguous()
    assert int(qs[-1]) == T
    out = np.zeros((T, Hq, D), dtype=np.float64)
    rc = lib().oracle_paged_prefill(
        out.ctypes.data, _ptr(query), dtype_code(query), _ptr(key_cache), _ptr(value_cache),
        dtype_code(key_cache), _ptr(bt), bt.shape[1], _ptr(sl), _ptr(qs), sl.shape[0], Hq, Hkv, D,
        bs, NB, float(scale), float(k_scale), float(v_scale), int(num_threads))
    if rc != 0:
        raise ValueError(f"oracle_paged_prefill failed: {rc}")
    return out


def blockwise_attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float,
                     part: int) -> np.ndarray:
    q, K, V = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, K, V))
    out = np.empty(q.shape[0], dtype=np.float64)
    rc = lib().oracle_blockwise_attend(out.ctypes.data, q.ctypes.data, K.ctypes.data,
                                       V.ctypes.data, K.shape[0], q.shape[0], scale, part)
    assert rc == 0
    return out


def contiguous_attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    q, K, V = (np.ascontiguousarray(a, dtype=np.float64) for a in (q, K, V))
    out = np.empty(q.shape[0], dtype=np.float64)
    lib().oracle_contiguous_attend(out.ctypes.data, q.ctypes.data, K.ctypes.data,
                                   V.ctypes.data, K.shape[0], q.shape[0], scale)
    return out


def gather_kv(key_cache, value_cache, table_row, L: int, kvh: int,
              k_scale: float = 1.0, v_scale: float = 1.0):
    """fp64 K[L, D], V[L, D] of one kv head through one block-table row."""
    NB, bs, Hkv, D = key_cache.shape
    tr = torch.as_tensor(table_row, dtype=torch.int32).contiguous()
    K = np.empty((max(L, 1), D), dtype=np.float64)
    V = np.empty((max(L, 1), D), dtype=np.float64)
    rc = lib().oracle_gather_kv(K.ctypes.data, V.ctypes.data, _ptr(key_cache), _ptr(value_cache),
                                dtype_code(key_cache), _ptr(tr), L, bs, NB, Hkv, kvh, D,
                                float(k_scale), float(v_scale))
    if rc != 0:
        raise ValueError(f"oracle_gather_kv failed: {rc}")
    return K[:L], V[:L]


def num_threads_available() -> int:
    return lib().oracle_num_threads_available()
