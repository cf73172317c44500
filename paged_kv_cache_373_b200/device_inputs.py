"""Put a seeded decode workload (workloads.py) on the device.

Input staging only: the tensors are copied as they are, except FP8 pools,
which are given as bf16 sources plus per-tensor scales and are quantised on
the device by this library's own reshape_and_cache (every slot of the pool).
Used by bench.py and by the tests; nothing here computes attention.
"""
from __future__ import annotations

import torch

from . import reshape_and_cache


def fp8_pool(wl, dev="cuda"):
    """(key_cache, value_cache, k_scale, v_scale) on `dev`: the FP8 E4M3 codes of
    the workload's bf16 pool sources, written by reshape_and_cache in bounded
    slices (about 256 MB of bf16 staging at a time)."""
    NB, bs, Hkv, D = wl.key_src.shape
    kc = torch.empty((NB, bs, Hkv, D), dtype=torch.uint8, device=dev)
    vc = torch.empty_like(kc)
    ks = torch.tensor([wl.k_scale], dtype=torch.float32, device=dev)
    vs = torch.tensor([wl.v_scale], dtype=torch.float32, device=dev)
    rows = NB * bs
    step = max(1, (1 << 28) // (Hkv * D * 2))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        k = wl.key_src.reshape(rows, Hkv, D)[r0:r1].to(dev)
        v = wl.value_src.reshape(rows, Hkv, D)[r0:r1].to(dev)
        slots = torch.arange(r0, r1, dtype=torch.int64, device=dev)
        reshape_and_cache(k, v, kc, vc, slots, ks, vs)
    return kc, vc, ks, vs


def decode_inputs(wl, dev="cuda") -> dict:
    """Every input of one decode step, resident on `dev`:
    kc/vc (pools), ks/vs (FP8 scales or None), q, tables, lens, nk/nv (the new
    tokens' K/V rows), slots (their slot mapping) and pairs (copy-on-write)."""
    if wl.is_fp8:
        kc, vc, ks, vs = fp8_pool(wl, dev)
    else:
        kc, vc = wl.key_cache.to(dev), wl.value_cache.to(dev)
        ks = vs = None
    return dict(kc=kc, vc=vc, ks=ks, vs=vs, q=wl.query.to(dev), tables=wl.block_tables.to(dev),
                lens=wl.seq_lens.to(dev), nk=wl.new_key.to(dev), nv=wl.new_value.to(dev),
                slots=wl.slot_mapping.to(dev), pairs=wl.cow_pairs.to(dev))
