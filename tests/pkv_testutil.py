"""Shared helpers for the parity tests: run one decode step on the GPU
(through the C ABI) and on the fp64 oracle from the same seeded workload,
and compare them."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import paged_kv_cache_373_b200 as pkv
from paged_kv_cache_373_b200 import device_inputs
from paged_kv_cache_373_b200 import workloads as W

TOL_16 = 2e-3   # f16 / bf16 / f32 caches, fp32 accumulation (max-abs vs fp64)
TOL_FP8 = 2e-2  # FP8 E4M3 caches, against the oracle on the same dequantised values


def tol_for(wl) -> float:
    return TOL_FP8 if wl.is_fp8 else TOL_16


def half_ulp(x: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """Half a unit in the last place of the output dtype at |x| (storage rounding)."""
    mant = {torch.float32: 23, torch.float16: 10, torch.bfloat16: 7}[dtype]
    emin = {torch.float32: -126, torch.float16: -14, torch.bfloat16: -126}[dtype]
    a = np.maximum(np.abs(x), 2.0 ** emin)
    return 0.5 * 2.0 ** (np.floor(np.log2(a)) - mant)


def fp8_pool_gpu(wl, dev="cuda"):
    """Quantise the FP8 pool sources on the GPU with reshape_and_cache (all slots)."""
    return device_inputs.fp8_pool(wl, dev)


def gpu_inputs(wl, dev="cuda"):
    return device_inputs.decode_inputs(wl, dev)


def gpu_step(wl, g=None, num_ctas: int = 0, dev="cuda"):
    """copy_blocks -> reshape_and_cache -> paged_attention_decode on the GPU."""
    g = g or gpu_inputs(wl, dev)
    if g["pairs"].numel():
        pkv.copy_blocks([g["kc"]], [g["vc"]], g["pairs"])
    pkv.reshape_and_cache(g["nk"], g["nv"], g["kc"], g["vc"], g["slots"], g["ks"], g["vs"])
    out = torch.empty_like(g["q"])
    pkv.paged_attention_decode(out, g["q"], g["kc"], g["vc"], g["tables"], g["lens"], wl.scale,
                               g["ks"], g["vs"], num_ctas=num_ctas)
    err = pkv.get_device_error()
    return out, err, g


def oracle_caches(wl, seqs=None):
    """CPU caches after the oracle's copy_blocks + reshape.  For FP8 pools only
    the slots read by `seqs` (all when None) are quantised."""
    if wl.is_fp8:
        NB, bs, Hkv, D = wl.key_src.shape
        kc = torch.zeros((NB, bs, Hkv, D), dtype=torch.uint8)
        vc = torch.zeros_like(kc)
        sel = range(wl.num_seqs) if seqs is None else seqs
        slots = []
        for s in sel:
            L = int(wl.seq_lens[s])
            t = torch.arange(L)
            slots.append(wl.block_tables[s].long()[t // bs] * bs + t % bs)
        if wl.cow_pairs.numel():
            # copies read their source block: quantise those too
            for src in wl.cow_pairs[:, 0].tolist():
                slots.append(torch.arange(src * bs, (src + 1) * bs))
        sl = torch.unique(torch.cat(slots)) if slots else torch.zeros(0, dtype=torch.int64)
        # new tokens are written by the step itself; their slots are re-written below
        ksrc = wl.key_src.reshape(NB * bs, Hkv, D)[sl].contiguous()
        vsrc = wl.value_src.reshape(NB * bs, Hkv, D)[sl].contiguous()
        oracle.reshape_and_cache(ksrc, vsrc, kc, vc, sl, wl.k_scale, wl.v_scale)
    else:
        kc, vc = wl.key_cache.clone(), wl.value_cache.clone()
    if wl.cow_pairs.numel():
        oracle.copy_blocks([kc], [vc], wl.cow_pairs)
    oracle.reshape_and_cache(wl.new_key, wl.new_value, kc, vc, wl.slot_mapping, wl.k_scale,
                             wl.v_scale)
    return kc, vc


def oracle_step(wl, seqs=None, num_threads: int = 0):
    kc, vc = oracle_caches(wl, seqs)
    return oracle.paged_attention_decode(wl.query, kc, vc, wl.block_tables, wl.seq_lens, wl.scale,
                                         wl.k_scale, wl.v_scale, seq_subset=seqs,
                                         num_threads=num_threads)


def compare(gpu_out: torch.Tensor, ref: np.ndarray, wl, seqs=None):
    """Max-abs error over the compared rows; asserts the tolerance.

    Bound: tol + half an ulp of the output dtype at the reference value (the
    final RNE store to the q dtype is part of the contract)."""
    g = gpu_out.detach().float().cpu().double().numpy()
    if seqs is not None:
        g, ref = g[list(seqs)], ref[list(seqs)]
    assert np.isfinite(g).all(), "non-finite GPU output"
    err = np.abs(g - ref)
    bound = tol_for(wl) + half_ulp(ref, wl.q_dtype)
    worst = float((err - bound).max())
    assert worst <= 0.0, f"{wl.name}: max|err|={err.max():.3e} exceeds bound by {worst:.3e}"
    return float(err.max())
