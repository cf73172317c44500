"""pkv_paged_attention_decode_noalloc: decode attention for callers that cannot
allocate device memory when they decode (an engine whose KV pool already holds
the device memory, a plugin without access to its framework's allocator, a
decode loop that must not synchronise on cudaMalloc).  It uses the library's
static scratch array instead of a caller workspace.

Called through the C ABI and checked against the workspace entry point on the
same inputs, within the attention tolerance, on two calls in a row (the second
call finds the first call's leftovers in the shared array).  This file is
collected last so that a failure here leaves every other test already run."""
import ctypes

import pytest
import torch

import paged_kv_cache_373_b200 as pkv
from paged_kv_cache_373_b200 import workloads as W
from pkv_testutil import compare, gpu_inputs, gpu_step, oracle_step

pytestmark = pytest.mark.gpu

vp = ctypes.c_void_p


def _noalloc(wl, g, out, num_ctas=0):
    S, Hq, D = g["q"].shape
    NB, bs, Hkv, _ = g["kc"].shape
    ptr = lambda t: None if t is None else t.data_ptr()
    return pkv.lib().pkv_paged_attention_decode_noalloc(
        out.data_ptr(), g["q"].data_ptr(), pkv.dtype_code(g["q"]), g["kc"].data_ptr(),
        g["vc"].data_ptr(), pkv.dtype_code(g["kc"]), g["tables"].data_ptr(),
        g["tables"].shape[1], g["lens"].data_ptr(), S, Hq, Hkv, D, bs, NB, wl.scale,
        ptr(g["ks"]), ptr(g["vs"]), num_ctas, torch.cuda.current_stream().cuda_stream)


def test_noalloc_matches_workspace_entry_point_twice():
    cases = [W.build_decode("noalloc_gqa", [1, 40, 300, 1025, 2048], 32, 8, 128, 16,
                            torch.bfloat16, torch.bfloat16, seed=51),
             W.build_decode("noalloc_fp8", [7, 500, 3000], 64, 8, 128, 32, W.FP8,
                            torch.bfloat16, seed=52)]
    for wl in cases:                      # two calls in a row, different shapes
        ref, err, g = gpu_step(wl)        # workspace entry point (after the step's writes)
        assert err == 0
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(wl, g, out) == pkv.PKV_OK
        assert pkv.get_device_error() == 0
        compare(out, ref.double().cpu().numpy(), wl)
        compare(out, oracle_step(wl), wl)


def test_noalloc_repeat_same_inputs():
    wl = W.build_decode("noalloc_rep", [33, 700, 1500], 16, 2, 128, 16, torch.float16,
                        torch.float16, seed=53)
    ref, err, g = gpu_step(wl, num_ctas=20)
    outs = []
    for _ in range(2):
        out = torch.empty_like(ref)
        assert _noalloc(wl, g, out, num_ctas=20) == pkv.PKV_OK
        outs.append(out)
    assert pkv.get_device_error() == 0
    for out in outs:
        compare(out, ref.double().cpu().numpy(), wl)


def test_noalloc_rejects_oversize_request():
    # 4096 sequences x 8 kv heads x 2 head chunks needs more than the static scratch
    S, Hq, Hkv, D = 4096, 128, 8, 128
    need = pkv.paged_attention_workspace_bytes(S, Hq, Hkv, D, 0)
    assert need > pkv.STATIC_WORKSPACE_BYTES
    wl = W.build_decode("tiny", [5], 16, 8, 128, 16, torch.bfloat16, torch.bfloat16, seed=54)
    g = gpu_inputs(wl)
    st = pkv.lib().pkv_paged_attention_decode_noalloc(
        g["q"].data_ptr(), g["q"].data_ptr(), pkv.PKV_BF16, g["kc"].data_ptr(), g["vc"].data_ptr(),
        pkv.PKV_BF16, g["tables"].data_ptr(), 1, g["lens"].data_ptr(), S, Hq, Hkv, D, 16,
        wl.num_blocks, 0.1, None, None, 0, None)
    assert st == pkv.PKV_EINVAL
    assert b"static scratch" in pkv.lib().pkv_last_error_message()


def test_noalloc_warmup_then_no_device_allocation():
    """The set-up the header asks for: one num_seqs = 0 call per device (it
    commits the static scratch under lazy module loading); after it, decode
    calls leave the device's free memory unchanged."""
    wl = W.build_decode("noalloc_mem", [3, 90, 700, 1600], 32, 8, 128, 16, torch.bfloat16,
                        torch.bfloat16, seed=55)
    ref, err, g = gpu_step(wl)                       # loads the decode kernels, allocates the inputs
    assert err == 0
    NB, bs, Hkv, D = g["kc"].shape
    st = pkv.lib().pkv_paged_attention_decode_noalloc(
        None, None, pkv.PKV_BF16, None, None, pkv.PKV_BF16, None, g["tables"].shape[1], None, 0,
        32, Hkv, D, bs, NB, wl.scale, None, None, 0, torch.cuda.current_stream().cuda_stream)
    assert st == pkv.PKV_OK
    outs = [torch.empty_like(ref) for _ in range(2)]
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for out in outs:
        assert _noalloc(wl, g, out) == pkv.PKV_OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, f"device free memory changed by {free0 - free1} bytes"
    assert pkv.get_device_error() == 0
    for out in outs:
        compare(out, ref.double().cpu().numpy(), wl)
