"""GPU parity of reshape_and_cache and copy_blocks against the oracle
(bit-exact), through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_373_b200 as pkv

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,D,bs,Hkv", [(torch.float32, 64, 16, 4), (torch.float16, 128, 16, 32),
                                            (torch.bfloat16, 128, 32, 8), (torch.bfloat16, 64, 16, 2)])
def test_reshape_copy_bit_exact(dtype, D, bs, Hkv):
    g = torch.Generator().manual_seed(21)
    NB, T = 37, 200
    kc = torch.randn((NB, bs, Hkv, D), generator=g).to(dtype)
    vc = torch.randn((NB, bs, Hkv, D), generator=g).to(dtype)
    k = torch.randn((T, Hkv, D), generator=g).to(dtype)
    v = torch.randn((T, Hkv, D), generator=g).to(dtype)
    slots = torch.randperm(NB * bs, generator=g)[:T].to(torch.int64)
    slots[::7] = -1                                    # padding tokens
    ok, ov = kc.clone(), vc.clone()
    oracle.reshape_and_cache(k, v, ok, ov, slots)
    dk, dv = kc.cuda(), vc.cuda()
    pkv.reshape_and_cache(k.cuda(), v.cuda(), dk, dv, slots.cuda())
    assert pkv.get_device_error() == 0
    assert torch.equal(dk.cpu().view(torch.uint8), ok.view(torch.uint8))
    assert torch.equal(dv.cpu().view(torch.uint8), ov.view(torch.uint8))


def _fp8_probe_values(dtype):
    """Normal values plus the E4M3 edge cases: exact midpoints (ties), the
    subnormal range, saturation and signed zeros."""
    g = torch.Generator().manual_seed(5)
    x = [torch.randn(4096, generator=g) * 3]
    vals = sorted({oracle.fp8_decode(c) for c in range(0x7F)})
    mids = [(a + b) / 2 for a, b in zip(vals, vals[1:])]
    x.append(torch.tensor(vals + mids + [-v for v in vals + mids], dtype=torch.float64).float())
    x.append(torch.tensor([447.9, 448.0, 449.0, 464.0, 470.0, 1e5, -1e5, 0.0, -0.0,
                           2.0 ** -10, 3 * 2.0 ** -11, 2.0 ** -12, float("inf"), float("-inf")]))
    return torch.cat(x).to(dtype)


@pytest.mark.parametrize("src", [torch.float32, torch.float16, torch.bfloat16])
def test_reshape_fp8_bit_exact(src):
    D, Hkv, bs = 128, 2, 16
    x = _fp8_probe_values(src)
    n = (x.numel() + Hkv * D - 1) // (Hkv * D) * (Hkv * D)
    x = torch.cat([x, torch.zeros(n - x.numel(), dtype=src)])
    T = n // (Hkv * D)
    k = x.reshape(T, Hkv, D)
    v = (-x).reshape(T, Hkv, D).contiguous()
    NB = (T + bs - 1) // bs
    slots = torch.arange(T, dtype=torch.int64)
    for ks, vs in [(1.0, 1.0), (0.0123, 3.7), (2.0 ** -3, 2.0 ** 5)]:
        ok = torch.zeros((NB, bs, Hkv, D), dtype=torch.uint8)
        ov = torch.zeros_like(ok)
        ksf = float(torch.tensor(ks, dtype=torch.float32))
        vsf = float(torch.tensor(vs, dtype=torch.float32))
        oracle.reshape_and_cache(k, v, ok, ov, slots, ksf, vsf)
        dk = torch.zeros_like(ok).cuda()
        dv = torch.zeros_like(ov).cuda()
        pkv.reshape_and_cache(k.cuda(), v.cuda(), dk, dv, slots.cuda(),
                              torch.tensor([ksf], device="cuda"), torch.tensor([vsf], device="cuda"))
        assert pkv.get_device_error() == 0
        mism = (dk.cpu() != ok).nonzero()
        assert mism.numel() == 0, f"K codes differ at {mism[:5].tolist()}"
        assert torch.equal(dv.cpu(), ov)


def test_reshape_fp8_nan_is_nan():
    k = torch.full((1, 1, 128), float("nan"), dtype=torch.float32)
    dk = torch.zeros((1, 16, 1, 128), dtype=torch.uint8, device="cuda")
    dv = torch.zeros_like(dk)
    one = torch.ones(1, device="cuda")
    pkv.reshape_and_cache(k.cuda(), k.cuda(), dk, dv, torch.zeros(1, dtype=torch.int64, device="cuda"),
                          one, one)
    codes = dk[0, 0, 0].cpu()
    assert bool(((codes & 0x7F) == 0x7F).all())        # an E4M3 NaN (S.1111.111)


def test_reshape_bad_slot_flags_and_skips():
    kc = torch.zeros((4, 16, 2, 64), dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    k = torch.ones((2, 2, 64), dtype=torch.float16, device="cuda")
    pkv.reshape_and_cache(k, k, kc, vc, torch.tensor([3, 64], dtype=torch.int64, device="cuda"))
    assert pkv.get_device_error() == pkv.DEVERR_SLOT
    assert float(kc.float().sum()) == 2 * 64              # only the valid slot was written
    assert pkv.get_device_error() == 0                    # cleared


@pytest.mark.parametrize("layers", [1, 3])
def test_copy_blocks_bit_exact(layers):
    g = torch.Generator().manual_seed(layers)
    NB, bs, Hkv, D = 64, 16, 8, 128
    ks = [torch.randn((NB, bs, Hkv, D), generator=g).to(torch.bfloat16) for _ in range(layers)]
    vs = [torch.randn((NB, bs, Hkv, D), generator=g).to(torch.bfloat16) for _ in range(layers)]
    perm = torch.randperm(NB, generator=g)
    pairs = torch.stack([perm[:20], perm[20:40]], 1).to(torch.int64)
    ok, ov = [t.clone() for t in ks], [t.clone() for t in vs]
    oracle.copy_blocks(ok, ov, pairs)
    dk, dv = [t.cuda() for t in ks], [t.cuda() for t in vs]
    pkv.copy_blocks(dk, dv, pairs.cuda())
    assert pkv.get_device_error() == 0
    for a, b in zip(dk + dv, ok + ov):
        assert torch.equal(a.cpu().view(torch.int16), b.view(torch.int16))


def test_copy_blocks_bad_id_flags():
    kc = torch.zeros((4, 16, 2, 64), dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    pkv.copy_blocks([kc], [vc], torch.tensor([[0, 1], [2, 9]], dtype=torch.int64, device="cuda"))
    assert pkv.get_device_error() == pkv.DEVERR_COPY_ID
