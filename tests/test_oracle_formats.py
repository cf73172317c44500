"""Pins for the oracle's number formats and constants (CPU only).

Each check compares the oracle with something other than itself: values the
pages print, the format's published bit layout evaluated by brute force, or an
independent library conversion (numpy float16, torch bfloat16 / float8_e4m3fn).
"""
import math
import os

import numpy as np
import pytest
import torch

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLD, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_kv_bytes_per_token_matches_pages(orc):
    # zwxr.cn section 一: 512 KB/token (Llama-2-7B), 128 KB/token (Llama-3-8B),
    # ~1 GB for 2048 tokens and ~512 MB for 4096 tokens.
    for model, layers, kvh, dim, nb, per_tok, toks, total in _rows("kv_bytes_per_token.txt"):
        got = orc.kv_bytes_per_token(int(layers), int(kvh), int(dim), int(nb))
        assert got == int(per_tok), model
        assert got * int(toks) == int(total), model
    assert orc.kv_bytes_per_token(32, 32, 128, 2) == 512 * 1024
    assert orc.kv_bytes_per_token(32, 8, 128, 2) == 128 * 1024
    # FP8 halves it (zwxr.cn section 五)
    assert orc.kv_bytes_per_token(32, 8, 128, 1) * 2 == orc.kv_bytes_per_token(32, 8, 128, 2)


def test_fp8_reference_points(orc):
    for code, val in _rows("fp8_e4m3_points.txt"):
        c = int(code, 16)
        got = orc.fp8_decode(c)
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


def test_fp8_decode_matches_torch_all_codes(orc):
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        got = orc.fp8_decode(c)
        r = float(ref[c])
        if math.isnan(r):
            assert math.isnan(got)
        else:
            assert got == r, hex(c)


def _fp8_brute_force(x: float) -> int:
    """Nearest finite E4M3 value by exhaustive search; ties to the even code;
    saturate to +-448; NaN -> 0x7F."""
    if math.isnan(x):
        return 0x7F
    if abs(x) >= 448.0:                    # satfinite: clamp to the largest finite
        return 0x7E | (0x80 if x < 0 else 0)
    best, best_err = None, None
    for c in range(256):
        if (c & 0x7F) == 0x7F:
            continue
        s, e, m = c >> 7, (c >> 3) & 0xF, c & 7
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        v = -v if s else v
        if (s == 1) != (math.copysign(1.0, x) < 0):
            continue                       # keep the sign (signed zeros)
        err = abs(v - x)
        if best is None or err < best_err or (err == best_err and (c & 1) == 0 and (best & 1)):
            best, best_err = c, err
    return best


def test_fp8_encode_brute_force(orc):
    rng = np.random.default_rng(373)
    xs = list(rng.normal(0, 30, 3000).astype(np.float32))
    xs += list((rng.normal(0, 0.01, 1000)).astype(np.float32))
    # every midpoint between adjacent codes, and the codes themselves
    vals = sorted({orc.fp8_decode(c) for c in range(0x7F) if not math.isnan(orc.fp8_decode(c))})
    for a, b in zip(vals, vals[1:]):
        for x in (a, b, (a + b) / 2):
            xs += [np.float32(x), np.float32(-x)]
    xs += [np.float32(v) for v in (448.0, 449.0, 463.9, 464.0, 500.0, 1e30, -1e30, 0.0, -0.0,
                                   np.inf, -np.inf, 2.0 ** -10, 2.0 ** -11, 3 * 2.0 ** -11)]
    for x in xs:
        x = float(x)
        want = 0x7E | (0x80 if x < 0 else 0) if math.isinf(x) else _fp8_brute_force(x)
        assert orc.fp8_encode(x) == want, x


def test_fp8_encode_matches_torch_in_range(orc):
    rng = np.random.default_rng(7)
    x = torch.from_numpy(rng.normal(0, 40, 20000).astype(np.float32)).clamp(-440, 440)
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8)
    for i in range(x.numel()):
        assert orc.fp8_encode(float(x[i])) == int(ref[i]), float(x[i])


def test_fp8_nan_and_roundtrip(orc):
    assert orc.fp8_encode(float("nan")) == 0x7F
    for c in range(256):
        v = orc.fp8_decode(c)
        if math.isnan(v):
            continue
        assert orc.fp8_encode(v) == c, hex(c)


def test_f16_bf16_against_libraries(orc):
    rng = np.random.default_rng(11)
    xs = np.concatenate([rng.normal(0, 1, 4000), rng.normal(0, 1e-5, 1000),
                         rng.normal(0, 3e4, 1000), [0.0, -0.0, 65504, 65520, 1e-8, 6e-8, 1e40]])
    f16 = xs.astype(np.float16)
    for x, r in zip(xs, f16):
        assert orc.f16_encode(float(x)) == int(r.view(np.uint16)), x
        assert orc.f16_decode(int(r.view(np.uint16))) == float(r)
    # bf16: torch rounds fp32 -> bf16 with RNE; feed values that are exact in fp32
    xs32 = xs.astype(np.float32)
    bf = torch.from_numpy(xs32).to(torch.bfloat16)
    bits = bf.view(torch.int16).numpy().view(np.uint16)
    for x, b, r in zip(xs32, bits, bf.to(torch.float64).numpy()):
        assert orc.bf16_encode(float(x)) == int(b), x
        assert orc.bf16_decode(int(b)) == float(r)
    # all 65536 bf16 / f16 bit patterns decode like the libraries
    allb = np.arange(65536, dtype=np.uint16)
    ref16 = allb.view(np.float16).astype(np.float64)
    refbf = torch.from_numpy(allb.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    for i in range(0, 65536, 7):
        for got, ref in ((orc.f16_decode(i), ref16[i]), (orc.bf16_decode(i), refbf[i])):
            assert (math.isnan(got) and math.isnan(ref)) or got == ref, i
