"""Pins of the oracle's scalar codecs against the mathematics and library casts.

* E2M1: the value set {0, 0.5, 1, 1.5, 2, 3, 4, 6} and ties to even (model card
  "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct", "What this is", the rule after
  the equations); checked against an argmin over the 15 signed values written
  here and against ml_dtypes' float4_e2m1fn cast.
* E4M3: all 256 bytes decoded from the format's definition; every fp32 in the
  clamp range [2^-6, 448] of the S_b equation encoded, against torch's and
  ml_dtypes' float8_e4m3fn casts.
* bf16 rounding against torch's cast; sigmoid against a 50-digit evaluation.
"""
import ctypes
import decimal
import math

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

E2M1_VALUES = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def argmin_e2m1(u: float) -> int:
    """Nearest of the 15 signed E2M1 values; at a tie the even code; zero keeps u's sign."""
    best = None
    for code in range(16):
        if code == 8:
            continue  # -0 is handled by the sign rule below
        v = E2M1_VALUES[code & 7] * (-1.0 if code & 8 else 1.0)
        d = abs(u - v)
        if best is None or d < best[0] or (d == best[0] and (code & 1) == 0 and (best[1] & 1) == 1):
            best = (d, code)
    code = best[1]
    if (code & 7) == 0 and math.copysign(1.0, u) < 0:
        code = 8
    return code


def test_e2m1_value_set_and_ties():
    assert [oracle.e2m1_decode(c) for c in range(8)] == E2M1_VALUES
    assert [oracle.e2m1_decode(c) for c in range(8, 16)] == [-v for v in E2M1_VALUES]
    ties = {0.25: 0.0, 0.75: 1.0, 1.25: 1.0, 1.75: 2.0, 2.5: 2.0, 3.5: 4.0, 5.0: 4.0}
    for t, v in ties.items():
        assert oracle.e2m1_decode(oracle.e2m1_encode(t)) == v
        assert oracle.e2m1_decode(oracle.e2m1_encode(-t)) == -v
    assert oracle.e2m1_encode(-0.0) == 8 and oracle.e2m1_encode(0.0) == 0
    assert oracle.e2m1_encode(-0.1) == 8
    assert oracle.e2m1_encode(6.0) == 7 and oracle.e2m1_encode(-6.0) == 15


def _edge_values():
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0] + E2M1_VALUES[1:]
    vals = []
    for mpt in mids:
        x = np.float32(mpt)
        lo = hi = x
        for _ in range(4):
            lo = np.nextafter(lo, np.float32(-np.inf)); hi = np.nextafter(hi, np.float32(np.inf))
            vals += [lo, hi]
        vals.append(x)
    vals = np.array(vals, np.float32)
    return np.concatenate([vals, -vals, np.array([0.0, -0.0, 1e-30, -1e-30], np.float32)])


def test_e2m1_edges_against_argmin_and_ml_dtypes():
    vals = _edge_values()
    for u in vals:
        c = oracle.e2m1_encode(float(u))
        assert c == argmin_e2m1(float(u)), (u, c)
    lib = vals.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    ours = np.array([oracle.e2m1_encode(float(u)) for u in vals], np.uint8)
    np.testing.assert_array_equal(ours, lib)


def test_e2m1_all_bf16_in_range_against_ml_dtypes():
    h = np.arange(65536, dtype=np.uint32)
    f = (h << 16).view(np.float32)
    f = f[np.isfinite(f) & (np.abs(f) <= 6.0)]
    lib = f.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    # the oracle's encoder through its scalar entry point, on every 7th value plus all near edges
    sample = f[::7]
    ours = np.array([oracle.e2m1_encode(float(u)) for u in sample], np.uint8)
    np.testing.assert_array_equal(ours, lib[::7])


def test_e2m1_dense_random_against_ml_dtypes():
    rng = np.random.default_rng(11)
    u = (rng.uniform(-6.0, 6.0, 20000)).astype(np.float32)
    lib = u.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    ours = np.array([oracle.e2m1_encode(float(x)) for x in u], np.uint8)
    np.testing.assert_array_equal(ours, lib)


def e4m3_by_definition(b: int) -> float:
    s, e, mnt = (b >> 7) & 1, (b >> 3) & 15, b & 7
    if e == 15 and mnt == 7:
        return math.nan
    v = mnt * 2.0 ** -9 if e == 0 else (1 + mnt / 8) * 2.0 ** (e - 7)
    return -v if s else v


def test_e4m3_decode_all_bytes():
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for b in range(256):
        ours = oracle.e4m3_decode(b)
        ref = e4m3_by_definition(b)
        if math.isnan(ref):
            assert math.isnan(ours) and math.isnan(lib[b])
        else:
            assert ours == ref == lib[b], b
    assert oracle.e4m3_decode(0x7E) == 448.0 and oracle.e4m3_decode(0x08) == 2.0 ** -6
    assert oracle.e4m3_decode(0x38) == 1.0


def test_e4m3_roundtrip_and_midpoints():
    for b in range(0x00, 0x7F):
        v = e4m3_by_definition(b)
        assert oracle.e4m3_encode(v) == b, b
    # midpoints between neighbours in [2^-6, 448]: ties go to the even mantissa
    for b in range(0x08, 0x7E):
        lo, hi = e4m3_by_definition(b), e4m3_by_definition(b + 1)
        mid = (lo + hi) / 2
        assert np.float32(mid) == mid
        want = b if (b & 1) == 0 else b + 1
        assert oracle.e4m3_encode(mid) == want, (b, mid)
        assert oracle.e4m3_encode(float(np.nextafter(np.float32(mid), np.float32(0)))) == b
        assert oracle.e4m3_encode(float(np.nextafter(np.float32(mid), np.float32(1e9)))) == b + 1


def _fo_e4m3_vector():
    L = oracle.lib()
    return L.fo_e4m3_encode


def test_e4m3_strided_fp32_and_samples_against_torch():
    # fp32 in [1, 4) every 97 ulps and in [256, 448] every 13 ulps, plus 200k log-uniform samples over [2^-6, 448]
    a = np.arange(np.float32(1.0).view(np.uint32), np.float32(4.0).view(np.uint32), 97, dtype=np.uint32)
    b = np.arange(np.float32(256.0).view(np.uint32), np.float32(448.0).view(np.uint32) + 1, 13,
                  dtype=np.uint32)
    rng = np.random.default_rng(5)
    c = np.exp2(rng.uniform(-6, math.log2(448), 200000)).astype(np.float32)
    x = np.concatenate([a.view(np.float32), b.view(np.float32), c, np.float32([2.0 ** -6, 448.0])])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref2 = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(ref, ref2)
    enc = _fo_e4m3_vector()
    ours = np.fromiter((enc(float(v)) for v in x), dtype=np.int64, count=x.size).astype(np.uint8)
    np.testing.assert_array_equal(ours, ref)


def test_bf16_rounding_against_torch():
    rng = np.random.default_rng(3)
    u = rng.integers(0, 2 ** 32, 50000, dtype=np.uint64).astype(np.uint32)
    # add exact ties and their neighbours
    t = (rng.integers(0, 2 ** 16, 2000, dtype=np.uint64).astype(np.uint32) << 16) | 0x8000
    u = np.concatenate([u, t, t + 1, t - 1])
    f = u.view(np.float32)
    f = f[np.isfinite(f)]
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    ours = np.array([oracle.bf16_from_f32(float(v)) for v in f], np.uint16)
    np.testing.assert_array_equal(ours, ref)
    for h in (0x0000, 0x8000, 0x3F80, 0x7F7F, 0x0001, 0x8001):
        assert oracle.bf16_from_f32(oracle.f32_from_bf16(h)) == h


def _sigmoid_50(q: float) -> decimal.Decimal:
    with decimal.localcontext() as ctx:
        ctx.prec = 60
        return 1 / (1 + decimal.Decimal(-q).exp())


def test_sigmoid_correctly_rounded_on_sample():
    rng = np.random.default_rng(9)
    qs = np.concatenate([rng.normal(6, 2, 3000), rng.uniform(-20, 20, 3000),
                         [0.0, 6.0, -8.0, 12.0, 17.5, 30.0, -30.0]]).astype(np.float32)
    bad = 0
    for q in qs:
        s = oracle.sigmoid(float(q))
        exact = _sigmoid_50(float(q))
        # nearest binary32 to the exact value
        lo = np.float32(float(exact))
        cands = [np.nextafter(lo, np.float32(-1)), lo, np.nextafter(lo, np.float32(2))]
        best = min(cands, key=lambda c: abs(decimal.Decimal(float(c)) - exact))
        bad += (np.float32(s) != best)
    assert bad == 0
    assert oracle.sigmoid(0.0) == 0.5
    assert oracle.sigmoid(30.0) == 1.0 and oracle.sigmoid(17.5) == 1.0
    assert oracle.sigmoid(17.0) < 1.0
