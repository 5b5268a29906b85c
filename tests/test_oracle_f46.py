"""Pins of the oracle's FourOverSix quantizer (weights with a tensor scale,
activations with one scale per token).

Model card "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct (our reproduction)",
section "Calibration" (activation bullet) and section "Perplexity"
(round-to-nearest FourOverSix weights).  Pinned by: a hand-derived worked
example (tests/golden/fouroversix_worked.json); an independent numpy model of
the two candidates built on ml_dtypes' E4M3 and E2M1 casts, whose target-6
candidate is the plain NVFP4 round to nearest of the RTN pin; and invariants
(the chosen error is the smaller one, ties keep 6, per-token scales are
fl(amax/2688) and reduce each row to the tensor-scale case).
"""
import json
import os

import ml_dtypes
import numpy as np
import torch

import oracle
from tests.test_oracle_rtn import rtn_nvfp4

F = np.float32
HERE = os.path.dirname(os.path.abspath(__file__))


def bits(Wf):
    Wf = np.asarray(Wf, F)
    Wb = (Wf.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((Wb.astype(np.uint32) << 16).view(F), Wf), "values must be exact in bf16"
    return Wb


def test_worked_example_weights():
    gold = json.load(open(os.path.join(HERE, "golden", "fouroversix_worked.json")))
    u = gold["unit"]
    assert u == 2.0 ** -12
    g = gold["weights"]
    W = bits(np.array(g["W_over_u"], np.float64) * u)
    r = oracle.fouroversix(W, F(g["s_over_u"] * u))
    ex = g["expected"]
    np.testing.assert_array_equal(r.scales, np.array(ex["scales"], np.uint8))
    np.testing.assert_array_equal(r.four, np.array(ex["four"], np.uint8))
    np.testing.assert_array_equal(r.codes, np.array(ex["codes"], np.uint8))
    np.testing.assert_array_equal(r.errs, (np.array(ex["errs_over_u2"]) * u * u).astype(F))
    assert ex["Xq_equals_W"] and np.array_equal(r.Xq, W)


def test_worked_example_tokens():
    gold = json.load(open(os.path.join(HERE, "golden", "fouroversix_worked.json")))
    u = gold["unit"]
    g = gold["tokens"]
    X = bits(np.array(g["X_over_u"], np.float64) * u)
    r = oracle.fouroversix(X)
    ex = g["expected"]
    np.testing.assert_array_equal(r.row_scales, np.array(ex["row_scales_over_u"], F) * F(u))
    np.testing.assert_array_equal(r.scales, np.array(ex["scales"], np.uint8))
    np.testing.assert_array_equal(r.four, np.array(ex["four"], np.uint8))
    np.testing.assert_array_equal(r.codes[0], np.array(ex["codes_row0"], np.uint8))
    assert not r.codes[1].any()
    assert ex["Xq_equals_X"] and np.array_equal(r.Xq, X)


LD = np.longdouble


def fma32(a, b, c):
    """fl32(a*b + c) with one rounding, for binary32 arrays: a*b is exact in the
    64-bit significand of x87 extended precision, and so is the sum unless c
    dwarfs a*b, where both roundings give c's neighbourhood alike."""
    assert np.finfo(LD).nmant >= 63
    return (a.astype(LD) * b.astype(LD) + c.astype(LD)).astype(F)


def candidate(Wf, s, T):
    """Independent numpy model of one target: scale bytes, codes, bf16 values, squared errors
    (binary32: d = fl(w - c*S*s) in one rounding, even and odd elements summed apart by
    fused multiply-adds in index order, then added)."""
    out, inn = Wf.shape
    b = Wf.reshape(-1, 16)
    A = np.abs(b).max(1)
    x = A / (F(T) * s)
    x = np.where(x == 0, F(1), x)
    x = np.clip(x, F(2.0 ** -6), F(448)).astype(F)
    sb = x.astype(ml_dtypes.float8_e4m3fn)
    S = sb.astype(F)
    D = S * s
    y = b / D[:, None]
    c8 = np.clip(y, F(-6), F(6)).astype(ml_dtypes.float4_e2m1fn)
    c = c8.astype(F)
    cS = c * S[:, None]                                       # exact
    E = [np.zeros(b.shape[0], F), np.zeros(b.shape[0], F)]
    for i in range(16):
        d = fma32(-cS[:, i], np.full(b.shape[0], s, F), b[:, i])
        E[i & 1] = fma32(d, d, E[i & 1])
    err = (E[0] + E[1]).astype(F)
    wq = (c * S[:, None]) * s
    wq16 = torch.from_numpy(wq.astype(F)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return (sb.view(np.uint8).reshape(out, inn // 16), (c8.view(np.uint8) & 0xF).reshape(out, inn),
            wq16.reshape(out, inn), err.reshape(out, inn // 16))


def _weights(out, inn, seed, scale=0.02):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(out, inn, generator=g) * scale).to(torch.bfloat16)
    idx = torch.randint(0, out * inn, (out * inn // 300,), generator=g)
    W.view(-1)[idx] = (W.view(-1)[idx].float() * 20).to(torch.bfloat16)
    W[0, :16] = 0
    return W.view(torch.int16).numpy().view(np.uint16), W.float().numpy()


def test_target6_candidate_is_plain_rtn():
    Wb, Wf = _weights(64, 256, 3)
    s2 = oracle.s2(Wb)
    sb, codes, wq, _ = candidate(Wf, s2, 6)
    rsb, rcodes, rwq = rtn_nvfp4(Wf, s2)
    np.testing.assert_array_equal(sb, rsb)
    np.testing.assert_array_equal(codes, rcodes)
    np.testing.assert_array_equal(wq, rwq)


def test_against_independent_model_weights():
    Wb, Wf = _weights(96, 512, 4)
    s2 = oracle.s2(Wb)
    r = oracle.fouroversix(Wb, s2)
    c6 = candidate(Wf, s2, 6)
    c4 = candidate(Wf, s2, 4)
    np.testing.assert_array_equal(r.errs[..., 0], c6[3])
    np.testing.assert_array_equal(r.errs[..., 1], c4[3])
    four = c4[3] < c6[3]
    np.testing.assert_array_equal(r.four, four.astype(np.uint8))
    assert 0.05 < four.mean() < 0.95, "both targets should be chosen on Gaussian weights"
    np.testing.assert_array_equal(r.scales, np.where(four, c4[0], c6[0]))
    fe = np.repeat(four, 16, axis=1)
    np.testing.assert_array_equal(r.codes, np.where(fe, c4[1], c6[1]))
    np.testing.assert_array_equal(r.Xq, np.where(fe, c4[2], c6[2]))
    # the chosen error is the smaller one
    chosen = np.where(four, r.errs[..., 1], r.errs[..., 0])
    assert np.all(chosen <= r.errs.min(-1))


def test_per_token_rows_reduce_to_tensor_scale():
    Xb, Xf = _weights(40, 320, 5, scale=1.0)
    Xb[7, :] = 0                                     # a padding token
    Xf[7, :] = 0
    r = oracle.fouroversix(Xb)
    want = (np.abs(Xf).max(1).astype(F) / F(2688)).astype(F)
    np.testing.assert_array_equal(r.row_scales, want)
    for t in (0, 1, 13, 39):
        rt = oracle.fouroversix(Xb[t:t + 1], want[t])
        np.testing.assert_array_equal(r.codes[t], rt.codes[0])
        np.testing.assert_array_equal(r.scales[t], rt.scales[0])
        np.testing.assert_array_equal(r.Xq[t], rt.Xq[0])
    assert np.all(r.scales[7] == 0x38) and not r.codes[7].any() and not r.Xq[7].any()


def test_tie_keeps_six():
    # every block holds one value v*u, u = 2^-12, s = u: targets 6 and 4 both exact
    # (S6 = v/6, S4 = v/4 representable in E4M3) so both errors are 0
    u = 2.0 ** -12
    vals = [12.0, 24.0, 6.0, 48.0, 96.0]
    W = np.zeros((len(vals), 16))
    W[:, 3] = np.array(vals) * u
    r = oracle.fouroversix(bits(W), F(u))
    assert np.all(r.errs == 0) and not r.four.any()
    want = [int(np.float32(v / 6).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)) for v in vals]
    np.testing.assert_array_equal(r.scales[:, 0], want)
    assert np.all(r.codes[:, 3] == 7)
