"""Pins of the oracle's FourOverSix quantizer (weights with a tensor scale,
activations with one scale per token).

Model card "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct (our reproduction)",
section "Calibration" (activation bullet) and section "Perplexity"
(round-to-nearest FourOverSix weights).  The "lower error" is the squared
error of the dequantized block as an exact number.  Pinned by: a hand-derived
worked example (tests/golden/fouroversix_worked.json); an independent numpy
model of the two candidates built on ml_dtypes' E4M3 and E2M1 casts, whose
target-6 candidate is the plain NVFP4 round to nearest of the RTN pin, with
the errors summed as rationals (fractions.Fraction); blocks with equal nonzero
errors (ties keep 6); the exact comparison against rationals, including
differences binary64 sums lose; and invariants (per-token scales are
fl(amax/2688) and reduce each row to the tensor-scale case).
"""
import json
import os
from fractions import Fraction

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
    np.testing.assert_array_equal(r.errs, np.array(ex["errs_over_u2"]) * u * u)
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


def candidate(Wf, s, T):
    """Independent model of one target on ml_dtypes' E4M3 and E2M1 casts (the
    binary32 decisions: scale byte, codes, bf16 values).  Returns also c*S*s of
    every element, exact in binary64 (at most 30 significant bits)."""
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
    cS = c * S[:, None]                                       # exact in binary32
    v = cS.astype(np.float64) * np.float64(s)                 # exact in binary64
    wq = (c * S[:, None]) * s
    wq16 = torch.from_numpy(wq.astype(F)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return (sb.view(np.uint8).reshape(out, inn // 16), (c8.view(np.uint8) & 0xF).reshape(out, inn),
            wq16.reshape(out, inn), v)


def exact_sq_err(wrow, vrow):
    """sum_i (w_i - v_i)^2 as an exact rational (the definition of the error)."""
    return sum((Fraction(float(a)) - Fraction(float(b))) ** 2 for a, b in zip(wrow, vrow))


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
    """The choice follows the exact squared errors: computed here with rationals
    from the independent model's dequantized values, block by block."""
    Wb, Wf = _weights(96, 512, 4)
    s2 = oracle.s2(Wb)
    r = oracle.fouroversix(Wb, s2)
    c6 = candidate(Wf, s2, 6)
    c4 = candidate(Wf, s2, 4)
    wb = Wf.reshape(-1, 16)
    e6 = [exact_sq_err(w, v) for w, v in zip(wb, c6[3])]
    e4 = [exact_sq_err(w, v) for w, v in zip(wb, c4[3])]
    four = np.array([a < b for a, b in zip(e4, e6)]).reshape(r.four.shape)
    np.testing.assert_array_equal(r.four, four.astype(np.uint8))
    assert 0.05 < four.mean() < 0.95, "both targets should be chosen on Gaussian weights"
    np.testing.assert_array_equal(r.scales, np.where(four, c4[0], c6[0]))
    fe = np.repeat(four, 16, axis=1)
    np.testing.assert_array_equal(r.codes, np.where(fe, c4[1], c6[1]))
    np.testing.assert_array_equal(r.Xq, np.where(fe, c4[2], c6[2]))
    # the reported errors are the binary64 sums: within 2^-48 of the exact values
    for k, ex in ((0, e6), (1, e4)):
        got = r.errs[..., k].reshape(-1)
        for g, x in zip(got, ex):
            assert abs(Fraction(float(g)) - x) <= Fraction(1, 2 ** 48) * x


def test_ties_with_nonzero_error_keep_six():
    """Blocks found by search (s = 1) whose two targets have equal, nonzero exact
    squared errors: 6 is kept and both errors are reported equal."""
    blocks = [(1.125, 0.25), (1.125, 1.0), (1.5, 0.875), (1.875, 1.75), (2.25, 2.0), (3.0, 0.625)]
    W = np.zeros((len(blocks), 16))
    W[:, 0] = [a for a, _ in blocks]
    W[:, 5] = [b for _, b in blocks]
    Wb = bits(W)
    r = oracle.fouroversix(Wb, F(1))
    c6 = candidate(W.astype(F), F(1), 6)
    c4 = candidate(W.astype(F), F(1), 4)
    for j in range(len(blocks)):
        e6, e4 = exact_sq_err(W[j], c6[3][j]), exact_sq_err(W[j], c4[3][j])
        assert e6 == e4 != 0
        assert r.errs[j, 0, 0] == r.errs[j, 0, 1] == float(e6)
    assert not r.four.any()
    np.testing.assert_array_equal(r.scales, c6[0])


def _golden_ties():
    gold = json.load(open(os.path.join(HERE, "golden", "fouroversix_ties.json")))
    W = np.array([[int(x, 16) for x in b["w_bits"]] for b in gold["blocks"]], np.uint16)
    s2 = np.array([b["s2_bits"] for b in gold["blocks"]], np.uint32).view(F)
    return W, s2


def test_ties_in_gaussian_weights_keep_six():
    """Blocks of the synthetic 8B weights whose two targets tie exactly (inputs in
    tests/golden/fouroversix_ties.json): the tie is derived here with rationals,
    then the oracle must keep 6 and report equal errors."""
    W, s2 = _golden_ties()
    for wb, s in zip(W, s2):
        wf = (wb.astype(np.uint32) << 16).view(F)[None, :]
        c6, c4 = candidate(wf, s, 6), candidate(wf, s, 4)
        e6, e4 = exact_sq_err(wf[0], c6[3][0]), exact_sq_err(wf[0], c4[3][0])
        assert e6 == e4 != 0 and c6[0][0, 0] != c4[0][0, 0]
        r = oracle.fouroversix(wb[None, :], s)
        assert r.four[0, 0] == 0 and r.scales[0, 0] == c6[0][0, 0]
        np.testing.assert_array_equal(r.codes[0], c6[1][0])
        assert oracle.f46_exact_sign((wf[0]).astype(np.float64), c4[3][0], c6[3][0]) == 0


def test_exact_sign_against_rationals():
    """The exact comparison behind the choice, against rationals: random values,
    values spread over many binades, exact cancellations, and differences that
    binary64 sums in element order lose (so its answer is not a binary64 one)."""
    rng = np.random.default_rng(11)

    def want(w, v4, v6):
        d = exact_sq_err(w, v4) - exact_sq_err(w, v6)
        return (d > 0) - (d < 0)

    cases = []
    for _ in range(300):
        n = int(rng.integers(1, 17))
        w = rng.standard_normal(n) * 2.0 ** rng.integers(-60, 60, n)
        v4 = w + rng.standard_normal(n) * 2.0 ** rng.integers(-80, 0, n) * np.abs(w)
        v6 = w + rng.standard_normal(n) * 2.0 ** rng.integers(-80, 0, n) * np.abs(w)
        cases.append((w, v4, v6))
        cases.append((w, v4, v4.copy()))                      # equal errors: 0
        cases.append((w, v4, 2 * w - v4))                     # mirrored: 0
    # binary64 element-order sums give equal errors here, the exact ones differ by 2^-80
    one = np.array([1.0, 2.0 ** -40])
    cases.append((one, np.array([0.0, 0.0]), np.array([0.0, 2.0 ** -40])))       # e4 > e6: +1
    cases.append((one, np.array([0.0, 2.0 ** -40]), np.array([0.0, 0.0])))       # e4 < e6: -1
    # w - v inexact in binary64 (1 - 2^-60): its square's cross term 2*dh*dl and low
    # term dl^2 decide these signs; the other elements have w = 0 and exact squares
    z = 2.0 ** -30
    w = np.array([1.0, 0.0, 0.0, 0.0])
    cases.append((w, np.array([2.0 ** -60, z, z, 0.0]), np.array([0.0, 0.0, 0.0, 2.0 ** -60])))     # 0
    cases.append((w, np.array([2.0 ** -60, z, z, 0.0]), np.array([0.0, 0.0, 0.0, 2.0 ** -61])))     # +1
    cases.append((w, np.array([2.0 ** -60, z, z, 2.0 ** -80]), np.array([0.0, 0.0, 0.0, 2.0 ** -60])))  # +1
    cases.append((w, np.array([2.0 ** -60, z, z, 0.0]), np.array([0.0, 0.0, 2.0 ** -90, 2.0 ** -60])))  # -1
    # random values whose difference from w spans many binades (inexact differences)
    for _ in range(200):
        n = int(rng.integers(1, 17))
        w = rng.standard_normal(n) * 2.0 ** rng.integers(-20, 20, n)
        v4 = rng.standard_normal(n) * np.abs(w) * 2.0 ** rng.integers(-70, -20, n)
        v6 = rng.standard_normal(n) * np.abs(w) * 2.0 ** rng.integers(-70, -20, n)
        cases.append((w, v4, v6))
    tricky = 0
    for w, v4, v6 in cases:
        got = oracle.f46_exact_sign(w, v4, v6)
        assert got == want(w, v4, v6), (w, v4, v6)
        f64 = float(np.sum((w - v4) ** 2)) - float(np.sum((w - v6) ** 2))
        tricky += (f64 > 0) - (f64 < 0) != got
    assert tricky >= 2, "the cases must include differences binary64 sums miss"


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
