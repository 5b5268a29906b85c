"""The oracle on the hand-derived worked example and on the special cases.

The fixture tests/golden/worked_block.json states its derivation from the
equations of the model card "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct",
section "What this is"; every value there is an exact dyadic rational.
"""
import json
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def bf16_bits(x):
    x = np.asarray(x, np.float32)
    b = (x.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((b.astype(np.uint32) << 16).view(np.float32), x), "not exact in bf16"
    return b


def round_bf16(x):
    """Values rounded to bf16 (torch's cast), as float32."""
    import torch
    t = torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).float()
    return list(t.numpy())


def f32_of_bits(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


@pytest.fixture(scope="module")
def golden():
    with open(os.path.join(HERE, "golden", "worked_block.json")) as f:
        return json.load(f)


def test_worked_example_forward(golden):
    W = bf16_bits(golden["W"])
    m = np.array(golden["m"], np.float32)
    q = np.array(golden["q"], np.float32)
    ex = golden["expected"]
    s2 = oracle.s2(W)
    assert s2 == np.float32(ex["s2"])
    f = oracle.fwd(W, m, q, s2)
    np.testing.assert_array_equal(f.scales, np.array(ex["scales"], np.uint8))
    np.testing.assert_array_equal(f.codes, np.array(ex["codes"], np.uint8))
    np.testing.assert_array_equal(f.Wq, bf16_bits(ex["Wq"]))
    for r, c in ex["negative_zero_Wq"]:
        assert f.Wq[r, c] == 0x8000
    assert f.stats == ex["stats"]
    codes, scales, ts = oracle.pack(W, m, q, s2)
    np.testing.assert_array_equal(scales, f.scales)
    np.testing.assert_array_equal(codes, (f.codes[:, 0::2] | (f.codes[:, 1::2] << 4)).astype(np.uint8))
    assert ts == s2


def test_worked_example_gradients(golden):
    W = bf16_bits(golden["W"])
    m = np.array(golden["m"], np.float32)
    q = np.array(golden["q"], np.float32)
    g = bf16_bits(np.ones(W.shape, np.float32))
    ex = golden["expected"]
    s2 = oracle.s2(W)
    dm, dq = oracle.ste_bwd(W, g, m, q, s2)
    np.testing.assert_array_equal(dm, np.array(ex["dm"], np.float32))
    np.testing.assert_array_equal(dq, np.array(ex["dq"], np.float32))
    # accumulate adds
    dm2, dq2 = oracle.ste_bwd(W, g, m, q, s2, dm=dm.copy(), dq=dq.copy())
    np.testing.assert_array_equal(dm2, 2 * dm)
    np.testing.assert_array_equal(dq2, 2 * dq)


def _one_block(w, m_b=1.0, q2=(6.0, 6.0), s2=2.0 ** -12):
    W = bf16_bits(np.array([w], np.float32))
    return W, np.array([[m_b]], np.float32), np.array([q2], np.float32), np.float32(s2)


def test_all_zero_block():
    W, m, q, s2 = _one_block([0.0] * 16)
    f = oracle.fwd(W, m, q, s2)
    assert f.scales[0, 0] == 0x38  # scale 1
    assert not f.codes.any() and not f.Wq.any()
    dm, dq = oracle.ste_bwd(W, bf16_bits(np.ones((1, 16))), m, q, s2)
    assert dm[0, 0] == 0 and not dq.any()
    assert f.stats["zero_blocks"] == 1


def test_zero_factor_gives_scale_one_and_no_m_gradient():
    w = [0.01 * (i - 7) for i in range(16)]
    w = round_bf16(w)
    W, m, q, s2 = _one_block(w, m_b=0.0)
    f = oracle.fwd(W, m, q, s2)
    assert f.scales[0, 0] == 0x38
    dm, _ = oracle.ste_bwd(W, bf16_bits(np.ones((1, 16))), m, q, s2)
    assert dm[0, 0] == 0.0


def test_low_and_high_clamp():
    w = round_bf16([0.001 * (i + 1) for i in range(16)])
    # A_b = 0.016: x = 0.016*m/(6*2^-12) = 10.92*m
    W, m, q, s2 = _one_block(w, m_b=1e-4)
    f = oracle.fwd(W, m, q, s2)
    assert f.scales[0, 0] == 0x08 and f.stats["clamp_low"] == 1
    dm, _ = oracle.ste_bwd(W, bf16_bits(np.ones((1, 16))), m, q, s2)
    assert dm[0, 0] == 0.0
    W, m, q, s2 = _one_block(w, m_b=100.0)
    f = oracle.fwd(W, m, q, s2)
    assert f.scales[0, 0] == 0x7E and f.stats["clamp_high"] == 1
    dm, _ = oracle.ste_bwd(W, bf16_bits(np.ones((1, 16))), m, q, s2)
    assert dm[0, 0] == 0.0
    # a negative factor clamps to 2^-6 and blocks the gradient
    W, m, q, s2 = _one_block(w, m_b=-1.0)
    f = oracle.fwd(W, m, q, s2)
    assert f.scales[0, 0] == 0x08


def test_very_negative_logit_saturates():
    rng = np.random.default_rng(0)
    w = round_bf16(rng.normal(0, 0.02, 16))
    W, m, q, s2 = _one_block(w, q2=(-8.0, -8.0), s2=np.float32(0.02 * 4 / 2688))
    f = oracle.fwd(W, m, q, s2)
    # sigma(-8) ~ 3.35e-4: |y| ~ 6*|w|/(A_b*3.35e-4) > 6 for all but tiny elements
    big = np.abs(np.array(w)) > np.abs(np.array(w)).max() * 0.01
    assert np.all((f.codes[0][big] & 7) == 7)


def test_rejects_bad_arguments():
    W, m, q, s2 = _one_block([0.0] * 16)
    with pytest.raises(oracle.OracleError):
        oracle.fwd(W, m, q, np.float32(0.0))
    with pytest.raises(oracle.OracleError):
        oracle.fwd(W, m, q, np.float32(np.inf))
    Wn = W.copy(); Wn[0, 3] = 0x7FC0
    with pytest.raises(oracle.OracleError):
        oracle.fwd(Wn, m, q, s2)
    with pytest.raises(oracle.OracleError):
        oracle.s2(Wn)


# (A_b, m_b) pairs, s2 = 2^-12, for which fl(fl(A*m)/fl(6*s2)) and fl(fl(A/fl(6*s2))*m)
# fall on different sides of an E4M3 midpoint: the scale pins the evaluation order
# max|w_b| * m_b / (6 * s2), left to right, as the S_b equation is written.
ORDER_CASES = [(0.3203125, 0.014291158877313137), (0.306640625, 1.605095624923706),
               (0.15625, 0.01992187649011612), (0.1611328125, 0.03068181686103344),
               (0.1669921875, 0.050438594073057175), (0.30078125, 0.014001622796058655)]


def test_scale_uses_left_to_right_order():
    import ml_dtypes
    F = np.float32
    s2 = F(2.0 ** -12)
    W = np.zeros((len(ORDER_CASES), 16), np.float32)
    m = np.zeros((len(ORDER_CASES), 1), np.float32)
    for r, (A, mb) in enumerate(ORDER_CASES):
        W[r, 5] = A
        m[r, 0] = mb
    f = oracle.fwd(bf16_bits(W), m, np.zeros((len(ORDER_CASES), 2), F), s2)
    for r, (A, mb) in enumerate(ORDER_CASES):
        x = F(F(A) * F(mb)) / (F(6) * s2)
        other = F(F(A) / (F(6) * s2)) * F(mb)
        want = np.array([x], F).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)[0]
        alt = np.array([other], F).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)[0]
        assert want != alt
        assert f.scales[r, 0] == want
