"""The m = 1, q -> +inf reduction to plain NVFP4 round-to-nearest, and brute force.

Model card "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct", section
"Perplexity": the NVFP4 row is round-to-nearest NVFP4 weights.  With m = 1 the
block scale is e4m3(clamp(max|w|/(6*s2))) and with sigmoid(q) = 1 (binary32
sigmoid(30) is exactly 1) every element is quantized with D = S_b*s2: that is
plain RTN.  The RTN below is written independently, in numpy binary32 with
ml_dtypes' E4M3 and E2M1 casts.
"""
import ml_dtypes
import numpy as np
import torch

import oracle
from tests.test_oracle_codecs import argmin_e2m1

F = np.float32


def rtn_nvfp4(Wf: np.ndarray, s2: np.float32):
    out, inn = Wf.shape
    b = Wf.reshape(-1, 16)
    A = np.abs(b).max(1)
    x = A / (F(6) * s2)
    x = np.where(x == 0, F(1), x)
    x = np.clip(x, F(2.0 ** -6), F(448)).astype(F)
    sb = x.astype(ml_dtypes.float8_e4m3fn)
    S = sb.astype(F)
    D = S * s2
    y = b / D[:, None]
    c8 = np.clip(y, F(-6), F(6)).astype(ml_dtypes.float4_e2m1fn)
    c = c8.astype(F)
    wq = (c * S[:, None]) * s2
    wq16 = torch.from_numpy(wq.astype(F)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return (sb.view(np.uint8).reshape(out, inn // 16), (c8.view(np.uint8) & 0xF).reshape(out, inn),
            wq16.reshape(out, inn))


def _weights(out, inn, seed):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(out, inn, generator=g) * 0.02).to(torch.bfloat16)
    idx = torch.randint(0, out * inn, (out * inn // 500,), generator=g)
    W.view(-1)[idx] = (W.view(-1)[idx].float() * 20).to(torch.bfloat16)
    W[0, :16] = 0  # one zero block
    return W.view(torch.int16).numpy().view(np.uint16), W.float().numpy()


def test_rtn_reduction_bit_exact():
    Wb, Wf = _weights(96, 256, 0)
    s2 = oracle.s2(Wb)
    m = np.ones((96, 16), F)
    q = np.full((96, 32), 30.0, F)
    f = oracle.fwd(Wb, m, q, s2)
    sb, codes, wq = rtn_nvfp4(Wf, s2)
    np.testing.assert_array_equal(f.scales, sb)
    np.testing.assert_array_equal(f.codes, codes)
    np.testing.assert_array_equal(f.Wq, wq)


def test_large_finite_logit_is_rtn_too():
    # sigmoid(q) rounds to 1.0f from q = 17.5 on; then the result is RTN as well
    Wb, Wf = _weights(32, 128, 1)
    s2 = oracle.s2(Wb)
    f = oracle.fwd(Wb, np.ones((32, 8), F), np.full((32, 16), 17.5, F), s2)
    _, codes, wq = rtn_nvfp4(Wf, s2)
    np.testing.assert_array_equal(f.codes, codes)
    np.testing.assert_array_equal(f.Wq, wq)


GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
MIDS = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]


def test_brute_force_every_position_and_value():
    """Block with S = 64, s2 = 2^-12, q = (0, 30): D = 2^-7 in sub-block 0 and
    2^-6 in sub-block 1.  Every value v of the E2M1 grid, every midpoint and
    values beyond 6, both signs, at every position: w = v * D_k must give
    argmin(v).  A wrong sub-block index would use the other D (a factor 2)."""
    vals = GRID + MIDS + [7.0, 12.0]
    vals = vals + [-v for v in vals]
    rows, want = [], []
    for pos in range(16):
        for v in vals:
            k = pos // 8
            D = 2.0 ** -7 if k == 0 else 2.0 ** -6
            w = np.zeros(16, F)
            mx = 15 if pos != 15 else 0
            w[mx] = 0.09375
            w[pos] = v * D
            if abs(w[pos]) > 0.09375:      # keep the block max (and S = 64) fixed
                continue
            rows.append(w)
            exp = [argmin_e2m1(float(w[i] / (2.0 ** -7 if i < 8 else 2.0 ** -6))) for i in range(16)]
            want.append(exp)
    Wf = np.array(rows, F)
    Wb = (Wf.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((Wb.astype(np.uint32) << 16).view(F), Wf)
    n = len(rows)
    m = np.ones((n, 1), F)
    q = np.tile(np.array([0.0, 30.0], F), (n, 1))
    f = oracle.fwd(Wb, m, q, F(2.0 ** -12))
    assert np.all(f.scales == 0x68)
    np.testing.assert_array_equal(f.codes, np.array(want, np.uint8))
