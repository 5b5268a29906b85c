"""Pins of the oracle's MXFP4 variant (32-element blocks, E8M0 block scale,
four sub-blocks of 8; no tensor scale).

Sources: "Technische Samenvatting: FOCUS ...", sections "Probleemstelling"
and "Methodologie" items 2-3 (MXFP4 blocks of 32 with an E8M0 scale;
sub-blocks of 8 with their own coefficient); the block scale follows the OCP
Microscaling rule 2^(floor(log2 max) - 2) applied to the scaled maximum.
Pinned by: the m = 1, sigmoid = 1 reduction to plain MXFP4 round to nearest
written independently (numpy frexp and ml_dtypes' E2M1 cast); a hand-derived
block (floor rule, the clip above 6, ties, signed zero, the exponent clamp,
gradients); central finite differences of the straight-through surrogate;
and every E2M1 value at every position of the four sub-blocks.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

F = np.float32


def bits(Wf):
    Wf = np.asarray(Wf, F)
    Wb = (Wf.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((Wb.astype(np.uint32) << 16).view(F), Wf), "values must be exact in bf16"
    return Wb


def mx_rtn(Wf):
    """Plain MXFP4 round to nearest: per 32 values X = 2^(floor(log2 max) - 2)."""
    out, inn = Wf.shape
    b = Wf.reshape(-1, 32)
    A = np.abs(b).max(1)
    _, e = np.frexp(A)                     # A = f * 2^e, f in [0.5, 1)
    X = np.where(A == 0, F(1), np.ldexp(F(1), np.clip(e - 1 - 2, -127, 127))).astype(F)
    y = b / X[:, None]
    c8 = np.clip(y, F(-6), F(6)).astype(ml_dtypes.float4_e2m1fn)
    wq = c8.astype(F) * X[:, None]
    sb = np.where(A == 0, 127, np.clip(e - 3, -127, 127) + 127).astype(np.uint8)
    wq16 = torch.from_numpy(wq.astype(F)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return sb.reshape(out, inn // 32), (c8.view(np.uint8) & 0xF).reshape(out, inn), wq16.reshape(out, inn)


def test_mx_reduces_to_plain_mxfp4_rtn():
    g = torch.Generator().manual_seed(5)
    W = (torch.randn(64, 512, generator=g) * 0.02).to(torch.bfloat16)
    W[0, :32] = 0
    W[1, 32:64] *= 1e-30                               # tiny block: exponent near the clamp
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    f = oracle.mx_fwd(Wb, np.ones((64, 16), F), np.full((64, 64), 30.0, F))
    sb, codes, wq = mx_rtn(W.float().numpy())
    np.testing.assert_array_equal(f.scales, sb)
    np.testing.assert_array_equal(f.codes, codes)
    np.testing.assert_array_equal(f.Wq, wq)


def test_mx_worked_blocks():
    # row 0 block 0: m = 1, q = [30, 0, 30, 30]; row 0 block 1: m = 2, q = 30;
    # row 1 block 0: zeros; row 1 block 1: one value 2^-120 with m = 2^-10 (x = 2^-130, clamped).
    W = np.zeros((2, 64))
    W[0, :11] = [0.9375, 0.75, 0.0625, 0.03125, 0.09375, -0.3125, -0.0, 0.5, 0.0625, -0.1875, 0.40625]
    W[0, 32] = 0.9375
    W[1, 32] = 2.0 ** -120
    m = np.array([[1.0, 2.0], [1.0, 2.0 ** -10]], F)
    q = np.full((2, 8), 30.0, F)
    q[0, 1] = 0.0
    Wb = bits(W)
    f = oracle.mx_fwd(Wb, m, q)
    # S: floor(log2 0.9375) = -1 -> 2^-3 (E8M0 124); floor(log2 1.875) = 0 -> 2^-2 (125);
    # zero block -> 1 (127); floor(log2 2^-130) - 2 = -132 clamps to -127 (byte 0)
    np.testing.assert_array_equal(f.scales, np.array([[124, 125], [127, 0]], np.uint8))
    # y (sub-block 0, D = 1/8): 7.5 (clipped to 6), 6, 0.5, 0.25 (tie -> 0), 0.75 (tie -> 1),
    # -2.5 (tie -> -2), -0 (code 8), 4; sub-block 1 (D = 1/16): 1, -3, 6.5 (clipped)
    want0 = [7, 7, 1, 0, 2, 12, 8, 6, 2, 13, 7] + [0] * 21 + [6] + [0] * 31
    np.testing.assert_array_equal(f.codes[0], np.array(want0, np.uint8))
    assert f.codes[1, 32] == 7 and not f.codes[1, :32].any()
    wq = (f.Wq.astype(np.uint32) << 16).view(F)
    np.testing.assert_array_equal(wq[0, :11], np.array([0.75, 0.75, 0.0625, 0, 0.125, -0.25, -0.0, 0.5, 0.125,
                                                         -0.375, 0.75], F))
    assert f.Wq[0, 6] == 0x8000 and wq[0, 32] == 1.0 and wq[1, 32] == F(6 * 2.0 ** -127)
    # gradients with dL/dw' = 1: dm = (A/4) sum(in ? c - y : c), dq_k = -(1 - sigma_k) S sum(in y)
    dm, dq = oracle.mx_ste_bwd(Wb, bits(np.ones((2, 64))), m, q)
    np.testing.assert_array_equal(dm, np.array([[0.234375 * 12.5, 0.234375 * 0.25], [0, 0]], F))
    want_dq = np.zeros((2, 8), F)
    want_dq[0, 1] = 0.125                     # -(0.5)(1/8)(1 - 3)
    np.testing.assert_array_equal(dq, want_dq)


def sig(v):
    return 1.0 / (1.0 + math.exp(-v))


def surrogate(w, g, m, q, fr):
    A = float(np.max(np.abs(w)))
    z = A * m / 4.0
    S = fr["S0"] + (z - fr["z0"])
    L = 0.0
    for k in range(4):
        D = S * sig(q[k])
        for j in range(8):
            i = 8 * k + j
            u = min(max(w[i] / D, -6.0), 6.0)
            L += g[i] * (fr["c0"][i] + (u - fr["u0"][i])) * S
    return L


def freeze(w, m, q):
    A = float(np.max(np.abs(w)))
    z0 = A * m / 4.0
    S0 = 2.0 ** math.floor(math.log2(A * m) - 2)
    u0, c0 = [], []
    for i in range(32):
        u = min(max(w[i] / (S0 * sig(q[i // 8])), -6.0), 6.0)
        u0.append(u)
        c0.append(float(np.float32(u).astype(ml_dtypes.float4_e2m1fn).astype(np.float64)))
    return {"S0": S0, "z0": z0, "u0": u0, "c0": c0}


def near_edge(w, m, q, rel=2e-3):
    A = float(np.max(np.abs(w)))
    lg = math.log2(A * m)
    if abs(lg - round(lg)) < 3e-3:
        return True
    S0 = 2.0 ** math.floor(lg - 2)
    for i in range(32):
        y = abs(w[i] / (S0 * sig(q[i // 8])))
        if any(abs(y - e) < rel * e for e in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0)):
            return True
    return False


def test_mx_ste_matches_finite_differences():
    rng = np.random.default_rng(77)
    rows = []
    while len(rows) < 200:
        w = (rng.normal(0, 0.02, 32).astype(F).view(np.uint32) & 0xFFFF0000).view(F)
        gg = (rng.normal(0, 1e-3, 32).astype(F).view(np.uint32) & 0xFFFF0000).view(F)
        m = float(F(rng.uniform(0.3, 3.0)))
        q = [float(F(v)) for v in rng.normal(0.0, 3.0, 4)]
        if not near_edge(w.astype(np.float64), m, q):
            rows.append((w, gg, m, q))
    Wf = np.array([r[0] for r in rows]); Gf = np.array([r[1] for r in rows])
    m = np.array([r[2] for r in rows], F).reshape(-1, 1)
    q = np.array([r[3] for r in rows], F)
    dm, dq = oracle.mx_ste_bwd(bits(Wf), bits(Gf), m, q)
    n_out = 0
    for r, (w, gg, mm, qq) in enumerate(rows):
        w = w.astype(np.float64); gg = gg.astype(np.float64)
        fr = freeze(w, mm, qq)
        h = 1e-4 * mm
        fd_m = (surrogate(w, gg, mm + h, qq, fr) - surrogate(w, gg, mm - h, qq, fr)) / (2 * h)
        scale_m = float(np.max(np.abs(w))) / 4 * float(np.sum(np.abs(gg))) * 12.0
        assert abs(fd_m - float(dm[r, 0])) <= 1e-6 * scale_m + 1e-15, (r, fd_m, dm[r, 0])
        for k in range(4):
            qp, qm = list(qq), list(qq)
            qp[k] += 1e-4; qm[k] -= 1e-4
            fd_q = (surrogate(w, gg, mm, qp, fr) - surrogate(w, gg, mm, qm, fr)) / 2e-4
            ys = np.abs(w[8 * k:8 * k + 8]) / (fr["S0"] * sig(qq[k]))
            n_out += int(np.sum(ys > 6))
            scale_q = (1 - sig(qq[k])) * fr["S0"] * float(np.sum(np.abs(gg[8 * k:8 * k + 8]) * np.minimum(ys, 6)))
            sig_err = 2.0 ** -25 * max(sig(qq[k]), 0.5) / (1 - sig(qq[k]))
            assert abs(fd_q - float(dq[r, k])) <= (1e-6 + sig_err) * scale_q + 1e-15, (r, k, fd_q, dq[r, k])
    assert n_out > 50


GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
MIDS = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]


def argmin_e2m1(u):
    a = min(abs(u), 6.0)
    best = min(range(8), key=lambda c: (abs(GRID[c] - a), c % 2))
    return best | (8 if math.copysign(1.0, u) < 0 else 0)


def test_mx_every_value_at_every_position():
    """Block max 0.75 (S = 2^-3) fixed in element 31 (or 0); q = (30, 0, 30, 0):
    D = 2^-3, 2^-4, 2^-3, 2^-4 by sub-block.  A wrong sub-block index uses the
    other D (a factor 2)."""
    D = [2.0 ** -3, 2.0 ** -4, 2.0 ** -3, 2.0 ** -4]
    vals = GRID + MIDS + [7.0]
    vals = vals + [-v for v in vals]
    rows, want = [], []
    for pos in range(32):
        for v in vals:
            w = np.zeros(32)
            mx = 31 if pos != 31 else 0
            w[mx] = 0.75
            w[pos] = v * D[pos // 8]
            if abs(w[pos]) > 0.75:
                continue
            rows.append(w)
            want.append([argmin_e2m1(w[i] / D[i // 8]) for i in range(32)])
    n = len(rows)
    f = oracle.mx_fwd(bits(np.array(rows)), np.ones((n, 1), F), np.tile(np.array([30, 0, 30, 0], F), (n, 1)))
    assert np.all(f.scales == 124)
    np.testing.assert_array_equal(f.codes, np.array(want, np.uint8))


def test_mx_shape_rule():
    with pytest.raises(oracle.OracleError):
        oracle.mx_fwd(np.zeros((2, 48), np.uint16), np.ones((2, 1), F), np.zeros((2, 6), F))
