"""The straight-through gradients against central finite differences.

"Technische Samenvatting: FOCUS ...", section "Methodologie", item 1: the
scales are learned through the straight-through estimator.  The surrogate
below replaces each rounding R(z) -- the E2M1 code and the E4M3 block scale --
by R(z0) + (z - z0), z0 being its value at the evaluation point (rounding
passed straight through), keeps the clamps, and is evaluated in binary64,
written here independently of the oracle.  Its central differences in m and q
must match the oracle's closed form.  Blocks are drawn so that no step crosses
a clamp edge or a rounding boundary.
"""
import math

import ml_dtypes
import numpy as np

import oracle

F = np.float32


def sig(q):
    return 1.0 / (1.0 + math.exp(-q))


def surrogate(w, g, m, q, s2, frozen):
    A = float(np.max(np.abs(w)))
    x = A * m / (6.0 * s2)
    xc = min(max(x, 2.0 ** -6), 448.0)
    S = frozen["S0"] + (xc - frozen["xc0"])
    L = 0.0
    for k in range(2):
        D = S * sig(q[k]) * s2
        for j in range(8):
            i = 8 * k + j
            u = min(max(w[i] / D, -6.0), 6.0)
            c = frozen["c0"][i] + (u - frozen["u0"][i])
            L += g[i] * c * S * s2
    return L


def freeze(w, m, q, s2):
    A = float(np.max(np.abs(w)))
    xc0 = min(max(A * m / (6.0 * s2), 2.0 ** -6), 448.0)
    S0 = float(np.float32(xc0).astype(ml_dtypes.float8_e4m3fn).astype(np.float64))
    u0, c0 = [], []
    for i in range(16):
        D = S0 * sig(q[i // 8]) * s2
        u = min(max(w[i] / D, -6.0), 6.0)
        u0.append(u)
        c0.append(float(np.float32(u).astype(ml_dtypes.float4_e2m1fn).astype(np.float64)))
    return {"S0": S0, "xc0": xc0, "u0": u0, "c0": c0}


def near_edge(w, m, q, s2, rel=2e-3):
    A = float(np.max(np.abs(w)))
    x = A * m / (6.0 * s2)
    if abs(x - 2.0 ** -6) < rel * x or abs(x - 448.0) < rel * x or x < 2.0 ** -6 or x > 448:
        return True
    S0 = float(np.float32(x).astype(ml_dtypes.float8_e4m3fn).astype(np.float64))
    for i in range(16):
        y = abs(w[i] / (S0 * sig(q[i // 8]) * s2))
        for e in (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0):
            if abs(y - e) < rel * e + 1e-9:
                return True
    return False


def test_ste_matches_finite_differences():
    rng = np.random.default_rng(2024)
    s2 = float(F(0.08 / 2688))
    rows_w, rows_g, rows_m, rows_q = [], [], [], []
    while len(rows_w) < 300:
        w = rng.normal(0, 0.02, 16).astype(F)
        w = (w.view(np.uint32) & 0xFFFF0000).view(F)        # bf16-exact values
        g = rng.normal(0, 1e-3, 16).astype(F)
        g = (g.view(np.uint32) & 0xFFFF0000).view(F)
        m = float(F(rng.uniform(0.3, 3.0)))
        q = [float(F(v)) for v in rng.normal(0.0, 3.0, 2)]
        if near_edge(w.astype(np.float64), m, q, s2):
            continue
        rows_w.append(w); rows_g.append(g); rows_m.append(m); rows_q.append(q)
    Wf = np.array(rows_w); Gf = np.array(rows_g)
    Wb = (Wf.view(np.uint32) >> 16).astype(np.uint16)
    Gb = (Gf.view(np.uint32) >> 16).astype(np.uint16)
    m = np.array(rows_m, F).reshape(-1, 1)
    q = np.array(rows_q, F)
    dm, dq = oracle.ste_bwd(Wb, Gb, m, q, F(s2))
    n_out = 0
    for r in range(len(rows_w)):
        w = Wf[r].astype(np.float64); g = Gf[r].astype(np.float64)
        mm = float(m[r, 0]); qq = [float(q[r, 0]), float(q[r, 1])]
        fr = freeze(w, mm, qq, s2)
        h = 1e-4 * mm
        fd_m = (surrogate(w, g, mm + h, qq, s2, fr) - surrogate(w, g, mm - h, qq, s2, fr)) / (2 * h)
        A = float(np.max(np.abs(w)))
        scale_m = A / 6 * float(np.sum(np.abs(g))) * 12.0     # bound of sum |g| * (|c| + |y|)
        assert abs(fd_m - float(dm[r, 0])) <= 1e-6 * scale_m + 1e-15, (r, fd_m, dm[r, 0])
        for k in range(2):
            hq = 1e-4
            qp = list(qq); qm = list(qq)
            qp[k] += hq; qm[k] -= hq
            fd_q = (surrogate(w, g, mm, qp, s2, fr) - surrogate(w, g, mm, qm, s2, fr)) / (2 * hq)
            ys = np.abs(w[8 * k:8 * k + 8]) / (fr["S0"] * sig(qq[k]) * s2)
            n_out += int(np.sum(ys > 6))
            scale_q = (1 - sig(qq[k])) * fr["S0"] * s2 * float(np.sum(np.abs(g[8 * k:8 * k + 8]) * np.minimum(ys, 6)))
            # the closed form uses 1 - sigma with sigma the forward's binary32 value: its
            # rounding (half an ulp of sigma) is a relative error of 2^-25/(1 - sigma)
            sig_err = 2.0 ** -25 * max(sig(qq[k]), 0.5) / (1 - sig(qq[k]))
            assert abs(fd_q - float(dq[r, k])) <= (1e-6 + sig_err) * scale_q + 1e-15, (r, k, fd_q, dq[r, k])
    assert n_out > 100   # the clamp gating was exercised


def test_surrogate_at_point_equals_forward():
    rng = np.random.default_rng(7)
    w = (rng.normal(0, 0.02, 16).astype(F).view(np.uint32) & 0xFFFF0000).view(F)
    s2 = float(F(0.08 / 2688))
    m, q = 1.1, [0.5, -1.0]
    fr = freeze(w.astype(np.float64), m, q, s2)
    f = oracle.fwd((w.view(np.uint32) >> 16).astype(np.uint16).reshape(1, 16), np.array([[m]], F),
                   np.array([q], F), F(s2))
    wq = ((f.Wq.astype(np.uint32) << 16).view(F)).astype(np.float64)[0]
    for i in range(16):
        c = fr["c0"][i]
        assert abs(c * fr["S0"] * s2 - wq[i]) <= 2 ** -8 * abs(wq[i]) + 1e-30
