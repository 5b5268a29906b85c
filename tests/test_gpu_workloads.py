"""GPU parity at the five workloads' sizes (seeded synthetic inputs, synth/).

* C1: W[2048, 2048], forward + NVFP4 pack through the single-tensor calls: full
  parity.
* C4: the stress tensor W[8192, 8192] (Student-t, planted zero, tie and clamp
  blocks): forward, pack and straight-through backward, full parity, and the
  counts of the planted cases.
* C2: all 112 Llama-3.2-1B linears, one fused step as one multi-tensor launch
  (step 1 with zero AdamW moments, and step 5 with warm ones):
  full parity of W', gradients, m, q and moments.
* C3: all 224 Llama-3.1-8B linears in exactly the launch configuration the
  benchmark times (the fused step with W', the export of the updated
  parameters and the tensor maxima, then s2 from those maxima): full parity on
  one tensor of each shape, a 1/64 row sample of every other tensor, every
  tensor's maximum and its s2 after the step.
* C5: Llama-3.1-70B layers 0, 40 and 79, one layer at a time: a 1/256 row
  sample.
* A single tensor of more than 2^31 weights (byte offsets past 2^32): s2,
  forward, pack and the fused step, s2 in full and rows at both ends and the
  middle against the oracle.

The export of the updated parameters is compared with the oracle's pack of the
oracle's own updated m and q.  The two updates agree within the tolerance, not
bit for bit, so a scale byte may differ only where the updated x_b lies within
2^-20 relative of an E4M3 rounding boundary, and a code only where y does
(the oracle's band flag); the elements such mismatches cover are held at or
below 1e-6 of the elements checked over each workload.  Every test records its
counts (tests/parity.py), printed at the end of the run.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity import (MAX_MISMATCH_FRAC, assert_close, block_mask, check_forward, forward_counts, host,
                          host_bits, record, unpack_codes)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    from fp4_post_weight_b200 import focus
    return focus


def _e4m3_midpoints():
    vals = []
    for b in range(0x08, 0x7E):
        e, mn = (b >> 3) & 15, b & 7
        v = (1 + mn / 8) * 2.0 ** (e - 7)
        e2, mn2 = (e, mn + 1) if mn < 7 else (e + 1, 0)
        vals.append((v + (1 + mn2 / 8) * 2.0 ** (e2 - 7)) / 2)
    return np.array(vals)


MIDS = _e4m3_midpoints()
BAND = 2.0 ** -20


def _near_e4m3_boundary(x):
    """x (float64 array of scaled maxima) within 2^-20 relative of an E4M3 rounding
    boundary or of a clamp edge."""
    x = np.asarray(x, np.float64)
    edges = np.concatenate([MIDS, [2.0 ** -6, 448.0]])
    j = np.clip(np.searchsorted(edges, x), 1, len(edges) - 1)
    d = np.minimum(np.abs(x - edges[j - 1]), np.abs(x - edges[j]))
    return d <= BAND * np.abs(x)


def check_export(Wb, m_new, q_new, s2, codes_gpu_packed, scales_gpu):
    """The export of the updated parameters against the oracle's pack of the
    oracle's own updated m and q.  The two updates agree within the tolerance,
    not bit for bit, so a scale byte may differ only where the updated x_b lies
    within 2^-20 relative of an E4M3 rounding boundary, and a code only where y
    does (the oracle's band flag).  Returns (scale mismatches, code mismatches
    outside those blocks, elements); the caller holds the elements they cover
    at or below 1e-6 of all the elements it checked."""
    ref = oracle.fwd(Wb, m_new, q_new, s2, want_y=False)
    A = (np.abs(Wb.view(np.int16).astype(np.int32)) & 0x7FFF)      # bf16 magnitude bits
    A = (A.astype(np.uint32) << 16).view(np.float32).reshape(Wb.shape[0], -1, 16).max(-1)
    x = (A.astype(np.float32) * m_new) / (np.float32(6) * np.float32(s2))
    sc_bad = scales_gpu != ref.scales
    if sc_bad.any():
        assert np.all(_near_e4m3_boundary(x[sc_bad])), "scale mismatch away from an E4M3 boundary"
    codes = unpack_codes(codes_gpu_packed)
    cbad = (codes != ref.codes) & ~np.repeat(sc_bad, 16, axis=1)
    if cbad.any():
        assert np.all(ref.band[cbad] == 1), "export code mismatch outside the 2^-20 band"
    return int(sc_bad.sum()), int(cbad.sum()), codes.size


# ---------------------------------------------------------------------------

def test_c1_single_2048_forward_and_pack(F):
    t = synth.single_2048("cuda")
    o, i = t.W.shape
    ws = torch.empty(F.focus_s2_workspace_bytes(o, i), dtype=torch.uint8, device="cuda")
    s2d = torch.zeros(1, device="cuda")
    F.focus_s2(t.W, s2d, ws)
    s2 = float(host(s2d)[0])
    Wq = torch.empty_like(t.W)
    F.focus_fwd(t.W, t.m, t.q, s2, Wq)
    codes = torch.empty((o, i // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((o, i // 16), dtype=torch.uint8, device="cuda")
    ts = torch.zeros(1, device="cuda")
    F.focus_pack_nvfp4(t.W, t.m, t.q, s2, codes, scales, ts)
    assert F.focus_get_error() == 0
    Wb = host_bits(t.W)
    assert oracle.s2(Wb) == np.float32(s2)
    ref = oracle.fwd(Wb, host(t.m), host(t.q), s2)
    mism = check_forward(ref, Wq=host_bits(Wq), codes=unpack_codes(host(codes)), scales=host(scales))
    rc, rs, rt = oracle.pack(Wb, host(t.m), host(t.q), s2)
    assert rt == host(ts)[0]
    record("C1 W[2048,2048] forward + pack, full", {**forward_counts(ref, mism), "scale_mismatch": 0})


def test_c4_stress_forward_backward(F):
    t, info = synth.stress(8192, 8192, "cuda")
    o, i = t.W.shape
    ws = torch.empty(F.focus_s2_workspace_bytes(o, i), dtype=torch.uint8, device="cuda")
    s2d = torch.zeros(1, device="cuda")
    F.focus_s2(t.W, s2d, ws)
    s2 = float(host(s2d)[0])
    assert s2 == info["s2"]                      # the construction makes s2 a power of two
    Wq = torch.empty_like(t.W)
    F.focus_fwd(t.W, t.m, t.q, s2, Wq)
    codes = torch.empty((o, i // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((o, i // 16), dtype=torch.uint8, device="cuda")
    F.focus_pack_nvfp4(t.W, t.m, t.q, s2, codes, scales, torch.zeros(1, device="cuda"))
    dm = torch.empty_like(t.m)
    dq = torch.empty_like(t.q)
    F.focus_ste_bwd(t.W, t.dWq, t.m, t.q, s2, dm, dq)
    assert F.focus_get_error() == 0
    Wb, Gb, m, q = host_bits(t.W), host_bits(t.dWq), host(t.m), host(t.q)
    ref = oracle.fwd(Wb, m, q, s2)
    mism = check_forward(ref, Wq=host_bits(Wq), codes=unpack_codes(host(codes)), scales=host(scales))
    skip = block_mask(mism)
    rdm, rdq = oracle.ste_bwd(Wb, Gb, m, q, s2)
    assert_close(host(dm), rdm, "dm", skip)
    assert_close(host(dq), rdq, "dq", np.repeat(skip, 2, axis=1))
    st = ref.stats
    nb = o * i // 16
    record("C4 stress W[8192,8192] forward + pack + backward, full", {**forward_counts(ref, mism), "scale_mismatch": 0})
    assert st["zero_blocks"] >= int(0.01 * nb)
    assert st["clamp_high"] >= 1000 and st["clamp_low"] >= 1000
    assert st["exact_ties"] >= 15 * int(0.01 * nb) // 2
    assert st["out_of_range"] > 0


def _table_entries(tensors, want_grad=True, export=False):
    from fp4_post_weight_b200.table import Entry
    ents = []
    for t in tensors:
        o, i = t.W.shape
        e = Entry(W=t.W, m=t.m, q=t.q, s2=torch.zeros(1, device="cuda"), dWq=t.dWq, Wq=torch.empty_like(t.W),
                  m_exp_avg=t.m_v1, m_exp_avg_sq=t.m_v2, q_exp_avg=t.q_v1, q_exp_avg_sq=t.q_v2)
        if want_grad:
            e.dm = torch.empty_like(t.m)
            e.dq = torch.empty_like(t.q)
        if export:
            e.codes = torch.empty((o, i // 2), dtype=torch.uint8, device="cuda")
            e.scales = torch.empty((o, i // 16), dtype=torch.uint8, device="cuda")
        ents.append(e)
    return ents


def _snapshot(t, rows=None):
    sel = (lambda x: x) if rows is None else (lambda x: x[rows])
    return [host_bits(sel(t.W)), host_bits(sel(t.dWq))] + [host(sel(x)).copy() for x in
                                                           (t.m, t.q, t.m_v1, t.m_v2, t.q_v1, t.q_v2)]


def _compare_step(e, snap, s2, step, rows=None, export=False):
    """One tensor (or its sampled rows) after the fused step against the oracle."""
    Wb, Gb, m, q, mv1, mv2, qv1, qv2 = snap
    sel = (lambda x: x) if rows is None else (lambda x: x[rows])
    ref_f = oracle.fwd(Wb, m, q, s2, want_y=False)
    mism = check_forward(ref_f, Wq=host_bits(sel(e.Wq)))
    skip = block_mask(mism)
    skq = np.repeat(skip, 2, axis=1)
    _, gm, gq = oracle.step(Wb, Gb, m, q, mv1, mv2, qv1, qv2, s2, step, want_wq=False)
    if e.dm is not None:
        assert_close(host(sel(e.dm)), gm, "dm", skip)
        assert_close(host(sel(e.dq)), gq, "dq", skq)
    assert_close(host(sel(e.m)), m, "m", skip)
    assert_close(host(sel(e.q)), q, "q", skq)
    assert_close(host(sel(e.m_exp_avg)), mv1, "m exp_avg", skip)
    assert_close(host(sel(e.m_exp_avg_sq)), mv2, "m exp_avg_sq", skip)
    assert_close(host(sel(e.q_exp_avg)), qv1, "q exp_avg", skq)
    assert_close(host(sel(e.q_exp_avg_sq)), qv2, "q exp_avg_sq", skq)
    out = forward_counts(ref_f, mism)
    if export:
        sb, cb, n = check_export(Wb, m, q, s2, host(sel(e.codes)), host(sel(e.scales)))
        out.update(export_scale_mismatch=sb, export_code_mismatch=cb, export_elements=n)
    return out


@pytest.mark.parametrize("step,warm", [(1, False), (5, True)])
def test_c2_llama_1b_fused_step_full(F, step, warm):
    """All 112 Llama-3.2-1B linears in one fused step: at step 1 with zero AdamW
    moments, and at step 5 with warm ones (random, non-negative second moments)."""
    from fp4_post_weight_b200.table import FocusTable, hparams
    tensors = []
    g = torch.Generator(device="cuda").manual_seed(77)
    for j, (_, sh) in enumerate(synth.LLAMA_1B.tensors()):
        t = synth.llama_1b_tensor(j, sh, "cuda")
        synth.adam_states(t, g, warm=warm)
        tensors.append(t)
    snaps = [_snapshot(t) for t in tensors]
    ents = _table_entries(tensors)
    tab = FocusTable(ents)
    tab.s2()
    tab.step(step, hparams(), flags=F.FOCUS_STEP_WRITE_GRAD)
    assert F.focus_get_error() == 0
    tot = {}
    for e, snap in zip(ents, snaps):
        s2 = oracle.s2(snap[0])
        assert host(e.s2)[0] == s2
        r = _compare_step(e, snap, s2, step)
        for k, v in r.items():
            tot[k] = tot.get(k, 0) + v
    n = synth.LLAMA_1B.n_elements()
    assert tot["elements"] == n
    record(f"C2 Llama-3.2-1B fused step {step}, full", tot)
    assert tot["code_mismatch"] <= MAX_MISMATCH_FRAC * n


def _rows(out, stride):
    r = list(range(0, out, stride))
    if r[-1] != out - 1:
        r.append(out - 1)
    return torch.tensor(r, device="cuda")


def test_c3_llama_8b_bench_configuration(F):
    """The benchmark's launch: s2 over all 224 tensors, then the fused step with W',
    the NVFP4 export of the updated parameters and the tensor maxima, then s2 of
    every tensor from those maxima (equal to the first s2: W is frozen)."""
    from fp4_post_weight_b200.table import FocusTable, hparams
    tensors = []
    for j, (_, sh) in enumerate(synth.LLAMA_8B.tensors()):
        t = synth.llama_8b_tensor(j, sh, "cuda")
        synth.adam_states(t)
        tensors.append(t)
    full_idx = {j for j in range(7)}                  # layer 0: one tensor of each shape, in full
    samples = [None if j in full_idx else _rows(t.W.shape[0], 64) for j, t in enumerate(tensors)]
    snaps = [_snapshot(t, rows) for t, rows in zip(tensors, samples)]
    s2s, amax_bits = [], []
    for t in tensors:                                 # over every row, from the generated W
        wb = host_bits(t.W)
        s2s.append(oracle.s2(wb))
        amax_bits.append(int(np.max(wb & 0x7FFF)))    # max |w| as bf16 magnitude bits
        del wb
    ents = _table_entries(tensors, want_grad=False, export=True)
    tab = FocusTable(ents)
    tab.s2()
    ws = torch.zeros(max(tab.n, 4), dtype=torch.int32, device="cuda")
    F.focus_step_fused_amax(tab.dev, tab.n, tab.total_tiles, hparams(), 1, ws, F.FOCUS_STEP_PACK_UPDATED)
    assert F.focus_get_error() == 0
    assert host(ws)[:tab.n].tolist() == amax_bits    # the maxima the step reduced, every tensor
    F.focus_s2_from_amax(tab.dev, tab.n, ws)
    assert F.focus_get_error() == 0
    assert not host(ws).any()                         # cleared for the next step
    tot = {}
    checked = 0
    for e, snap, rows, s2 in zip(ents, snaps, samples, s2s):
        assert host(e.s2)[0] == s2
        r = _compare_step(e, snap, s2, 1, rows=rows, export=True)
        for k, v in r.items():
            tot[k] = tot.get(k, 0) + v
        checked += snap[0].size
    assert tot["elements"] == checked
    record("C3 Llama-3.1-8B bench launch, layer 0 full + 1/64 rows", tot)
    assert tot["code_mismatch"] <= MAX_MISMATCH_FRAC * checked
    assert 16 * tot["export_scale_mismatch"] + tot["export_code_mismatch"] <= MAX_MISMATCH_FRAC * checked


def test_c5_llama_70b_layers_sampled(F):
    """Llama-3.1-70B layers 0, 40 and 79, each generated on the device, stepped
    (s2, then the fused step with the export) and freed in turn: a 1/256 row
    sample of every tensor against the oracle."""
    from fp4_post_weight_b200.table import FocusTable, hparams
    tot = {}
    for layer in (0, 40, 79):
        tensors = synth.llama_70b_layer(layer, "cuda")
        for t in tensors:
            synth.adam_states(t)
        # s2 of each tensor over all its rows, by the oracle, from the generated weights
        s2s = [oracle.s2(host_bits(t.W)) for t in tensors]
        samples = [_rows(t.W.shape[0], 256) for t in tensors]
        snaps = [_snapshot(t, rows) for t, rows in zip(tensors, samples)]
        ents = _table_entries(tensors, want_grad=False, export=True)
        tab = FocusTable(ents)
        tab.s2()
        tab.step(1, hparams(), flags=F.FOCUS_STEP_PACK_UPDATED)
        assert F.focus_get_error() == 0
        for e, snap, rows, s2 in zip(ents, snaps, samples, s2s):
            assert host(e.s2)[0] == s2
            r = _compare_step(e, snap, s2, 1, rows=rows, export=True)
            for k, v in r.items():
                tot[k] = tot.get(k, 0) + v
        del tab, ents, tensors
        torch.cuda.empty_cache()
    record("C5 Llama-3.1-70B layers 0, 40, 79, 1/256 rows", tot)
    assert tot["code_mismatch"] <= MAX_MISMATCH_FRAC * tot["elements"]
    assert 16 * tot["export_scale_mismatch"] + tot["export_code_mismatch"] <= MAX_MISMATCH_FRAC * tot["elements"]


def test_tensor_above_four_gigabytes(F):
    """A single tensor of more than 2^31 weights (4.3 GB of bf16, byte offsets past
    2^32): s2, forward and pack through the single-tensor calls, then the fused
    step through a one-entry table; s2 over the whole tensor and a row sample at
    the start, the middle and the end against the oracle."""
    from fp4_post_weight_b200.table import Entry, FocusTable, hparams
    o, i = 131072, 16512                              # 2,164,260,864 weights
    g = torch.Generator(device="cuda").manual_seed(31)
    W = synth.normal_bf16((o, i), 0.02, g, "cuda")
    m = synth.uniform((o, i // 16), 0.8, 1.2, g, "cuda")
    q = synth.normal((o, i // 8), 6.0, 2.0, g, "cuda")
    ws = torch.empty(F.focus_s2_workspace_bytes(o, i), dtype=torch.uint8, device="cuda")
    s2d = torch.zeros(1, device="cuda")
    F.focus_s2(W, s2d, ws)
    Wq = torch.empty_like(W)
    s2 = float(host(s2d)[0])
    F.focus_fwd(W, m, q, s2, Wq)
    codes = torch.empty((o, i // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((o, i // 16), dtype=torch.uint8, device="cuda")
    F.focus_pack_nvfp4(W, m, q, s2, codes, scales, torch.zeros(1, device="cuda"))
    assert F.focus_get_error() == 0
    rows = torch.tensor([0, 1, o // 2, o // 2 + 1, o - 2, o - 1], device="cuda")
    assert np.float32(s2) == oracle.s2(host_bits(W))
    Wb, mb, qb = host_bits(W[rows]), host(m[rows]).copy(), host(q[rows]).copy()
    ref = oracle.fwd(Wb, mb, qb, s2)
    mism = check_forward(ref, Wq=host_bits(Wq[rows]), codes=unpack_codes(host(codes[rows])),
                         scales=host(scales[rows]))
    del Wq, codes, scales
    torch.cuda.empty_cache()
    # the fused step over the same tensor (dW' and the moments: another ~13 GB)
    dW = synth.normal_bf16((o, i), 1e-3, g, "cuda")
    Gb = host_bits(dW[rows])
    e = Entry(W=W, m=m, q=q, s2=s2d, dWq=dW, Wq=None, m_exp_avg=torch.zeros_like(m), m_exp_avg_sq=torch.zeros_like(m),
              q_exp_avg=torch.zeros_like(q), q_exp_avg_sq=torch.zeros_like(q))
    tab = FocusTable([e])
    tab.step(1, hparams())
    assert F.focus_get_error() == 0
    z = [np.zeros_like(mb), np.zeros_like(mb), np.zeros_like(qb), np.zeros_like(qb)]
    oracle.step(Wb, Gb, mb, qb, *z, np.float32(s2), 1, want_wq=False)
    skip = block_mask(mism)                           # blocks whose code sits in the 2^-20 band
    assert_close(host(m[rows]), mb, "m", skip)
    assert_close(host(q[rows]), qb, "q", np.repeat(skip, 2, axis=1))
