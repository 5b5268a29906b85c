"""GPU parity of the later rows at the benchmark's sizes, in the launch
configurations bench.py times:

* FourOverSix weights over all 224 Llama-3.1-8B linears in one multi-tensor
  launch (codes, scales and W'), layer 0 in full and a 1/64 row sample of
  every other tensor, bit for bit against the oracle with each tensor's s2;
* FourOverSix with one scale per token over one decoder layer's linear inputs
  for a micro-batch of 4096 tokens (one launch over the four tensors), in full;
* the calibration step over four micro-batches (bench order) on layer 0 of the
  8B shapes, a 1/16 row sample;
* plain NVFP4 round to nearest: the weights over all 224 linears in one launch
  (layer 0 in full, a 1/64 row sample of the rest) and the same per-token
  inputs in one launch, in full;
* the MXFP4 fused step, one launch per tensor, on layer 0 of the 8B shapes
  with the benchmark's parameters (m = 1, q = 6, zero moments), a 1/16 row
  sample against the oracle, and the same step as one launch over a table of
  all 224 tensors (layer 0 at 1/16, the rest at 1/128 of the rows); the table
  step with the export of the updated parameters on layer 0, against the
  table forward after a plain step.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity import (MAX_MISMATCH_FRAC, assert_close, check_fouroversix, f46_tie_counts, host, host_bits,
                          record, unpack_codes)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    from fp4_post_weight_b200 import focus
    return focus


def _rows(out, stride):
    r = list(range(0, out, stride))
    if r[-1] != out - 1:
        r.append(out - 1)
    return torch.tensor(r, device="cuda")


def test_fouroversix_weights_llama_8b_one_launch(F):
    from fp4_post_weight_b200.table import Entry, FocusTable, PURPOSE_FOUROVERSIX
    ents, samples = [], []
    for j, (_, (o, i)) in enumerate(synth.LLAMA_8B.tensors()):
        t = synth.llama_8b_tensor(j, (o, i), "cuda", with_grad=False)
        ents.append(Entry(W=t.W, m=None, q=None, s2=torch.zeros(1, device="cuda"),
                          codes=torch.empty((o, i // 2), dtype=torch.uint8, device="cuda"),
                          scales=torch.empty((o, i // 16), dtype=torch.uint8, device="cuda"),
                          Wq=torch.empty_like(t.W)))
        samples.append(None if j < 7 else _rows(o, 64))
    tab = FocusTable(ents, PURPOSE_FOUROVERSIX)
    tab.s2()
    tab.fouroversix()
    assert F.focus_get_error() == 0
    total = {}
    for e, rows in zip(ents, samples):
        s2 = oracle.s2(host_bits(e.W))
        assert host(e.s2)[0] == s2
        sel = (lambda x: x) if rows is None else (lambda x: x[rows])
        ref = oracle.fouroversix(host_bits(sel(e.W)), s2)
        c = check_fouroversix(ref, unpack_codes(host(sel(e.codes))), host(sel(e.scales)), host_bits(sel(e.Wq)))
        c.update(f46_tie_counts(ref, host_bits(sel(e.W)), s2))
        for k, v in c.items():
            total[k] = total.get(k, 0) + v
    assert total["mismatched_blocks"] <= MAX_MISMATCH_FRAC * total["blocks"]
    record("FourOverSix weights, Llama-3.1-8B layer 0 full + 1/64 rows (blocks)", total)


def _layer_inputs():
    """One decoder layer's linear inputs for 4096 tokens (q/k/v, o, gate/up, down), as one
    activation table (the benchmark's launch), with X' written."""
    from fp4_post_weight_b200.table import ActTable, act_entry
    ents = []
    for j, h in enumerate((4096, 4096, 4096, 14336)):
        X = synth.activations(4096, h, "cuda", seed=50 + j)
        ents.append(act_entry(X, torch.empty(4096, device="cuda"),
                              torch.empty((4096, h // 2), dtype=torch.uint8, device="cuda"),
                              torch.empty((4096, h // 16), dtype=torch.uint8, device="cuda"), torch.empty_like(X)))
    return ents, ActTable(ents)


def test_fouroversix_activations_one_layer_4096_tokens(F):
    ents, tab = _layer_inputs()
    tab.fouroversix()
    assert F.focus_get_error() == 0
    for e in ents:
        ref = oracle.fouroversix(host_bits(e.W))
        np.testing.assert_array_equal(host(e.s2), ref.row_scales)
        c = check_fouroversix(ref, unpack_codes(host(e.codes)), host(e.scales), host_bits(e.Wq))
        assert c["mismatched_blocks"] <= MAX_MISMATCH_FRAC * c["blocks"], c
        c.update(f46_tie_counts(ref, host_bits(e.W), ref.row_scales))
        record("FourOverSix per token, one 8B layer's inputs, 4096 tokens (blocks)", c)


def test_mx_step_llama_8b_layer0_sampled(F):
    from fp4_post_weight_b200.table import hparams
    for j, (_, (o, i)) in enumerate(synth.LLAMA_8B.tensors()[:7]):
        t = synth.llama_8b_tensor(j, (o, i), "cuda")
        m = torch.ones((o, i // 32), device="cuda")
        q = torch.full((o, i // 8), 6.0, device="cuda")
        mo = [torch.zeros_like(m), torch.zeros_like(m), torch.zeros_like(q), torch.zeros_like(q)]
        rows = _rows(o, 16)
        Wb, Gb = host_bits(t.W[rows]), host_bits(t.dWq[rows])
        hm, hq = host(m[rows]).copy(), host(q[rows]).copy()
        hmo = [host(x[rows]).copy() for x in mo]
        Wq = torch.empty_like(t.W)
        F.focus_mx_step(t.W, t.dWq, m, q, *mo, hparams(), 1, 0, Wq)
        assert F.focus_get_error() == 0
        np.testing.assert_array_equal(host_bits(Wq[rows]), oracle.mx_fwd(Wb, hm, hq).Wq)
        gm, gq = oracle.mx_ste_bwd(Wb, Gb, hm, hq)
        oracle.adamw(hm, gm, hmo[0], hmo[1], 5e-3, 1)
        oracle.adamw(hq, gq, hmo[2], hmo[3], 1e-3, 1)
        assert_close(host(m[rows]), hm, "m")
        assert_close(host(q[rows]), hq, "q")
        for name, x, r in zip(("m exp_avg", "m exp_avg_sq", "q exp_avg", "q exp_avg_sq"), mo, hmo):
            assert_close(host(x[rows]), r, name)


def test_mx_step_table_llama_8b_sampled(F):
    """The MXFP4 step as one launch over a table of all 224 8B linears (the bench's
    one-launch line): a 1/16 row sample of layer 0 and a 1/128 row sample of every
    other tensor against the oracle."""
    from fp4_post_weight_b200.table import PURPOSE_MX, Entry, FocusTable, hparams
    ents, checks = [], []
    for j, (_, (o, i)) in enumerate(synth.LLAMA_8B.tensors()):
        t = synth.llama_8b_tensor(j, (o, i), "cuda")
        m = torch.ones((o, i // 32), device="cuda")
        q = torch.full((o, i // 8), 6.0, device="cuda")
        e = Entry(W=t.W, m=m, q=q, s2=None, dWq=t.dWq, Wq=torch.empty_like(t.W),
                  m_exp_avg=torch.zeros_like(m), m_exp_avg_sq=torch.zeros_like(m),
                  q_exp_avg=torch.zeros_like(q), q_exp_avg_sq=torch.zeros_like(q))
        ents.append(e)
        rows = _rows(o, 16 if j < 7 else 128)
        checks.append((rows, host_bits(t.W[rows]), host_bits(t.dWq[rows])))
    tab = FocusTable(ents, PURPOSE_MX)
    tab.mx_step(1, hparams())
    assert F.focus_get_error() == 0
    checked = 0
    for e, (rows, Wb, Gb) in zip(ents, checks):
        o, i = e.W.shape
        hm = np.ones((len(rows), i // 32), np.float32)
        hq = np.full((len(rows), i // 8), 6.0, np.float32)
        hmo = [np.zeros_like(hm), np.zeros_like(hm), np.zeros_like(hq), np.zeros_like(hq)]
        np.testing.assert_array_equal(host_bits(e.Wq[rows]), oracle.mx_fwd(Wb, hm, hq).Wq)
        gm, gq = oracle.mx_ste_bwd(Wb, Gb, hm, hq)
        oracle.adamw(hm, gm, hmo[0], hmo[1], 5e-3, 1)
        oracle.adamw(hq, gq, hmo[2], hmo[3], 1e-3, 1)
        assert_close(host(e.m[rows]), hm, "m")
        assert_close(host(e.q[rows]), hq, "q")
        for name, x, r in zip(("m exp_avg", "m exp_avg_sq", "q exp_avg", "q exp_avg_sq"),
                              (e.m_exp_avg, e.m_exp_avg_sq, e.q_exp_avg, e.q_exp_avg_sq), hmo):
            assert_close(host(x[rows]), r, name)
        checked += Wb.size
    print(f"MXFP4 table step: {checked} weights checked over {len(ents)} tensors")


def test_nvfp4_weights_llama_8b_one_launch(F):
    """Plain NVFP4 round to nearest over all 224 8B linears in one launch (the bench's
    line): layer 0 in full, a 1/64 row sample of every other tensor, against the
    oracle's forward with m = 1, sigmoid = 1."""
    from fp4_post_weight_b200.table import Entry, FocusTable, PURPOSE_FOUROVERSIX
    ents, samples = [], []
    for j, (_, (o, i)) in enumerate(synth.LLAMA_8B.tensors()):
        t = synth.llama_8b_tensor(j, (o, i), "cuda", with_grad=False)
        ents.append(Entry(W=t.W, m=None, q=None, s2=torch.zeros(1, device="cuda"),
                          codes=torch.empty((o, i // 2), dtype=torch.uint8, device="cuda"),
                          scales=torch.empty((o, i // 16), dtype=torch.uint8, device="cuda")))
        samples.append(None if j < 7 else _rows(o, 64))
    tab = FocusTable(ents, PURPOSE_FOUROVERSIX)
    tab.s2()
    tab.nvfp4_rtn()
    assert F.focus_get_error() == 0
    for e, rows in zip(ents, samples):
        Wb = host_bits(e.W if rows is None else e.W[rows])
        s2 = oracle.s2(host_bits(e.W))
        o, i = Wb.shape
        ref = oracle.fwd(Wb, np.ones((o, i // 16), np.float32), np.full((o, i // 8), 30.0, np.float32), s2)
        sel = (lambda x: x) if rows is None else (lambda x: x[rows])
        np.testing.assert_array_equal(host(sel(e.scales)), ref.scales)
        np.testing.assert_array_equal(unpack_codes(host(sel(e.codes))), ref.codes)


def test_nvfp4_activations_one_layer_4096_tokens(F):
    ents, tab = _layer_inputs()
    tab.nvfp4()
    assert F.focus_get_error() == 0
    for e in ents:
        ref = oracle.nvfp4_rows(host_bits(e.W))
        np.testing.assert_array_equal(host(e.s2), ref.row_scales)
        np.testing.assert_array_equal(host(e.scales), ref.scales)
        np.testing.assert_array_equal(unpack_codes(host(e.codes)), ref.codes)
        np.testing.assert_array_equal(host_bits(e.Wq), ref.Xq)


def test_micro_batch_step_llama_8b_layer0_sampled(F):
    """The calibration step over four micro-batches as the bench times it (table
    backward, two accumulating backward passes, then the accumulating step with the
    next step's W') on layer 0 of the 8B shapes with the bench's parameters (m = 1,
    q = 6, zero moments), a 1/16 row sample against the oracle."""
    from fp4_post_weight_b200.table import Entry, FocusTable, hparams
    from tests.parity import block_mask, check_forward
    ents, grads, samples = [], [], []
    g = torch.Generator(device="cuda").manual_seed(21)
    for j, (_, (o, i)) in enumerate(synth.LLAMA_8B.tensors()[:7]):
        t = synth.llama_8b_tensor(j, (o, i), "cuda")
        ents.append(Entry(W=t.W, m=t.m, q=t.q, s2=torch.zeros(1, device="cuda"), dWq=t.dWq, Wq=torch.empty_like(t.W),
                          m_exp_avg=torch.zeros_like(t.m), m_exp_avg_sq=torch.zeros_like(t.m),
                          q_exp_avg=torch.zeros_like(t.q), q_exp_avg_sq=torch.zeros_like(t.q),
                          dm=torch.zeros_like(t.m), dq=torch.zeros_like(t.q)))
        grads.append([synth.normal_bf16((o, i), 1e-3, g, "cuda") for _ in range(4)])
        samples.append(_rows(o, 16))
    host_in = [(host_bits(e.W[r]), host(e.m[r]).copy(), host(e.q[r]).copy(), [host_bits(x[r]) for x in gs])
               for e, gs, r in zip(ents, grads, samples)]
    tab = FocusTable(ents)
    tab.s2()
    for j in range(3):
        for e, gs in zip(ents, grads):
            e.dWq.copy_(gs[j])
        tab.bwd(accumulate=j > 0)
    for e, gs in zip(ents, grads):
        e.dWq.copy_(gs[3])
    tab.step(1, hparams(), flags=F.FOCUS_STEP_ACCUMULATE | F.FOCUS_STEP_WRITE_GRAD | F.FOCUS_STEP_WQ_UPDATED)
    assert F.focus_get_error() == 0
    for e, r, (Wb, m, q, Gs) in zip(ents, samples, host_in):
        s2 = host(e.s2)[0]
        assert s2 == oracle.s2(host_bits(e.W))
        skip = block_mask(check_forward(oracle.fwd(Wb, m, q, s2)))
        dm, dq = oracle.ste_bwd(Wb, Gs[0], m, q, s2)
        for j in (1, 2):
            oracle.ste_bwd(Wb, Gs[j], m, q, s2, dm=dm, dq=dq)
        z = [np.zeros_like(m), np.zeros_like(m), np.zeros_like(q), np.zeros_like(q)]
        _, gm, gq = oracle.step(Wb, Gs[3], m, q, *z, s2, 1, want_wq=False, dm_acc=dm, dq_acc=dq)
        skq = np.repeat(skip, 2, axis=1)
        assert_close(host(e.dm[r]), gm, "dm over four micro-batches", skip)
        assert_close(host(e.dq[r]), gq, "dq over four micro-batches", skq)
        assert_close(host(e.m[r]), m, "m", skip)
        assert_close(host(e.q[r]), q, "q", skq)
        # W' of the updated parameters: the oracle's forward of the device's updated m
        # and q; a value may differ only where its quotient lies in the 2^-20 band
        ref = oracle.fwd(Wb, host(e.m[r]).copy(), host(e.q[r]).copy(), s2)
        diff = host_bits(e.Wq[r]) != ref.Wq
        assert not (diff & (ref.band == 0)).any()
        assert diff.sum() <= 1e-6 * diff.size + 1


def test_mx_step_export_llama_8b_layer0(F):
    """The MXFP4 table step with the export of the updated parameters (the bench's
    one_launch_export line) on layer 0 of the 8B shapes: codes, E8M0 scales and W'
    bit for bit what the table forward writes after a plain step, and the updated
    m, q and moments identical to the plain step's."""
    from fp4_post_weight_b200.table import PURPOSE_MX, Entry, FocusTable, hparams

    def table():
        ents = []
        for j, (_, (o, i)) in enumerate(synth.LLAMA_8B.tensors()[:7]):
            t = synth.llama_8b_tensor(j, (o, i), "cuda")
            m = torch.ones((o, i // 32), device="cuda")
            q = torch.full((o, i // 8), 6.0, device="cuda")
            ents.append(Entry(W=t.W, m=m, q=q, s2=None, dWq=t.dWq, Wq=torch.empty_like(t.W),
                              m_exp_avg=torch.zeros_like(m), m_exp_avg_sq=torch.zeros_like(m),
                              q_exp_avg=torch.zeros_like(q), q_exp_avg_sq=torch.zeros_like(q),
                              codes=torch.empty((o, i // 2), dtype=torch.uint8, device="cuda"),
                              scales=torch.empty((o, i // 32), dtype=torch.uint8, device="cuda")))
        return FocusTable(ents, PURPOSE_MX)
    ta = table()
    ta.mx_step(1, hparams(), F.FOCUS_STEP_PACK_UPDATED | F.FOCUS_STEP_WQ_UPDATED)
    assert F.focus_get_error() == 0
    tb = table()
    tb.mx_step(1, hparams())
    tb.mx_fwd()
    assert F.focus_get_error() == 0
    for a, b in zip(ta.entries, tb.entries):
        for name in ("codes", "scales", "Wq", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq"):
            x, y = getattr(a, name), getattr(b, name)
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), name
