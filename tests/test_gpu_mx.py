"""GPU parity of the MXFP4 variant (32-element blocks, E8M0 scale, four
sub-blocks of 8) against the oracle: forward (W', codes, E8M0 scales) bit for
bit, straight-through gradients and the fused step (m, q, moments) within
|gpu - ref| <= 1e-7 + 1e-5 |ref|, on shapes spanning many blocks with ragged
grid tails, a Llama-sized tensor, and the non-finite flag; then the same three
over a table of tensors, one launch each (an empty entry, ragged tiles, an
incomplete entry skipped and flagged)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity import assert_close, host, host_bits, unpack_codes

pytestmark = pytest.mark.gpu

SHAPES = [(1, 32), (3, 96), (37, 1056), (128, 2048), (7, 4128), (257, 160)]


@pytest.fixture(scope="module")
def F():
    from fp4_post_weight_b200 import focus
    return focus


def make(shape, seed, dev="cuda"):
    g = torch.Generator(device=dev).manual_seed(seed)
    o, i = shape
    W = synth.add_outliers(synth.normal_bf16(shape, 0.02, g, dev), 2e-3, 20.0, g)
    if o * i >= 128:
        W.view(-1)[:32] = 0                     # a zero block
        W.view(-1)[32:64] *= 1e-30              # a tiny block: x near the E8M0 clamp
    m = synth.uniform((o, i // 32), 0.3, 2.5, g, dev)
    q = synth.normal((o, i // 8), 3.0, 3.0, g, dev)
    dW = synth.normal_bf16(shape, 1e-3, g, dev)
    return W, m, q, dW


def forward(F, W, m, q):
    o, i = W.shape
    Wq = torch.empty_like(W)
    codes = torch.empty((o, i // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((o, i // 32), dtype=torch.uint8, device="cuda")
    F.focus_mx_fwd(W, m, q, Wq, codes, scales)
    return Wq, codes, scales


@pytest.mark.parametrize("shape", SHAPES)
def test_mx_forward(F, shape):
    W, m, q, _ = make(shape, 30 + shape[0])
    Wq, codes, scales = forward(F, W, m, q)
    assert F.focus_get_error() == 0
    ref = oracle.mx_fwd(host_bits(W), host(m), host(q))
    np.testing.assert_array_equal(host(scales), ref.scales)
    np.testing.assert_array_equal(unpack_codes(host(codes)), ref.codes)
    np.testing.assert_array_equal(host_bits(Wq), ref.Wq)


@pytest.mark.parametrize("shape", SHAPES)
def test_mx_backward(F, shape):
    W, m, q, dW = make(shape, 50 + shape[0])
    o, i = shape
    dm = torch.empty((o, i // 32), device="cuda")
    dq = torch.empty((o, i // 8), device="cuda")
    F.focus_mx_ste_bwd(W, dW, m, q, dm, dq)
    rdm, rdq = oracle.mx_ste_bwd(host_bits(W), host_bits(dW), host(m), host(q))
    assert_close(host(dm), rdm, "dm")
    assert_close(host(dq), rdq, "dq")
    F.focus_mx_ste_bwd(W, dW, m, q, dm, dq, accumulate=True)
    oracle.mx_ste_bwd(host_bits(W), host_bits(dW), host(m), host(q), dm=rdm, dq=rdq)
    assert_close(host(dm), rdm, "dm (accumulated)")
    assert_close(host(dq), rdq, "dq (accumulated)")
    assert F.focus_get_error() == 0


@pytest.mark.parametrize("shape,step,warm", [((37, 1056), 1, False), ((128, 2048), 5, True), ((1024, 14336), 1, False)])
def test_mx_step(F, shape, step, warm):
    from fp4_post_weight_b200.table import hparams
    W, m, q, dW = make(shape, 70 + step)
    g = torch.Generator(device="cuda").manual_seed(9)
    if warm:
        # moments as a run leaves them: exp_avg_sq >= exp_avg^2 (else the update is not bounded by ~lr
        # and amplifies rounding differences in the gradient)
        v1m, v1q = synth.normal(m.shape, 0, 1e-4, g, "cuda"), synth.normal(q.shape, 0, 1e-6, g, "cuda")
        mo = [v1m, v1m ** 2 + synth.normal(m.shape, 0, 1e-4, g, "cuda") ** 2,
              v1q, v1q ** 2 + synth.normal(q.shape, 0, 1e-6, g, "cuda") ** 2]
    else:
        mo = [torch.zeros_like(m), torch.zeros_like(m), torch.zeros_like(q), torch.zeros_like(q)]
    hm, hq, hmo = host(m).copy(), host(q).copy(), [host(x).copy() for x in mo]
    Wb, Gb = host_bits(W), host_bits(dW)
    Wq = torch.empty_like(W)
    dm, dq = torch.empty_like(m), torch.empty_like(q)
    F.focus_mx_step(W, dW, m, q, *mo, hparams(), step, F.FOCUS_STEP_WRITE_GRAD, Wq, dm, dq)
    assert F.focus_get_error() == 0
    ref = oracle.mx_fwd(Wb, hm, hq)
    np.testing.assert_array_equal(host_bits(Wq), ref.Wq)               # W' of the parameters before the update
    gm, gq = oracle.mx_ste_bwd(Wb, Gb, hm, hq)
    assert_close(host(dm), gm, "dm")
    assert_close(host(dq), gq, "dq")
    oracle.adamw(hm, gm, hmo[0], hmo[1], 5e-3, step)
    oracle.adamw(hq, gq, hmo[2], hmo[3], 1e-3, step)
    assert_close(host(m), hm, "m")
    assert_close(host(q), hq, "q")
    for name, t, r in zip(("m exp_avg", "m exp_avg_sq", "q exp_avg", "q exp_avg_sq"), mo, hmo):
        assert_close(host(t), r, name)


def test_mx_nonfinite_sets_flag(F):
    W, m, q, _ = make((4, 64), 3)
    W[2, 5] = float("nan")
    assert F.focus_get_error() == 0
    forward(F, W, m, q)
    assert F.focus_get_error() == 7
    assert F.focus_get_error() == 0


# ---------------------------------------------------------------------------
# many tensors in one launch (a table prepared for the MXFP4 calls)
# ---------------------------------------------------------------------------

MULTI_SHAPES = [(1, 32), (3, 96), (37, 1056), (0, 64), (128, 2048), (7, 4128), (257, 160)]


def mx_table(F, seed, moments="zero", missing=None):
    """A table over MULTI_SHAPES (an empty tensor in the middle; 4096-weight tiles with
    ragged ends) with every output present, except the fields named in `missing` on
    entry 2."""
    from fp4_post_weight_b200.table import PURPOSE_MX, Entry, FocusTable
    g = torch.Generator(device="cuda").manual_seed(seed)
    ents, hosts = [], []
    for j, shape in enumerate(MULTI_SHAPES):
        o, i = shape
        if o * i:
            W, m, q, dW = make(shape, seed + 10 * j)
        else:
            W, dW = torch.empty(shape, dtype=torch.bfloat16, device="cuda"), torch.empty(shape, dtype=torch.bfloat16,
                                                                                         device="cuda")
            m, q = torch.empty((o, i // 32), device="cuda"), torch.empty((o, i // 8), device="cuda")
        if moments == "warm":
            v1m, v1q = synth.normal(m.shape, 0, 1e-4, g, "cuda"), synth.normal(q.shape, 0, 1e-6, g, "cuda")
            mo = [v1m, v1m ** 2 + synth.normal(m.shape, 0, 1e-4, g, "cuda") ** 2,
                  v1q, v1q ** 2 + synth.normal(q.shape, 0, 1e-6, g, "cuda") ** 2]
        else:
            mo = [torch.zeros_like(m), torch.zeros_like(m), torch.zeros_like(q), torch.zeros_like(q)]
        e = Entry(W=W, m=m, q=q, s2=None, dWq=dW, Wq=torch.empty_like(W), m_exp_avg=mo[0], m_exp_avg_sq=mo[1],
                  q_exp_avg=mo[2], q_exp_avg_sq=mo[3],
                  codes=torch.empty((o, i // 2), dtype=torch.uint8, device="cuda"),
                  scales=torch.empty((o, i // 32), dtype=torch.uint8, device="cuda"),
                  dm=torch.zeros_like(m), dq=torch.zeros_like(q))
        if j == 2 and missing:
            for name in missing:
                setattr(e, name, None)
        ents.append(e)
        hosts.append((host_bits(W), host_bits(dW), host(m).copy(), host(q).copy(), [host(x).copy() for x in mo]))
    return FocusTable(ents, PURPOSE_MX), hosts


def test_mx_multi_forward(F):
    tab, hosts = mx_table(F, 300)
    tab.mx_fwd()
    assert F.focus_get_error() == 0
    for e, (Wb, _, hm, hq, _) in zip(tab.entries, hosts):
        if e.W.numel() == 0:
            continue
        ref = oracle.mx_fwd(Wb, hm, hq)
        np.testing.assert_array_equal(host(e.scales), ref.scales)
        np.testing.assert_array_equal(unpack_codes(host(e.codes)), ref.codes)
        np.testing.assert_array_equal(host_bits(e.Wq), ref.Wq)


def test_mx_multi_backward(F):
    tab, hosts = mx_table(F, 400)
    tab.mx_bwd()
    tab.mx_bwd(accumulate=True)
    assert F.focus_get_error() == 0
    for e, (Wb, Gb, hm, hq, _) in zip(tab.entries, hosts):
        if e.W.numel() == 0:
            continue
        rdm, rdq = oracle.mx_ste_bwd(Wb, Gb, hm, hq)
        oracle.mx_ste_bwd(Wb, Gb, hm, hq, dm=rdm, dq=rdq)
        assert_close(host(e.dm), rdm, "dm (two micro-batches)")
        assert_close(host(e.dq), rdq, "dq (two micro-batches)")


@pytest.mark.parametrize("step,moments", [(1, "zero"), (5, "warm")])
def test_mx_multi_step(F, step, moments):
    from fp4_post_weight_b200.table import hparams
    tab, hosts = mx_table(F, 500 + step, moments)
    tab.mx_step(step, hparams(), F.FOCUS_STEP_WRITE_GRAD)
    assert F.focus_get_error() == 0
    for e, (Wb, Gb, hm, hq, hmo) in zip(tab.entries, hosts):
        if e.W.numel() == 0:
            continue
        ref = oracle.mx_fwd(Wb, hm, hq)
        np.testing.assert_array_equal(host_bits(e.Wq), ref.Wq)          # W' of the parameters before the update
        gm, gq = oracle.mx_ste_bwd(Wb, Gb, hm, hq)
        assert_close(host(e.dm), gm, "dm")
        assert_close(host(e.dq), gq, "dq")
        oracle.adamw(hm, gm, hmo[0], hmo[1], 5e-3, step)
        oracle.adamw(hq, gq, hmo[2], hmo[3], 1e-3, step)
        assert_close(host(e.m), hm, "m")
        assert_close(host(e.q), hq, "q")
        for name, t, r in zip(("m exp_avg", "m exp_avg_sq", "q exp_avg", "q exp_avg_sq"),
                              (e.m_exp_avg, e.m_exp_avg_sq, e.q_exp_avg, e.q_exp_avg_sq), hmo):
            assert_close(host(t), r, name)


def test_mx_multi_step_skips_an_incomplete_entry(F):
    """An entry without a pointer the step needs (its second moment of q) is skipped
    and flagged; the other entries are stepped as usual."""
    from fp4_post_weight_b200.table import hparams
    tab, hosts = mx_table(F, 600, missing=("q_exp_avg_sq",))
    m2 = host(tab.entries[2].m).copy()
    assert F.focus_get_error() == 0
    tab.mx_step(1, hparams())
    assert F.focus_get_error() == 7
    np.testing.assert_array_equal(host(tab.entries[2].m), m2)          # untouched
    Wb, Gb, hm, hq, hmo = hosts[1]
    gm, gq = oracle.mx_ste_bwd(Wb, Gb, hm, hq)
    oracle.adamw(hm, gm, hmo[0], hmo[1], 5e-3, 1)
    assert_close(host(tab.entries[1].m), hm, "m of the entry before")
    Wb, Gb, hm, hq, hmo = hosts[4]
    gm, gq = oracle.mx_ste_bwd(Wb, Gb, hm, hq)
    oracle.adamw(hq, gq, hmo[2], hmo[3], 1e-3, 1)
    assert_close(host(tab.entries[4].q), hq, "q of an entry after")


def test_mx_multi_step_exports_the_update(F):
    """FOCUS_STEP_PACK_UPDATED | FOCUS_STEP_WQ_UPDATED on the table step: codes, E8M0
    scales and W' are bit for bit what focus_mx_fwd_multi writes after a plain step,
    and m, q and the moments are those of the plain step."""
    from fp4_post_weight_b200.table import hparams
    ta, _ = mx_table(F, 700, "warm")
    tb, _ = mx_table(F, 700, "warm")
    ta.mx_step(4, hparams(), F.FOCUS_STEP_PACK_UPDATED | F.FOCUS_STEP_WQ_UPDATED)
    tb.mx_step(4, hparams())
    tb.mx_fwd()
    assert F.focus_get_error() == 0
    for a, b in zip(ta.entries, tb.entries):
        for name in ("codes", "scales", "Wq", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq"):
            x, y = getattr(a, name), getattr(b, name)
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), name


def test_mx_step_wq_of_the_update(F):
    """FOCUS_STEP_WQ_UPDATED on the single-tensor step: W' is bit for bit what
    focus_mx_fwd writes after a plain step."""
    from fp4_post_weight_b200.table import hparams
    W, m, q, dW = make((37, 1056), 710)
    mo = [torch.zeros_like(m), torch.zeros_like(m), torch.zeros_like(q), torch.zeros_like(q)]
    m2, q2, mo2 = m.clone(), q.clone(), [x.clone() for x in mo]
    Wq_a = torch.empty_like(W)
    F.focus_mx_step(W, dW, m, q, *mo, hparams(), 1, F.FOCUS_STEP_WQ_UPDATED, Wq_a)
    F.focus_mx_step(W, dW, m2, q2, *mo2, hparams(), 1, 0, torch.empty_like(W))
    Wq_b, _, _ = forward(F, W, m2, q2)
    assert F.focus_get_error() == 0
    assert torch.equal(m, m2) and torch.equal(q, q2)
    assert torch.equal(Wq_a.view(torch.int16), Wq_b.view(torch.int16))


@pytest.mark.parametrize("wqu", [False, True])
def test_mx_export_kernels_for_fixed_options_match_the_runtime_one(F, wqu):
    """The table step with the export runs in a kernel compiled for its options
    (the export with or without W' of the update, no accumulation, no gradient
    output) and otherwise in the kernel that reads them at run time, which
    FOCUS_STEP_WRITE_GRAD selects: both leave bit-identical parameters,
    moments, W', codes and scales from the same inputs."""
    from fp4_post_weight_b200.table import hparams
    flags = F.FOCUS_STEP_PACK_UPDATED | (F.FOCUS_STEP_WQ_UPDATED if wqu else 0)
    ta, _ = mx_table(F, 720, "warm")
    tb, _ = mx_table(F, 720, "warm")
    ta.mx_step(3, hparams(), flags)
    tb.mx_step(3, hparams(), flags | F.FOCUS_STEP_WRITE_GRAD)
    assert F.focus_get_error() == 0
    for a, b in zip(ta.entries, tb.entries):
        for name in ("codes", "scales", "Wq", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq"):
            x, y = getattr(a, name), getattr(b, name)
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), name
