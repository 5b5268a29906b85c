"""GPU parity of every C-ABI entry point against the oracle, on small shapes
that span several tiles (4096 weights each) and end in ragged tails."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity import (assert_close, block_mask, check_forward, host, host_bits, unpack_codes)

pytestmark = pytest.mark.gpu

SHAPES = [(1, 16), (3, 48), (2, 4096), (37, 1040), (7, 4112), (128, 2048), (257, 160)]


@pytest.fixture(scope="module")
def F():
    from fp4_post_weight_b200 import focus
    return focus


def make(shape, seed, q_mean=3.0, q_std=3.0, dev="cuda"):
    g = torch.Generator(device=dev).manual_seed(seed)
    o, i = shape
    W = synth.add_outliers(synth.normal_bf16(shape, 0.02, g, dev), 2e-3, 20.0, g) if o * i else \
        torch.zeros(shape, dtype=torch.bfloat16, device=dev)
    if o * i >= 64:
        W.view(-1)[:16] = 0          # a zero block
    m = synth.uniform((o, i // 16), 0.3, 2.5, g, dev)
    q = synth.normal((o, i // 8), q_mean, q_std, g, dev)
    dW = synth.normal_bf16(shape, 1e-3, g, dev)
    return W, m, q, dW


@pytest.mark.parametrize("shape", SHAPES + [(0, 64), (8, 0)])
def test_s2(F, shape):
    W, *_ = make(shape, 1)
    o, i = shape
    ws = torch.empty(max(F.focus_s2_workspace_bytes(o, i), 16), dtype=torch.uint8, device="cuda")
    s2 = torch.full((1,), -1.0, device="cuda")
    F.focus_s2(W, s2, ws)
    want = oracle.s2(host_bits(W))
    assert host(s2)[0] == want


@pytest.mark.parametrize("shape", SHAPES)
def test_fwd_and_pack(F, shape):
    W, m, q, _ = make(shape, 2)
    o, i = shape
    s2 = float(oracle.s2(host_bits(W)))
    Wq = torch.empty_like(W)
    F.focus_fwd(W, m, q, s2, Wq)
    codes = torch.empty((o, i // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((o, i // 16), dtype=torch.uint8, device="cuda")
    ts = torch.zeros(1, device="cuda")
    F.focus_pack_nvfp4(W, m, q, s2, codes, scales, ts)
    assert F.focus_get_error() == 0
    ref = oracle.fwd(host_bits(W), host(m), host(q), s2)
    check_forward(ref, Wq=host_bits(Wq), codes=unpack_codes(host(codes)), scales=host(scales))
    assert host(ts)[0] == np.float32(s2)
    rc, rs, rt = oracle.pack(host_bits(W), host(m), host(q), s2)
    assert rt == host(ts)[0]


@pytest.mark.parametrize("shape", SHAPES)
def test_ste_bwd(F, shape):
    W, m, q, dW = make(shape, 3)
    o, i = shape
    s2 = float(oracle.s2(host_bits(W)))
    dm = torch.empty((o, i // 16), device="cuda")
    dq = torch.empty((o, i // 8), device="cuda")
    F.focus_ste_bwd(W, dW, m, q, s2, dm, dq)
    ref_f = oracle.fwd(host_bits(W), host(m), host(q), s2)
    codes = torch.empty((o, i // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((o, i // 16), dtype=torch.uint8, device="cuda")
    F.focus_pack_nvfp4(W, m, q, s2, codes, scales, torch.zeros(1, device="cuda"))
    mism = check_forward(ref_f, codes=unpack_codes(host(codes)))
    skip = block_mask(mism)
    rdm, rdq = oracle.ste_bwd(host_bits(W), host_bits(dW), host(m), host(q), s2)
    assert_close(host(dm), rdm, "dm", skip)
    assert_close(host(dq), rdq, "dq", np.repeat(skip, 2, axis=1))
    # accumulate: add a second gradient
    F.focus_ste_bwd(W, dW, m, q, s2, dm, dq, accumulate=True)
    rdm2, rdq2 = oracle.ste_bwd(host_bits(W), host_bits(dW), host(m), host(q), s2, dm=rdm.copy(), dq=rdq.copy())
    assert_close(host(dm), rdm2, "dm (accumulated)", skip)
    assert_close(host(dq), rdq2, "dq (accumulated)", np.repeat(skip, 2, axis=1))
    assert F.focus_get_error() == 0


@pytest.mark.parametrize("n,wd", [(1, 0.0), (7, 0.0), (4099, 0.0), (4099, 0.01), (100000, 0.0)])
def test_adamw(F, n, wd):
    g = torch.Generator(device="cuda").manual_seed(n)
    p = synth.normal((n,), 6.0, 2.0, g, "cuda")
    v1 = torch.zeros(n, device="cuda"); v2 = torch.zeros(n, device="cuda")
    hp, hv1, hv2 = host(p).copy(), host(v1).copy(), host(v2).copy()
    for t in range(1, 6):
        gr = synth.normal((n,), 0.0, 1e-4, g, "cuda")
        F.focus_adamw_step(p, gr, v1, v2, 1e-3, t, weight_decay=wd)
        oracle.adamw(hp, host(gr), hv1, hv2, 1e-3, t, weight_decay=wd)
    assert_close(host(p), hp, "p")
    assert_close(host(v1), hv1, "exp_avg")
    assert_close(host(v2), hv2, "exp_avg_sq")


def _entries(shapes, seed, with_pack=True, warm=False):
    from fp4_post_weight_b200.table import Entry
    ents = []
    for j, sh in enumerate(shapes):
        W, m, q, dW = make(sh, seed + j)
        o, i = sh
        e = Entry(W=W, m=m, q=q, s2=torch.zeros(1, device="cuda"), dWq=dW, Wq=torch.empty_like(W))
        g = torch.Generator(device="cuda").manual_seed(100 + j)
        if warm:
            # moments as a run leaves them: exp_avg_sq >= exp_avg^2
            e.m_exp_avg = synth.normal(m.shape, 0, 1e-4, g, "cuda")
            e.m_exp_avg_sq = e.m_exp_avg ** 2 + synth.normal(m.shape, 0, 1e-4, g, "cuda") ** 2
            e.q_exp_avg = synth.normal(q.shape, 0, 1e-6, g, "cuda")
            e.q_exp_avg_sq = e.q_exp_avg ** 2 + synth.normal(q.shape, 0, 1e-6, g, "cuda") ** 2
        else:
            e.m_exp_avg = torch.zeros_like(m); e.m_exp_avg_sq = torch.zeros_like(m)
            e.q_exp_avg = torch.zeros_like(q); e.q_exp_avg_sq = torch.zeros_like(q)
        if with_pack:
            e.codes = torch.empty((o, i // 2), dtype=torch.uint8, device="cuda")
            e.scales = torch.empty((o, i // 16), dtype=torch.uint8, device="cuda")
        e.dm = torch.zeros_like(m); e.dq = torch.zeros_like(q)
        ents.append(e)
    return ents


@pytest.mark.parametrize("warm,step", [(False, 1), (True, 5)])
def test_step_fused_table(F, warm, step):
    from fp4_post_weight_b200.table import FocusTable, hparams
    shapes = SHAPES + [(0, 32)]
    ents = _entries(shapes, 10, warm=warm)
    host_in = [(host_bits(e.W), host_bits(e.dWq), host(e.m).copy(), host(e.q).copy(),
                [host(x).copy() for x in (e.m_exp_avg, e.m_exp_avg_sq, e.q_exp_avg, e.q_exp_avg_sq)])
               for e in ents]
    tab = FocusTable(ents)
    tab.s2()
    tab.step(step, hparams(), flags=F.FOCUS_STEP_WRITE_GRAD)
    assert F.focus_get_error() == 0
    for e, (Wb, Gb, m, q, st) in zip(ents, host_in):
        if Wb.size == 0:
            continue
        s2 = oracle.s2(Wb)
        assert host(e.s2)[0] == s2
        ref_f = oracle.fwd(Wb, m, q, s2)
        mism = check_forward(ref_f, Wq=host_bits(e.Wq), codes=unpack_codes(host(e.codes)), scales=host(e.scales))
        skip = block_mask(mism)
        skq = np.repeat(skip, 2, axis=1)
        _, gm, gq = oracle.step(Wb, Gb, m, q, *st, s2, step, want_wq=False)
        assert_close(host(e.dm), gm, "dm", skip)
        assert_close(host(e.dq), gq, "dq", skq)
        assert_close(host(e.m), m, "m", skip)
        assert_close(host(e.q), q, "q", skq)
        assert_close(host(e.m_exp_avg), st[0], "m exp_avg", skip)
        assert_close(host(e.m_exp_avg_sq), st[1], "m exp_avg_sq", skip)
        assert_close(host(e.q_exp_avg), st[2], "q exp_avg", skq)
        assert_close(host(e.q_exp_avg_sq), st[3], "q exp_avg_sq", skq)


def test_step_accumulate_and_pack_multi(F):
    from fp4_post_weight_b200.table import FocusTable, hparams
    shapes = [(37, 1040), (64, 512)]
    ents = _entries(shapes, 40)
    g = torch.Generator(device="cuda").manual_seed(7)
    for e in ents:
        e.dm.copy_(synth.normal(e.dm.shape, 0, 1e-5, g, "cuda"))
        e.dq.copy_(synth.normal(e.dq.shape, 0, 1e-7, g, "cuda"))
    host_in = [(host_bits(e.W), host_bits(e.dWq), host(e.m).copy(), host(e.q).copy(), host(e.dm).copy(),
                host(e.dq).copy()) for e in ents]
    tab = FocusTable(ents)
    tab.s2()
    tab.pack()          # codes/scales of the generated m, q; W' is not written by the pack
    torch.cuda.synchronize()
    for e, (Wb, _, m, q, _, _) in zip(ents, host_in):
        s2 = oracle.s2(Wb)
        codes, scales, _ = oracle.pack(Wb, m, q, s2)
        np.testing.assert_array_equal(host(e.scales), scales)
        ref = oracle.fwd(Wb, m, q, s2)
        check_forward(ref, codes=unpack_codes(host(e.codes)))
    tab.step(1, hparams(), flags=F.FOCUS_STEP_ACCUMULATE | F.FOCUS_STEP_WRITE_GRAD)
    assert F.focus_get_error() == 0
    for e, (Wb, Gb, m, q, dm0, dq0) in zip(ents, host_in):
        s2 = oracle.s2(Wb)
        z = [np.zeros_like(m), np.zeros_like(m), np.zeros_like(q), np.zeros_like(q)]
        _, gm, gq = oracle.step(Wb, Gb, m, q, *z, s2, 1, want_wq=False, dm_acc=dm0, dq_acc=dq0)
        assert_close(host(e.dm), gm, "accumulated dm")
        assert_close(host(e.dq), gq, "accumulated dq")
        assert_close(host(e.m), m, "m"); assert_close(host(e.q), q, "q")


def test_step_pack_updated_equals_pack_after_step(F):
    """FOCUS_STEP_PACK_UPDATED: the step's codes and scales are bit for bit what
    focus_pack_multi writes after the step (the pack is checked against the
    oracle on generated inputs elsewhere); everything else is unchanged."""
    from fp4_post_weight_b200.table import FocusTable, hparams
    shapes = [(37, 1040), (64, 512), (128, 2048), (3, 48)]
    ea = _entries(shapes, 70)
    eb = _entries(shapes, 70)
    ta, tb = FocusTable(ea), FocusTable(eb)
    ta.s2(); tb.s2()
    ta.step(1, hparams(), flags=F.FOCUS_STEP_PACK_UPDATED)
    tb.step(1, hparams())
    tb.pack()
    assert F.focus_get_error() == 0
    for a, b in zip(ea, eb):
        for name in ("codes", "scales", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq"):
            assert torch.equal(getattr(a, name), getattr(b, name)), name
        assert np.array_equal(host_bits(a.Wq), host_bits(b.Wq))


def test_step_with_both_updated_outputs(F):
    """FOCUS_STEP_PACK_UPDATED | FOCUS_STEP_WQ_UPDATED together (the next step's W'
    and the export of the updated parameters from one pass): codes and scales are
    bit for bit focus_pack_multi after the step, W' is bit for bit focus_fwd_multi
    after the step, and m, q and the moments are those of the plain step."""
    from fp4_post_weight_b200.table import FocusTable, hparams
    shapes = [(37, 1040), (64, 512), (128, 2048), (3, 48), (0, 32)]
    ea, eb = _entries(shapes, 140, warm=True), _entries(shapes, 140, warm=True)
    ta, tb = FocusTable(ea), FocusTable(eb)
    ta.s2(); tb.s2()
    ta.step(3, hparams(), flags=F.FOCUS_STEP_PACK_UPDATED | F.FOCUS_STEP_WQ_UPDATED)
    tb.step(3, hparams())
    tb.pack()
    tb.fwd()
    assert F.focus_get_error() == 0
    for a, b in zip(ea, eb):
        for name in ("codes", "scales", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq"):
            assert torch.equal(getattr(a, name), getattr(b, name)), name
        assert np.array_equal(host_bits(a.Wq), host_bits(b.Wq))


@pytest.mark.parametrize("acc", [False, True])
@pytest.mark.parametrize("pack", [False, True])
@pytest.mark.parametrize("wqu", [False, True])
@pytest.mark.parametrize("amax", [False, True])
def test_step_kernels_for_fixed_options_match_the_runtime_one(F, acc, pack, wqu, amax):
    """The step runs in a kernel compiled for the caller's options where one
    exists (the export with or without the tensor maxima, either alone,
    neither, the accumulating step with W' of the update) and otherwise in the
    kernel that reads them at run time, which FOCUS_STEP_WRITE_GRAD always
    selects.  For every combination of the other options, both kernels leave
    bit-identical parameters, moments, W', codes, scales and tensor maxima from
    the same inputs (the run-time kernel is checked against the oracle by the
    tests above)."""
    from fp4_post_weight_b200.table import FocusTable, hparams
    shapes = [(37, 1040), (64, 512), (3, 48), (0, 32), (9, 4096)]
    flags = ((F.FOCUS_STEP_ACCUMULATE if acc else 0) | (F.FOCUS_STEP_PACK_UPDATED if pack else 0)
             | (F.FOCUS_STEP_WQ_UPDATED if wqu else 0))
    ea, eb = _entries(shapes, 210, warm=True), _entries(shapes, 210, warm=True)
    g = torch.Generator(device="cuda").manual_seed(11)
    for a, b in zip(ea, eb):
        a.dm.copy_(synth.normal(a.dm.shape, 0, 1e-5, g, "cuda")); b.dm.copy_(a.dm)
        a.dq.copy_(synth.normal(a.dq.shape, 0, 1e-7, g, "cuda")); b.dq.copy_(a.dq)
    ta, tb = FocusTable(ea), FocusTable(eb)
    ta.s2(); tb.s2()
    wa = torch.zeros(8, dtype=torch.int32, device="cuda")
    wb = torch.zeros(8, dtype=torch.int32, device="cuda")
    hp = hparams()
    if amax:
        F.focus_step_fused_amax(ta.dev, ta.n, ta.total_tiles, hp, 4, wa, flags)
        F.focus_step_fused_amax(tb.dev, tb.n, tb.total_tiles, hp, 4, wb, flags | F.FOCUS_STEP_WRITE_GRAD)
    else:
        ta.step(4, hp, flags)
        tb.step(4, hp, flags | F.FOCUS_STEP_WRITE_GRAD)
    assert F.focus_get_error() == 0
    assert torch.equal(wa, wb)
    if amax:
        assert int(wa[:5].ne(0).sum()) == 4            # every non-empty tensor got its maximum
    for a, b in zip(ea, eb):
        for name in ("codes", "scales", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq"):
            assert torch.equal(getattr(a, name), getattr(b, name)), name
        assert np.array_equal(host_bits(a.Wq), host_bits(b.Wq))


def _outside_fast_range_entries(seed):
    """Entries whose blocks leave the step's fast range in each way it has:
    logits above 80 (the direct sigmoid; sigma rounds to 1), logits near -50
    (sigma ~ 2^-72, so D = S*sigma*s2 is normal but below 2^-60: the IEEE
    quotient), a tensor whose weights reach 2^60 (A > 2^60), next to ordinary
    blocks in the same warps."""
    ents = _entries([(64, 512), (48, 256)], seed, warm=True)
    e0, e1 = ents
    g = torch.Generator(device="cuda").manual_seed(seed)
    q = e0.q
    q[0:2] = torch.where(torch.rand(q[0:2].shape, generator=g, device="cuda") < 0.5, 95.0, 110.0)
    q[2:4, ::3] = 81.5
    q[4:8] = synth.normal(q[4:8].shape, -50.0, 2.0, g, "cuda")
    e1.W.copy_((e1.W.float() * 2.0 ** 66).to(torch.bfloat16))      # |w| ~ 0.02 * 2^66 > 2^60
    return ents


def test_step_blocks_outside_the_fast_range(F):
    """Warps with a block outside the fast range take the general code: the
    forward (W', codes, scales) bit for bit the oracle's outside the rounding
    band, m, q and the moments within tolerance, through the kernel compiled for
    the plain step.  The gradients of the 2^66-scaled tensor are 2^66 times an
    ordinary tensor's, so its moments are compared in units of 2^66 (2^132 for
    the second moments), where the tolerances mean what they do elsewhere."""
    from fp4_post_weight_b200.table import FocusTable, hparams
    ents = _outside_fast_range_entries(230)
    host_in = [(host_bits(e.W), host_bits(e.dWq), host(e.m).copy(), host(e.q).copy(),
                [host(x).copy() for x in (e.m_exp_avg, e.m_exp_avg_sq, e.q_exp_avg, e.q_exp_avg_sq)])
               for e in ents]
    tab = FocusTable(ents)
    tab.s2()
    tab.step(3, hparams())
    assert F.focus_get_error() == 0
    for e, (Wb, Gb, m, q, st), f in zip(ents, host_in, (1.0, 2.0 ** 66)):
        s2 = oracle.s2(Wb)
        ref_f = oracle.fwd(Wb, m, q, s2)
        mism = check_forward(ref_f, Wq=host_bits(e.Wq), codes=unpack_codes(host(e.codes)), scales=host(e.scales))
        skip = block_mask(mism)
        skq = np.repeat(skip, 2, axis=1)
        oracle.step(Wb, Gb, m, q, *st, s2, 3, want_wq=False)
        assert_close(host(e.m), m, "m", skip)
        assert_close(host(e.q), q, "q", skq)
        d64 = lambda x: np.asarray(x, np.float64)              # 2^132 does not fit binary32
        assert_close(d64(host(e.m_exp_avg)) / f, d64(st[0]) / f, "m exp_avg", skip)
        assert_close(d64(host(e.m_exp_avg_sq)) / f ** 2, d64(st[1]) / f ** 2, "m exp_avg_sq", skip)
        assert_close(d64(host(e.q_exp_avg)) / f, d64(st[2]) / f, "q exp_avg", skq)
        assert_close(d64(host(e.q_exp_avg_sq)) / f ** 2, d64(st[3]) / f ** 2, "q exp_avg_sq", skq)


def test_step_export_outside_the_fast_range(F):
    """The same blocks with FOCUS_STEP_PACK_UPDATED (and the tensor maxima): the
    exported codes and scales are bit for bit what focus_pack_multi writes after
    a plain step, and W' of the forward and the parameters agree bit for bit."""
    from fp4_post_weight_b200.table import FocusTable, hparams
    ea, eb = _outside_fast_range_entries(240), _outside_fast_range_entries(240)
    ta, tb = FocusTable(ea), FocusTable(eb)
    ta.s2(); tb.s2()
    ta.step_s2(2, hparams(), F.FOCUS_STEP_PACK_UPDATED)
    tb.step(2, hparams())
    tb.pack()
    assert F.focus_get_error() == 0
    for a, b in zip(ea, eb):
        for name in ("codes", "scales", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq"):
            assert torch.equal(getattr(a, name), getattr(b, name)), name
        assert np.array_equal(host_bits(a.Wq), host_bits(b.Wq))


def test_round_to_nearest_weights_outside_the_fast_range(F):
    """Plain NVFP4 round to nearest of weights (its kernel takes the fast code
    for a warp whose blocks are all in range, else the general one): a tensor
    with blocks of 2^61-sized weights next to ordinary ones, and a tensor scale
    outside the fast range, bit for bit the oracle's RTN."""
    from fp4_post_weight_b200.table import PURPOSE_FOUROVERSIX, Entry, FocusTable
    g = torch.Generator(device="cuda").manual_seed(250)
    W0 = synth.normal_bf16((64, 512), 0.02, g, "cuda")
    W0[::7] = (W0[::7].float() * 2.0 ** 66).to(torch.bfloat16)      # some rows far above the rest
    W1 = (synth.normal_bf16((16, 256), 0.02, g, "cuda").float() * 2.0 ** -110).to(torch.bfloat16)  # tiny s2
    ents = [Entry(W=W, m=None, q=None, s2=torch.zeros(1, device="cuda"),
                  codes=torch.empty((W.shape[0], W.shape[1] // 2), dtype=torch.uint8, device="cuda"),
                  scales=torch.empty((W.shape[0], W.shape[1] // 16), dtype=torch.uint8, device="cuda"))
            for W in (W0, W1)]
    tab = FocusTable(ents, PURPOSE_FOUROVERSIX)
    tab.s2()
    tab.nvfp4_rtn()
    assert F.focus_get_error() == 0
    for e in ents:
        Wb = host_bits(e.W)
        s2 = oracle.s2(Wb)
        ref = oracle.fwd(Wb, np.ones((Wb.shape[0], Wb.shape[1] // 16), np.float32),
                         np.full((Wb.shape[0], Wb.shape[1] // 8), 30.0, np.float32), s2)
        np.testing.assert_array_equal(host(e.scales), ref.scales)
        np.testing.assert_array_equal(unpack_codes(host(e.codes)), ref.codes)


def test_pack_multi_leaves_wq_alone(F):
    from fp4_post_weight_b200.table import FocusTable
    ents = _entries([(16, 256)], 60)
    for e in ents:
        e.Wq.fill_(3.0)
    tab = FocusTable(ents)
    tab.s2()
    tab.pack()
    torch.cuda.synchronize()
    assert bool((ents[0].Wq == 3.0).all())


def test_worked_example_on_gpu(F):
    here = os.path.dirname(os.path.abspath(__file__))
    gold = json.load(open(os.path.join(here, "golden", "worked_block.json")))
    Wf = torch.tensor(gold["W"], dtype=torch.float32)
    W = Wf.to(torch.bfloat16).cuda()
    assert torch.equal(W.float().cpu(), Wf)
    m = torch.tensor(gold["m"], dtype=torch.float32).cuda()
    q = torch.tensor(gold["q"], dtype=torch.float32).cuda()
    ex = gold["expected"]
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    s2 = torch.zeros(1, device="cuda")
    F.focus_s2(W, s2, ws)
    assert host(s2)[0] == np.float32(ex["s2"])
    Wq = torch.empty_like(W)
    F.focus_fwd(W, m, q, ex["s2"], Wq)
    want = torch.tensor(ex["Wq"], dtype=torch.float32).to(torch.bfloat16)
    assert np.array_equal(host_bits(Wq), host_bits(want))
    for r, c in ex["negative_zero_Wq"]:
        assert host_bits(Wq)[r, c] == 0x8000
    codes = torch.empty((2, 16), dtype=torch.uint8, device="cuda")
    scales = torch.empty((2, 2), dtype=torch.uint8, device="cuda")
    F.focus_pack_nvfp4(W, m, q, ex["s2"], codes, scales, torch.zeros(1, device="cuda"))
    np.testing.assert_array_equal(unpack_codes(host(codes)), np.array(ex["codes"], np.uint8))
    np.testing.assert_array_equal(host(scales), np.array(ex["scales"], np.uint8))
    ones = torch.ones_like(W)
    dm = torch.empty((2, 2), device="cuda"); dq = torch.empty((2, 4), device="cuda")
    F.focus_ste_bwd(W, ones, m, q, ex["s2"], dm, dq)
    np.testing.assert_array_equal(host(dm), np.array(ex["dm"], np.float32))
    np.testing.assert_array_equal(host(dq), np.array(ex["dq"], np.float32))


def test_codec_sweep(F):
    """E4M3 and E2M1 decisions on crafted blocks: x on every E4M3 midpoint and
    its neighbours (A = 0.375 = 6*s2 with s2 = 2^-4, so x = fl(0.375*m)/0.375),
    plus E2M1 ties and signed zeros through y = w/D."""
    mids = []
    for b in range(0x08, 0x7E):
        e, mn = (b >> 3) & 15, b & 7
        v = (1 + mn / 8) * 2.0 ** (e - 7)
        e2, mn2 = (e, mn + 1) if mn < 7 else (e + 1, 0)
        v2 = (1 + mn2 / 8) * 2.0 ** (e2 - 7)
        mids.append((v + v2) / 2)
    xs = []
    for x in mids:
        x32 = np.float32(x)
        xs += [x32, np.nextafter(x32, np.float32(0)), np.nextafter(x32, np.float32(1e9))]
    rng = np.random.default_rng(0)
    xs += list(np.exp2(rng.uniform(-8, 10, 20000)).astype(np.float32))
    n = len(xs)
    m = torch.tensor(np.array(xs, np.float32)).view(n, 1).cuda()
    Wf = torch.zeros(n, 16)
    Wf[:, 0] = 0.375
    tvals = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.0, 0.1, -0.1, 6.0, 7.0, -7.0, 3.0]
    W = Wf.to(torch.bfloat16).cuda()
    q = torch.zeros((n, 2), device="cuda")
    s2 = 2.0 ** -4
    codes = torch.empty((n, 8), dtype=torch.uint8, device="cuda")
    scales = torch.empty((n, 1), dtype=torch.uint8, device="cuda")
    F.focus_pack_nvfp4(W, m, q, s2, codes, scales, torch.zeros(1, device="cuda"))
    ref = oracle.fwd(host_bits(W), host(m), host(q), s2)
    np.testing.assert_array_equal(host(scales), ref.scales)
    # E2M1: elements t * D for every block scale reached above (D = S * 0.5 * s2)
    S = np.array([oracle.e4m3_decode(int(b)) for b in ref.scales[:, 0]], np.float64)
    D = S * 0.5 * s2
    for j, t in enumerate(tvals):
        val = np.float32(t) * D.astype(np.float32)
        Wf[:, 1 + j] = torch.tensor(val)
    W2 = Wf.to(torch.bfloat16).cuda()
    F.focus_pack_nvfp4(W2, m, q, s2, codes, scales, torch.zeros(1, device="cuda"))
    Wq = torch.empty_like(W2)
    F.focus_fwd(W2, m, q, s2, Wq)
    ref2 = oracle.fwd(host_bits(W2), host(m), host(q), s2)
    np.testing.assert_array_equal(host(scales), ref2.scales)
    np.testing.assert_array_equal(unpack_codes(host(codes)), ref2.codes)
    np.testing.assert_array_equal(host_bits(Wq), ref2.Wq)


def test_nonfinite_input_sets_flag(F):
    W, m, q, _ = make((4, 64), 5)
    W[1, 7] = float("nan")
    Wq = torch.empty_like(W)
    assert F.focus_get_error() == 0
    F.focus_fwd(W, m, q, 1e-4, Wq)
    assert F.focus_get_error() == F.FOCUS_OK + 7
    assert F.focus_get_error() == 0          # cleared
    W[1, 7] = 0.0
    m[0, 0] = float("inf")
    F.focus_fwd(W, m, q, 1e-4, Wq)
    assert F.focus_get_error() == 7


@pytest.mark.parametrize("accumulate", [False, True])
def test_fwd_and_bwd_multi(F, accumulate):
    """The one-launch forward and straight-through backward over a table."""
    from fp4_post_weight_b200.table import FocusTable, PURPOSE_BACKWARD
    shapes = SHAPES + [(0, 32)]
    ents = _entries(shapes, 80)
    g = torch.Generator(device="cuda").manual_seed(8)
    if accumulate:
        for e in ents:
            e.dm.copy_(synth.normal(e.dm.shape, 0, 1e-5, g, "cuda"))
            e.dq.copy_(synth.normal(e.dq.shape, 0, 1e-7, g, "cuda"))
    host_in = [(host_bits(e.W), host_bits(e.dWq), host(e.m).copy(), host(e.q).copy(), host(e.dm).copy(),
                host(e.dq).copy()) for e in ents]
    tab = FocusTable(ents, PURPOSE_BACKWARD)
    tab.s2()
    tab.fwd()
    tab.bwd(accumulate=accumulate)
    assert F.focus_get_error() == 0
    for e, (Wb, Gb, m, q, dm0, dq0) in zip(ents, host_in):
        if Wb.size == 0:
            continue
        s2 = oracle.s2(Wb)
        ref = oracle.fwd(Wb, m, q, s2)
        mism = check_forward(ref, Wq=host_bits(e.Wq), codes=unpack_codes(host(e.codes)), scales=host(e.scales))
        skip = block_mask(mism)
        if accumulate:
            rdm, rdq = oracle.ste_bwd(Wb, Gb, m, q, s2, dm=dm0, dq=dq0)
        else:
            rdm, rdq = oracle.ste_bwd(Wb, Gb, m, q, s2)
        assert_close(host(e.dm), rdm, "dm", skip)
        assert_close(host(e.dq), rdq, "dq", np.repeat(skip, 2, axis=1))
        assert np.array_equal(host(e.m), m) and np.array_equal(host(e.q), q)


def test_micro_batch_step(F):
    """A calibration step over four micro-batches (gradient accumulation, as the
    card's calibration runs it): W' of the current m and q from the table
    forward, the straight-through gradients of micro-batches 1-3 summed into
    dm/dq, then the fused step adds micro-batch 4, updates m and q, and with
    FOCUS_STEP_WQ_UPDATED writes the next step's W' in the same pass."""
    from fp4_post_weight_b200.table import FocusTable, hparams
    shapes = [(37, 1040), (64, 512), (128, 2048), (3, 48)]
    ents = _entries(shapes, 90, with_pack=False)
    g = torch.Generator(device="cuda").manual_seed(9)
    grads = [[synth.normal_bf16(e.W.shape, 1e-3, g, "cuda") for _ in range(4)] for e in ents]
    host_in = [(host_bits(e.W), host(e.m).copy(), host(e.q).copy(), [host_bits(x) for x in gs])
               for e, gs in zip(ents, grads)]
    tab = FocusTable(ents)
    tab.s2()
    tab.fwd()
    torch.cuda.synchronize()
    for e, (Wb, m, q, _) in zip(ents, host_in):
        check_forward(oracle.fwd(Wb, m, q, oracle.s2(Wb)), Wq=host_bits(e.Wq))
    for j in range(3):
        for e, gs in zip(ents, grads):
            e.dWq.copy_(gs[j])
        tab.bwd(accumulate=j > 0)
    for e, gs in zip(ents, grads):
        e.dWq.copy_(gs[3])
    tab.step(1, hparams(), flags=F.FOCUS_STEP_ACCUMULATE | F.FOCUS_STEP_WRITE_GRAD | F.FOCUS_STEP_WQ_UPDATED)
    assert F.focus_get_error() == 0
    wq_next = [e.Wq.clone() for e in ents]
    for e, (Wb, m, q, Gs) in zip(ents, host_in):
        s2 = oracle.s2(Wb)
        skip = block_mask(check_forward(oracle.fwd(Wb, m, q, s2)))
        dm, dq = oracle.ste_bwd(Wb, Gs[0], m, q, s2)
        for j in (1, 2):
            oracle.ste_bwd(Wb, Gs[j], m, q, s2, dm=dm, dq=dq)
        z = [np.zeros_like(m), np.zeros_like(m), np.zeros_like(q), np.zeros_like(q)]
        _, gm, gq = oracle.step(Wb, Gs[3], m, q, *z, s2, 1, want_wq=False, dm_acc=dm, dq_acc=dq)
        skq = np.repeat(skip, 2, axis=1)
        assert_close(host(e.dm), gm, "dm over four micro-batches", skip)
        assert_close(host(e.dq), gq, "dq over four micro-batches", skq)
        assert_close(host(e.m), m, "m", skip)
        assert_close(host(e.q), q, "q", skq)
        for name, want, sk in zip(("m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq"), z,
                                  (skip, skip, skq, skq)):
            assert_close(host(getattr(e, name)), want, name, sk)
    # the step's W' is bit for bit the table forward of the updated m and q
    tab.fwd()
    assert F.focus_get_error() == 0
    for e, w in zip(ents, wq_next):
        assert torch.equal(e.Wq.view(torch.int16), w.view(torch.int16))


def test_step_with_s2_for_the_next_step(F):
    """focus_step_fused_amax + focus_s2_from_amax: the step's outputs are bit for
    bit those of focus_step_fused, and afterwards every desc.s2 equals the oracle's
    s2 of its W (W is frozen), so the next step reads the same s2 a separate
    focus_s2_multi pass would give; two steps in a row agree with the plain path."""
    from fp4_post_weight_b200.table import FocusTable, hparams
    shapes = SHAPES + [(0, 32)]
    ea, eb = _entries(shapes, 95), _entries(shapes, 95)
    ta, tb = FocusTable(ea), FocusTable(eb)
    ta.s2(); tb.s2()
    for t in (1, 2):
        ta.step_s2(t, hparams(), flags=F.FOCUS_STEP_PACK_UPDATED)
        tb.s2()
        tb.step(t, hparams(), flags=F.FOCUS_STEP_PACK_UPDATED)
        assert F.focus_get_error() == 0
        for a, b in zip(ea, eb):
            for name in ("Wq", "codes", "scales", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq"):
                x, y = getattr(a, name), getattr(b, name)
                assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), (t, name)
            want = oracle.s2(host_bits(a.W)) if a.W.numel() else np.float32(0)
            assert host(a.s2)[0] == want and host(b.s2)[0] == want
    assert int(ta._amax.abs().sum()) == 0          # cleared for the next step


def test_step_skips_an_all_zero_tensor_and_reports_it(F):
    """A tensor whose W is all zero has s2 = 0, which the method cannot divide by:
    the table step leaves that entry untouched and sets the device flag
    (FOCUS_ERR_NONFINITE_INPUT); the other entries are stepped exactly as in a
    table without it, and the tensor maximum leaves s2 = 0 for the zero tensor."""
    from fp4_post_weight_b200.table import FocusTable, hparams
    shapes = [(37, 1040), (64, 256), (7, 4112)]
    ea, eb = _entries(shapes, 120), _entries(shapes, 120)
    ea[1].W.zero_()
    m_before = ea[1].m.clone()
    q_before = ea[1].q.clone()
    ta, tb = FocusTable(ea), FocusTable([eb[0], eb[2]])
    ta.s2(); tb.s2()
    assert F.focus_get_error() == 0
    assert host(ea[1].s2)[0] == 0.0
    ta.step_s2(1, hparams(), flags=F.FOCUS_STEP_PACK_UPDATED)
    assert F.focus_get_error() == 7
    assert F.focus_get_error() == 0                 # cleared
    tb.step_s2(1, hparams(), flags=F.FOCUS_STEP_PACK_UPDATED)
    assert F.focus_get_error() == 0
    assert torch.equal(ea[1].m, m_before) and torch.equal(ea[1].q, q_before)
    assert host(ea[1].s2)[0] == 0.0
    for a, b in ((ea[0], eb[0]), (ea[2], eb[2])):
        for name in ("Wq", "codes", "scales", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq", "s2"):
            x, y = getattr(a, name), getattr(b, name)
            assert torch.equal(x.view(torch.uint8), y.view(torch.uint8)), name


def test_step_on_a_table_without_moments_is_skipped_and_reported(F):
    """A table prepared for the forward (purpose 0: no AdamW moments) handed to the
    step: the kernel meets entries lacking pointers it needs, skips them without
    dereferencing anything and sets the device flag; nothing is written."""
    from fp4_post_weight_b200.table import PURPOSE_FORWARD, Entry, FocusTable, hparams
    W, m, q, dW = make((37, 1040), 130)
    e = Entry(W=W, m=m, q=q, s2=torch.zeros(1, device="cuda"), dWq=dW, Wq=torch.zeros_like(W))
    tab = FocusTable([e], PURPOSE_FORWARD)
    tab.s2()
    assert F.focus_get_error() == 0
    m0, q0 = m.clone(), q.clone()
    tab.step(1, hparams())
    assert F.focus_get_error() == 7
    assert torch.equal(m, m0) and torch.equal(q, q0)
    assert not e.Wq.view(torch.int16).any()
