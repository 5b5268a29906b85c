"""GPU parity of the FourOverSix quantizer against the oracle, bit for bit:
weights with a tensor scale (single tensor and multi-tensor table, shapes
spanning several 4096-weight tiles and ragged tails), activations with one
scale per token (rows of one and of several blocks per thread, a zero row),
the hand-derived worked example, blocks whose two targets tie with a nonzero
error, and the non-finite flag.  The E4M3 and E2M1 decisions are taken in
binary32 on both sides and must match exactly; the target choice is the exact
order of the two squared errors in the oracle, and a kernel block may differ
from it only inside the 2^-47 band of tests/parity.py (none is expected)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity import check_fouroversix, host, host_bits, unpack_codes

pytestmark = pytest.mark.gpu

SHAPES = [(1, 16), (3, 48), (2, 4096), (37, 1040), (7, 4112), (128, 2048), (257, 160)]
HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def F():
    from fp4_post_weight_b200 import focus
    return focus


def weights(shape, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    W = synth.add_outliers(synth.normal_bf16(shape, 0.02, g, "cuda"), 2e-3, 20.0, g)
    if W.numel() >= 64:
        W.view(-1)[:16] = 0
    return W


def outputs(o, i, dev="cuda"):
    return (torch.empty((o, i // 2), dtype=torch.uint8, device=dev),
            torch.empty((o, i // 16), dtype=torch.uint8, device=dev),
            torch.empty((o, i), dtype=torch.bfloat16, device=dev))


def assert_same(ref, codes, scales, Xq):
    if ref.errs is not None:        # FourOverSix: the choice may differ only inside the band
        c = check_fouroversix(ref, unpack_codes(host(codes)), host(scales), host_bits(Xq))
        assert c["mismatched_blocks"] == 0, c
        return c
    np.testing.assert_array_equal(host(scales), ref.scales)
    np.testing.assert_array_equal(unpack_codes(host(codes)), ref.codes)
    np.testing.assert_array_equal(host_bits(Xq), ref.Xq)


@pytest.mark.parametrize("shape", SHAPES)
def test_weight(F, shape):
    W = weights(shape, 20 + shape[0])
    Wb = host_bits(W)
    s2 = oracle.s2(Wb)
    codes, scales, Wq = outputs(*shape)
    F.focus_fouroversix_weight(W, float(s2), codes, scales, Wq)
    assert F.focus_get_error() == 0
    ref = oracle.fouroversix(Wb, s2)
    assert_same(ref, codes, scales, Wq)
    if W.numel() >= 4096:
        assert 0 < ref.four.mean() < 1


def test_weight_outputs_optional(F):
    W = weights((64, 512), 3)
    Wb = host_bits(W)
    s2 = oracle.s2(Wb)
    ref = oracle.fouroversix(Wb, s2)
    codes, scales, Wq = outputs(64, 512)
    F.focus_fouroversix_weight(W, float(s2), codes, scales, None)
    Wq.fill_(7.0)
    F.focus_fouroversix_weight(W, float(s2), None, None, Wq)
    assert F.focus_get_error() == 0
    assert_same(ref, codes, scales, Wq)


def test_weight_table(F):
    from fp4_post_weight_b200.table import Entry, FocusTable, PURPOSE_FOUROVERSIX
    shapes = SHAPES + [(0, 32)]
    ents = []
    for j, sh in enumerate(shapes):
        W = weights(sh, 40 + j) if sh[0] * sh[1] else torch.zeros(sh, dtype=torch.bfloat16, device="cuda")
        c, s, q = outputs(*sh)
        ents.append(Entry(W=W, m=None, q=None, s2=torch.zeros(1, device="cuda"), codes=c, scales=s, Wq=q))
    tab = FocusTable(ents, PURPOSE_FOUROVERSIX)
    tab.s2()
    tab.fouroversix()
    assert F.focus_get_error() == 0
    for e in ents:
        if e.W.numel() == 0:
            continue
        Wb = host_bits(e.W)
        s2 = oracle.s2(Wb)
        assert host(e.s2)[0] == s2
        assert_same(oracle.fouroversix(Wb, s2), e.codes, e.scales, e.Wq)


def _rtn_ref(Wb, s2):
    """The oracle's forward with m = 1 and sigmoid(q) = 1 (q = 30): plain NVFP4 RTN."""
    o, i = Wb.shape
    return oracle.fwd(Wb, np.ones((o, i // 16), np.float32), np.full((o, i // 8), 30.0, np.float32), s2)


@pytest.mark.parametrize("shape", SHAPES)
def test_nvfp4_weight(F, shape):
    """Plain NVFP4 round to nearest of weights (focus_nvfp4_weight) against the
    oracle's forward with unit parameters, bit for bit; outputs optional."""
    W = weights(shape, 60 + shape[0])
    Wb = host_bits(W)
    s2 = oracle.s2(Wb)
    codes, scales, Wq = outputs(*shape)
    F.focus_nvfp4_weight(W, float(s2), codes, scales, Wq)
    assert F.focus_get_error() == 0
    ref = _rtn_ref(Wb, s2)
    np.testing.assert_array_equal(host(scales), ref.scales)
    np.testing.assert_array_equal(unpack_codes(host(codes)), ref.codes)
    np.testing.assert_array_equal(host_bits(Wq), ref.Wq)
    Wq2 = torch.full_like(Wq, 7.0)
    F.focus_nvfp4_weight(W, float(s2), None, None, Wq2)
    assert F.focus_get_error() == 0 and torch.equal(Wq2.view(torch.int16), Wq.view(torch.int16))


def test_nvfp4_weight_table(F):
    from fp4_post_weight_b200.table import Entry, FocusTable, PURPOSE_FOUROVERSIX
    shapes = SHAPES + [(0, 32)]
    ents = []
    for j, sh in enumerate(shapes):
        W = weights(sh, 80 + j) if sh[0] * sh[1] else torch.zeros(sh, dtype=torch.bfloat16, device="cuda")
        c, s, q = outputs(*sh)
        ents.append(Entry(W=W, m=None, q=None, s2=torch.zeros(1, device="cuda"), codes=c, scales=s, Wq=q))
    tab = FocusTable(ents, PURPOSE_FOUROVERSIX)
    tab.s2()
    tab.nvfp4_rtn()
    assert F.focus_get_error() == 0
    for e in ents:
        if e.W.numel() == 0:
            continue
        Wb = host_bits(e.W)
        ref = _rtn_ref(Wb, oracle.s2(Wb))
        np.testing.assert_array_equal(host(e.scales), ref.scales)
        np.testing.assert_array_equal(unpack_codes(host(e.codes)), ref.codes)
        np.testing.assert_array_equal(host_bits(e.Wq), ref.Wq)


@pytest.mark.parametrize("tokens,hidden", [(1, 16), (5, 48), (33, 4096), (17, 14336), (300, 1040), (3, 64),
                                           (3, 262144)])
def test_activations(F, tokens, hidden):
    X = synth.activations(tokens, hidden, "cuda", seed=tokens + hidden, zero_tokens=1 if tokens > 2 else 0)
    ts = torch.full((tokens,), -1.0, device="cuda")
    codes, scales, Xq = outputs(tokens, hidden)
    F.focus_fouroversix_act(X, ts, codes, scales, Xq)
    assert F.focus_get_error() == 0
    ref = oracle.fouroversix(host_bits(X))
    np.testing.assert_array_equal(host(ts), ref.row_scales)
    assert_same(ref, codes, scales, Xq)
    if tokens > 2:
        assert host(ts)[-1] == 0 and np.all(host(scales)[-1] == 0x38)


@pytest.mark.parametrize("tokens,hidden", [(1, 16), (5, 48), (33, 4096), (17, 14336), (300, 1040), (3, 64),
                                           (3, 262144)])
def test_nvfp4_activations(F, tokens, hidden):
    """Plain NVFP4 round to nearest per token (focus_nvfp4_act) against the oracle's
    fo_nvfp4_rows, bit for bit; one row carries a block far below the row maximum
    (the lower scale clamp) when the shape allows."""
    X = synth.activations(tokens, hidden, "cuda", seed=3 * tokens + hidden, zero_tokens=1 if tokens > 2 else 0)
    if tokens > 1 and hidden >= 64:
        X[0, 16:32] = 1e-4
        X[0, 40] = 40.0
    ts = torch.full((tokens,), -1.0, device="cuda")
    codes, scales, Xq = outputs(tokens, hidden)
    F.focus_nvfp4_act(X, ts, codes, scales, Xq)
    assert F.focus_get_error() == 0
    ref = oracle.nvfp4_rows(host_bits(X))
    np.testing.assert_array_equal(host(ts), ref.row_scales)
    assert_same(ref, codes, scales, Xq)
    if tokens > 1 and hidden >= 64:
        assert host(scales)[0, 1] == 0x08               # x below 2^-6: clamped to the smallest normal scale


@pytest.mark.parametrize("swizzled", [False, True], ids=["row-major", "128x4"])
@pytest.mark.parametrize("rtn", [False, True], ids=["fouroversix", "nvfp4"])
def test_activation_table_one_launch(F, rtn, swizzled):
    """Activation tensors of mixed widths in one launch (focus_*_act_multi): a zero
    row, rows of one block, ragged widths, an empty tensor, a token count not a
    multiple of 128 (padding rows of the 128x4 layout), the widest staged row, and
    bundles of several rows ending short of a full bundle; every tensor against the
    oracle (row scales, scale bytes, codes, X')."""
    from fp4_post_weight_b200.table import ActTable, act_entry
    shapes = [(33, 4096), (5, 48), (0, 64), (130, 1040), (17, 14336), (3, 16), (7, 16384)]
    ents, Xs = [], []
    for j, (t, h) in enumerate(shapes):
        X = synth.activations(t, h, "cuda", seed=90 + j, zero_tokens=1 if t > 2 else 0) if t else \
            torch.zeros((0, h), dtype=torch.bfloat16, device="cuda")
        nsc = F.focus_scales_swizzled_bytes(t, h // 16) if swizzled else t * (h // 16)
        ents.append(act_entry(X, torch.full((max(t, 1),), -1.0, device="cuda"),
                              torch.empty((max(t, 1), h // 2), dtype=torch.uint8, device="cuda"),
                              torch.full((max(nsc, 16),), 0xAB, dtype=torch.uint8, device="cuda"),
                              torch.empty_like(X) if t else None))
        Xs.append(X)
    tab = ActTable(ents, swizzled=swizzled)

    def bundles(rows, nb):            # rows per bundle: 256 threads, at most 4 blocks per thread
        tpr = 32
        while tpr < 256 and 4 * tpr < nb:
            tpr *= 2
        return -(-rows // (256 // tpr))
    assert tab.total_rows == sum(bundles((t + 127) // 128 * 128 if swizzled else t, h // 16) for t, h in shapes if t)
    tab.nvfp4() if rtn else tab.fouroversix()
    assert F.focus_get_error() == 0
    for (t, h), X, e in zip(shapes, Xs, ents):
        if t == 0:
            continue
        ref = oracle.nvfp4_rows(host_bits(X)) if rtn else oracle.fouroversix(host_bits(X))
        np.testing.assert_array_equal(host(e.s2)[:t], ref.row_scales)
        codes = unpack_codes(host(e.codes))
        if swizzled:
            nsc = F.focus_scales_swizzled_bytes(t, h // 16)
            np.testing.assert_array_equal(host(e.scales)[:nsc], oracle.scales_swizzle(ref.scales))
            lin = None
        else:
            lin = host(e.scales)[:t * (h // 16)].reshape(t, h // 16)
        if rtn:
            np.testing.assert_array_equal(codes, ref.codes)
            np.testing.assert_array_equal(host_bits(e.Wq), ref.Xq)
            if lin is not None:
                np.testing.assert_array_equal(lin, ref.scales)
        else:
            sc = lin if lin is not None else ref.scales      # the 128x4 bytes were checked above
            c = check_fouroversix(ref, codes, sc, host_bits(e.Wq))
            assert c["mismatched_blocks"] == 0, c


def test_activation_table_rejects_and_flags(F):
    """A row holding infinity in a table sets the device flag and leaves that row
    unwritten while the other rows and tensors match the oracle; a table entry wider
    than max_hidden is skipped and flagged; shapes above 16384 values per row are
    refused by the table preparation."""
    from fp4_post_weight_b200.table import ActTable, act_entry
    Xa = synth.activations(9, 1024, "cuda", seed=5, zero_tokens=0)
    Xb = synth.activations(4, 2048, "cuda", seed=6, zero_tokens=0)
    Xa[4, 100] = float("inf")
    mk = lambda X: act_entry(X, torch.zeros(X.shape[0], device="cuda"),
                             torch.zeros((X.shape[0], X.shape[1] // 2), dtype=torch.uint8, device="cuda"),
                             torch.zeros((X.shape[0], X.shape[1] // 16), dtype=torch.uint8, device="cuda"))
    ents = [mk(Xa), mk(Xb)]
    tab = ActTable(ents)
    assert F.focus_get_error() == 0
    tab.fouroversix()
    assert F.focus_get_error() == 7
    good = [r for r in range(9) if r != 4]
    ref = oracle.fouroversix(host_bits(Xa)[good])
    np.testing.assert_array_equal(host(ents[0].scales)[good], ref.scales)
    assert not host(ents[0].scales)[4].any() and not host(ents[0].codes)[4].any()
    refb = oracle.fouroversix(host_bits(Xb))
    np.testing.assert_array_equal(host(ents[1].scales), refb.scales)
    # max_hidden below an entry's width: that entry is skipped and reported
    tab2 = ActTable([mk(Xb)])
    F.focus_fouroversix_act_multi(tab2.dev, 1, tab2.total_rows, 1024)
    assert F.focus_get_error() == 7
    with pytest.raises(F.FocusError):
        ActTable([mk(torch.zeros((2, 16400), dtype=torch.bfloat16, device="cuda"))])
    with pytest.raises(F.FocusError):
        F.focus_fouroversix_act_multi(tab.dev, 2, tab.total_rows, 16400)


def test_nvfp4_activations_swizzled_and_nonfinite(F):
    from tests.parity import unpack_codes as _unpack
    tokens, hidden = 130, 1040
    X = synth.activations(tokens, hidden, "cuda", seed=9)
    ts = torch.empty(tokens, device="cuda")
    codes = torch.empty((tokens, hidden // 2), dtype=torch.uint8, device="cuda")
    sw = torch.full((F.focus_scales_swizzled_bytes(tokens, hidden // 16),), 0xAB, dtype=torch.uint8, device="cuda")
    F.focus_nvfp4_act_swizzled(X, ts, codes, sw)
    assert F.focus_get_error() == 0
    ref = oracle.nvfp4_rows(host_bits(X))
    np.testing.assert_array_equal(host(sw), oracle.scales_swizzle(ref.scales))
    np.testing.assert_array_equal(_unpack(host(codes)), ref.codes)
    X[7, 3] = float("nan")
    codes2, scales2, _ = outputs(tokens, hidden)
    F.focus_nvfp4_act(X, ts, codes2, scales2)
    assert F.focus_get_error() == 7


def test_ties_with_nonzero_error_keep_six(F):
    """Blocks whose two targets have equal, nonzero exact squared errors (the
    oracle's pins check the ties with rationals): found by search with s = 1, the
    same scaled by 2^-12 with s = 2^-12 and in a per-token row whose maximum makes
    s_t a power of two, and blocks of the synthetic 8B weights with their tensor's
    s2 (tests/golden/fouroversix_ties.json).  The kernel's screen sends them to the
    exact comparison, and 6 is kept."""
    blocks = [(1.125, 0.25), (1.125, 1.0), (1.5, 0.875), (1.875, 1.75), (2.25, 2.0), (3.0, 0.625)]
    Wn = np.zeros((len(blocks), 32))
    Wn[:, 0] = [a for a, _ in blocks]
    Wn[:, 5] = [b for _, b in blocks]
    Wn[:, 16:] = Wn[:, :16] * -1.0
    for scale in (1.0, 2.0 ** -12):
        W = torch.tensor(Wn * scale, dtype=torch.float32).to(torch.bfloat16).cuda()
        Wb = host_bits(W)
        ref = oracle.fouroversix(Wb, np.float32(scale))
        assert np.all(ref.errs[..., 0] == ref.errs[..., 1]) and np.all(ref.errs > 0) and not ref.four.any()
        codes, scales, Wq = outputs(*W.shape)
        F.focus_fouroversix_weight(W, scale, codes, scales, Wq)
        assert F.focus_get_error() == 0
        assert_same(ref, codes, scales, Wq)
    # blocks of the synthetic 8B weights that tie exactly under their tensor's s2
    gold = json.load(open(os.path.join(HERE, "golden", "fouroversix_ties.json")))
    for b in gold["blocks"]:
        wb = np.array([[int(x, 16) for x in b["w_bits"]]], np.uint16)
        s2 = np.array([b["s2_bits"]], np.uint32).view(np.float32)[0]
        ref = oracle.fouroversix(wb, s2)
        assert ref.errs[0, 0, 0] == ref.errs[0, 0, 1] or not ref.four.any()
        W = torch.from_numpy(wb.view(np.int16)).cuda().view(torch.bfloat16)
        codes, scales, Wq = outputs(1, 16)
        F.focus_fouroversix_weight(W, float(s2), codes, scales, Wq)
        assert F.focus_get_error() == 0
        assert_same(ref, codes, scales, Wq)
    # per token: a leading block with maximum 2688 * 2^-12 gives s_t = 2^-12
    X = np.zeros((len(blocks), 48))
    X[:, 0] = 2688.0
    X[:, 16:] = Wn
    X = torch.tensor(X * 2.0 ** -12, dtype=torch.float32).to(torch.bfloat16).cuda()
    ref = oracle.fouroversix(host_bits(X))
    assert np.all(ref.row_scales == np.float32(2.0 ** -12)) and not ref.four.any()
    ts = torch.empty(X.shape[0], device="cuda")
    codes, scales, Xq = outputs(*X.shape)
    F.focus_fouroversix_act(X, ts, codes, scales, Xq)
    assert F.focus_get_error() == 0
    assert_same(ref, codes, scales, Xq)


def test_worked_example_on_gpu(F):
    gold = json.load(open(os.path.join(HERE, "golden", "fouroversix_worked.json")))
    u = gold["unit"]
    W = torch.tensor(np.array(gold["weights"]["W_over_u"]) * u, dtype=torch.float32).to(torch.bfloat16).cuda()
    codes, scales, Wq = outputs(*W.shape)
    F.focus_fouroversix_weight(W, u * gold["weights"]["s_over_u"], codes, scales, Wq)
    ex = gold["weights"]["expected"]
    np.testing.assert_array_equal(host(scales), np.array(ex["scales"], np.uint8))
    np.testing.assert_array_equal(unpack_codes(host(codes)), np.array(ex["codes"], np.uint8))
    assert torch.equal(Wq.view(torch.int16), W.view(torch.int16))
    X = torch.tensor(np.array(gold["tokens"]["X_over_u"]) * u, dtype=torch.float32).to(torch.bfloat16).cuda()
    ts = torch.empty(X.shape[0], device="cuda")
    codes, scales, Xq = outputs(*X.shape)
    F.focus_fouroversix_act(X, ts, codes, scales, Xq)
    ex = gold["tokens"]["expected"]
    np.testing.assert_array_equal(host(ts), np.array(ex["row_scales_over_u"], np.float32) * np.float32(u))
    np.testing.assert_array_equal(host(scales), np.array(ex["scales"], np.uint8))
    np.testing.assert_array_equal(unpack_codes(host(codes))[0], np.array(ex["codes_row0"], np.uint8))
    assert torch.equal(Xq.view(torch.int16), X.view(torch.int16))
    assert F.focus_get_error() == 0


def test_nonfinite_sets_flag(F):
    X = synth.activations(8, 64, "cuda", zero_tokens=0)
    X[3, 5] = float("inf")
    ts = torch.zeros(8, device="cuda")
    codes, scales, Xq = outputs(8, 64)
    assert F.focus_get_error() == 0
    F.focus_fouroversix_act(X, ts, codes, scales, Xq)
    assert F.focus_get_error() == 7
    W = weights((4, 64), 1)
    W[2, 9] = float("nan")
    F.focus_fouroversix_weight(W, 1e-4, codes[:4], scales[:4], None)
    assert F.focus_get_error() == 7
    assert F.focus_get_error() == 0
