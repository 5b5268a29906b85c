"""The fused step over tensors held in host memory (focus_step_host): the same
results, bit for bit, as the device-resident table step (focus_step_fused_amax +
focus_s2_from_amax) on the same inputs -- m, q, the four moments, W', the NVFP4
export and s2 -- over more tensors than the executor has device slots (slot
reuse), with an empty tensor, ragged tile tails, pinned and pageable buffers,
two consecutive steps, and s2 computed in the call; one tensor also against the
oracle directly."""
import pytest
import torch

import oracle
import synth
from tests.parity import assert_close, host, host_bits

pytestmark = pytest.mark.gpu

SHAPES = [(64, 256), (37, 1040), (0, 64), (3, 16), (256, 4096), (129, 528), (8, 14336), (1, 4096)]


@pytest.fixture(scope="module")
def F():
    from fp4_post_weight_b200 import focus
    return focus


def state(seed):
    """Per tensor: W, dW', m, q and warm moments (exp_avg_sq >= exp_avg^2), on the device."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    res = []
    for j, (o, i) in enumerate(SHAPES):
        W = synth.add_outliers(synth.normal_bf16((o, i), 0.02, g, "cuda"), 1e-3, 20.0, g) if o * i else \
            torch.empty((o, i), dtype=torch.bfloat16, device="cuda")
        G = synth.normal_bf16((o, i), 1e-3, g, "cuda") if o * i else torch.empty_like(W)
        m = synth.uniform((o, i // 16), 0.8, 1.2, g, "cuda")
        q = synth.normal((o, i // 8), 6.0, 2.0, g, "cuda")
        v1m, v1q = synth.normal(m.shape, 0, 1e-4, g, "cuda"), synth.normal(q.shape, 0, 1e-5, g, "cuda")
        mo = [v1m, v1m ** 2 + synth.normal(m.shape, 0, 1e-4, g, "cuda") ** 2,
              v1q, v1q ** 2 + synth.normal(q.shape, 0, 1e-5, g, "cuda") ** 2]
        res.append((W, G, m, q, mo))
    return res


def device_entries(st):
    from fp4_post_weight_b200.table import Entry
    ents = []
    for W, G, m, q, mo in st:
        o, i = W.shape
        ents.append(Entry(W=W, m=m.clone(), q=q.clone(), s2=torch.zeros(1, device="cuda"), dWq=G,
                          Wq=torch.empty_like(W), m_exp_avg=mo[0].clone(), m_exp_avg_sq=mo[1].clone(),
                          q_exp_avg=mo[2].clone(), q_exp_avg_sq=mo[3].clone(),
                          codes=torch.empty((o, i // 2), dtype=torch.uint8, device="cuda"),
                          scales=torch.empty((o, i // 16), dtype=torch.uint8, device="cuda")))
    return ents


def host_entries(st, pinned=True, s2=None):
    from fp4_post_weight_b200.table import Entry

    def h(t):
        c = t.cpu()
        return c.pin_memory() if pinned else c.clone()
    ents = []
    for j, (W, G, m, q, mo) in enumerate(st):
        o, i = W.shape
        ents.append(Entry(W=h(W), m=h(m), q=h(q), s2=h(torch.tensor([0.0 if s2 is None else s2[j]])), dWq=h(G),
                          Wq=h(torch.empty_like(W)), m_exp_avg=h(mo[0]), m_exp_avg_sq=h(mo[1]),
                          q_exp_avg=h(mo[2]), q_exp_avg_sq=h(mo[3]),
                          codes=h(torch.empty((o, i // 2), dtype=torch.uint8)),
                          scales=h(torch.empty((o, i // 16), dtype=torch.uint8))))
    return ents


FIELDS = ("m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq", "Wq", "codes", "scales", "s2")


def assert_same(dev_ents, host_ents, what):
    for j, (d, h) in enumerate(zip(dev_ents, host_ents)):
        for name in FIELDS:
            a, b = getattr(d, name).cpu(), getattr(h, name)
            assert torch.equal(a.view(torch.uint8) if a.numel() else a, b.view(torch.uint8) if b.numel() else b), \
                f"{what}: entry {j} {tuple(d.W.shape)} field {name} differs"


@pytest.mark.parametrize("pinned", [True, False])
def test_host_step_equals_device_step(F, pinned):
    from fp4_post_weight_b200.table import FocusTable, HostTable, hparams
    st = state(11)
    dev = device_entries(st)
    tab = FocusTable(dev)
    tab.s2()
    s2 = [float(e.s2.item()) for e in dev]
    hst = host_entries(st, pinned, s2)
    htab = HostTable(hst)
    for t in (1, 2):                                       # two consecutive steps
        tab.step_s2(t, hparams(), F.FOCUS_STEP_PACK_UPDATED)
        htab.step(t, hparams(), F.FOCUS_STEP_PACK_UPDATED)
        assert F.focus_get_error() == 0
        assert_same(dev, hst, f"step {t}, {'pinned' if pinned else 'pageable'}")


def test_host_step_computes_s2_first_and_matches_oracle(F):
    from fp4_post_weight_b200.table import FocusTable, HostTable, hparams
    st = state(12)
    hst = host_entries(st)                                 # s2 = 0 in host memory
    htab = HostTable(hst)
    htab.step(1, hparams(), F.FOCUS_HOST_S2_FIRST | F.FOCUS_STEP_WQ_UPDATED)
    assert F.focus_get_error() == 0
    for (W, _, _, _, _), e in zip(st, hst):
        if W.numel():
            assert e.s2.item() == float(oracle.s2(host_bits(W)))
    # the same as the device-resident step with W' of the update
    dev = device_entries(st)
    tab = FocusTable(dev)
    tab.s2()
    tab.step_s2(1, hparams(), F.FOCUS_STEP_WQ_UPDATED)
    assert F.focus_get_error() == 0
    assert_same(dev, hst, "s2 first, W' of the update")
    # one tensor against the oracle: the updated m and q
    W, G, m, q, mo = st[1]
    hm, hq = host(m).copy(), host(q).copy()
    hmo = [host(x).copy() for x in mo]
    s2 = oracle.s2(host_bits(W))
    oracle.step(host_bits(W), host_bits(G), hm, hq, *hmo, s2, 1, want_wq=False)
    assert_close(hst[1].m.numpy(), hm, "m")
    assert_close(hst[1].q.numpy(), hq, "q")


def test_host_step_both_updated_outputs_and_a_zero_tensor(F):
    """Both updated outputs (export and next W') through the host executor, with an
    all-zero tensor among the others and s2 computed in the call: that tensor's s2
    is 0, so the step skips it and sets the device flag; every other tensor matches
    the device-resident step bit for bit."""
    from fp4_post_weight_b200.table import FocusTable, HostTable, hparams
    st = state(13)
    W0 = st[1][0]
    W0.zero_()
    flags = F.FOCUS_STEP_PACK_UPDATED | F.FOCUS_STEP_WQ_UPDATED
    hst = host_entries(st)
    m_before = hst[1].m.clone()
    HostTable(hst).step(2, hparams(), F.FOCUS_HOST_S2_FIRST | flags)
    assert F.focus_get_error() == 7
    assert F.focus_get_error() == 0
    assert hst[1].s2.item() == 0.0 and torch.equal(hst[1].m, m_before)
    dev = device_entries(st)
    tab = FocusTable(dev)
    tab.s2()
    tab.step_s2(2, hparams(), flags)
    assert F.focus_get_error() == 7                  # the device-resident step skips it the same way
    keep = [j for j in range(len(SHAPES)) if j != 1]
    assert_same([dev[j] for j in keep], [hst[j] for j in keep], "both updated outputs")
