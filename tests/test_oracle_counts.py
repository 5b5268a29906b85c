"""Counts the pages print, the s2 definition, and the step as a composition.

* Model card "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct", "What this is":
  112 layers, 60,817,408 m values (one per 16-block), 121,634,816 q values
  (one per 8-element sub-block); "Files": focus.pt is 729,889,075 bytes.
* Card "Llama-3.1-8B-Instruct FlipQuant MixFP4 maps", tile table: 13,631,488
  8x64 tiles, 6,815,744 16x64 tiles and 425,984 256x64 tiles.
* s2 = amax(|W|)/(6*448) (field table, row s2).
"""
import numpy as np
import torch

import oracle
import synth

F = np.float32


def test_llama_1b_block_counts():
    t = synth.LLAMA_1B.tensors()
    assert len(t) == 112
    n = synth.LLAMA_1B.n_elements()
    assert n // 16 == 60_817_408 and n % 16 == 0
    assert n // 8 == 121_634_816
    # focus.pt: m and q as FP32 are 729,808,896 bytes; the file is 80,179 bytes larger
    assert 4 * (n // 16 + n // 8) == 729_808_896
    assert 0 < 729_889_075 - 729_808_896 < 100_000


def test_llama_8b_tile_counts():
    t = synth.LLAMA_8B.tensors()
    assert len(t) == 224
    assert all(o % 256 == 0 and i % 64 == 0 for _, (o, i) in t)
    n = synth.LLAMA_8B.n_elements()
    assert n // (8 * 64) == 13_631_488
    assert n // (16 * 64) == 6_815_744
    assert n // (256 * 64) == 425_984


def test_llama_70b_shapes():
    t = synth.LLAMA_70B.tensors()
    assert len(t) == 560
    # ~140 GB of bf16 for the whole model is dominated by these linears
    assert 130e9 < 2 * synth.LLAMA_70B.n_elements() < 141e9


def test_s2_is_amax_over_2688():
    assert 6 * 448 == 2688
    g = torch.Generator().manual_seed(5)
    W = (torch.randn(300, 64, generator=g) * 0.02).to(torch.bfloat16)
    W[17, 33] = -0.75
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    s2 = oracle.s2(Wb)
    assert s2 == F(0.75) / F(2688)
    assert oracle.s2(np.zeros(32, np.uint16)) == 0.0


def test_step_is_fwd_then_bwd_then_adamw():
    g = torch.Generator().manual_seed(8)
    W = (torch.randn(64, 96, generator=g) * 0.02).to(torch.bfloat16)
    dW = (torch.randn(64, 96, generator=g) * 1e-3).to(torch.bfloat16)
    Wb = W.view(torch.int16).numpy().view(np.uint16)
    Gb = dW.view(torch.int16).numpy().view(np.uint16)
    rng = np.random.default_rng(1)
    m = rng.uniform(0.8, 1.2, (64, 6)).astype(F)
    q = rng.normal(6, 2, (64, 12)).astype(F)
    s2 = oracle.s2(Wb)
    f = oracle.fwd(Wb, m, q, s2)
    dm, dq = oracle.ste_bwd(Wb, Gb, m, q, s2)
    m1, q1 = m.copy(), q.copy()
    a = [np.zeros_like(m), np.zeros_like(m), np.zeros_like(q), np.zeros_like(q)]
    oracle.adamw(m1, dm, a[0], a[1], 5e-3, 1)
    oracle.adamw(q1, dq, a[2], a[3], 1e-3, 1)
    m2, q2 = m.copy(), q.copy()
    b = [np.zeros_like(m), np.zeros_like(m), np.zeros_like(q), np.zeros_like(q)]
    Wq, gm, gq = oracle.step(Wb, Gb, m2, q2, *b, s2, 1)
    np.testing.assert_array_equal(Wq, f.Wq)
    np.testing.assert_array_equal(gm, dm); np.testing.assert_array_equal(gq, dq)
    np.testing.assert_array_equal(m2, m1); np.testing.assert_array_equal(q2, q1)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
