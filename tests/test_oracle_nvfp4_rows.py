"""Pins of the oracle's per-token NVFP4 round to nearest (fo_nvfp4_rows).

Model card "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct", section
"Perplexity": the NVFP4 baseline quantizes activations to NVFP4 with one scale
per token.  The oracle reads it as the card's block equations with m = 1,
sigmoid = 1 and the row's own scale s_t = max_row|x| / 2688 in place of s2.
Pinned here by (1) the independent numpy RTN of test_oracle_rtn (ml_dtypes
casts) applied row by row with a row scale computed in numpy, (2) the
oracle's own forward with m = 1, q = 30 (binary32 sigmoid exactly 1) and
s2 = s_t, row by row, and (3) the zero-row rule.
"""
import numpy as np
import torch

import oracle
import synth
from tests.test_oracle_rtn import rtn_nvfp4

F = np.float32


def _acts(tokens, hidden, seed, zero_tokens=1):
    X = synth.activations(tokens, hidden, "cpu", seed=seed, zero_tokens=zero_tokens)
    return X.view(torch.int16).numpy().view(np.uint16), X.float().numpy()


def test_rows_equal_independent_rtn():
    Xb, Xf = _acts(24, 1040, 3)
    # a block far below its row's maximum (x_b under 2^-6: the lower clamp acts)
    # and a block whose maximum is the row's (x_b near 448)
    tiny = torch.full((16,), 1e-4).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    Xb[2, 32:48] = tiny
    Xb[2, 48] = np.float32(40.0).view(np.uint32) >> 16
    Xf = torch.from_numpy(Xb.view(np.int16)).view(torch.bfloat16).float().numpy()
    r = oracle.nvfp4_rows(Xb)
    for t in range(Xb.shape[0]):
        st = F(np.abs(Xf[t]).max()) / F(2688)
        assert r.row_scales[t] == st
        if st == 0:
            continue
        sb, codes, xq = rtn_nvfp4(Xf[t:t + 1], st)
        np.testing.assert_array_equal(r.scales[t:t + 1], sb)
        np.testing.assert_array_equal(r.codes[t:t + 1], codes)
        np.testing.assert_array_equal(r.Xq[t:t + 1], xq)


def test_rows_are_the_forward_with_unit_parameters():
    Xb, _ = _acts(9, 512, 4, zero_tokens=0)
    r = oracle.nvfp4_rows(Xb)
    for t in range(Xb.shape[0]):
        m = np.ones((1, 512 // 16), F)
        q = np.full((1, 512 // 8), 30.0, F)
        f = oracle.fwd(Xb[t:t + 1], m, q, r.row_scales[t])
        np.testing.assert_array_equal(r.scales[t:t + 1], f.scales)
        np.testing.assert_array_equal(r.codes[t:t + 1], f.codes)
        np.testing.assert_array_equal(r.Xq[t:t + 1], f.Wq)


def test_zero_row():
    Xb, _ = _acts(5, 64, 5, zero_tokens=1)
    r = oracle.nvfp4_rows(Xb)
    assert r.row_scales[-1] == 0
    assert np.all(r.scales[-1] == 0x38) and not r.codes[-1].any() and not r.Xq[-1].any()
    assert r.row_scales[0] > 0
