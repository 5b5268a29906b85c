"""focus_s2_noalloc: the per-tensor scale for callers that cannot allocate.

Some callers of this library cannot hand it device memory: a runtime whose own
memory pool owns every device allocation and forbids any other, or a code path
that must never call cudaMalloc (which can synchronize the device).  For them
focus_s2_noalloc keeps its scratch (one word per 4096-weight tile) in a fixed
array inside the library instead of a caller workspace.  This test calls it
through the C ABI twice in a row -- a large ragged tensor, then a small one,
so scratch left by the first call would show in the second -- and checks each
result against focus_s2 with a caller workspace (s2 is exact, so they must be
equal) and that the two calls took no device memory (after a warm-up call,
which may load the library's device code); then that an empty tensor gives
s2 = 0, as with focus_s2, and that a tensor larger than the array covers is
refused before anything runs.
"""
import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _call(F, W, out, inn, s2):
    stream = torch.cuda.current_stream().cuda_stream
    return F.raw_call("focus_s2_noalloc", ctypes.c_void_p(W.data_ptr()), ctypes.c_int64(out), ctypes.c_int64(inn),
                      ctypes.c_void_p(s2.data_ptr()), ctypes.c_void_p(stream))


def test_noalloc_s2_matches_workspace_s2_twice():
    from fp4_post_weight_b200 import focus as F
    g = torch.Generator(device="cuda").manual_seed(2026)
    cases = []
    for (out, inn), planted in (((4096, 4096 + 7 * 16), 0.6875), ((37, 1040), 0.4375)):
        W = (torch.randn((out, inn), generator=g, device="cuda") * 0.02).to(torch.bfloat16)
        W[out // 3, inn - 5] = -planted           # the tensor max, placed in a late tile
        ws = torch.empty(F.focus_s2_workspace_bytes(out, inn), dtype=torch.uint8, device="cuda")
        want = torch.full((1,), -1.0, device="cuda")
        F.focus_s2(W, want, ws)
        cases.append((W, out, inn, planted, want, torch.full((1,), -2.0, device="cuda")))
    # a warm-up call: the first call on a device may load the library's device code
    assert _call(F, cases[1][0], 37, 1040, torch.zeros(1, device="cuda")) == F.FOCUS_OK
    torch.cuda.synchronize()
    held, (free, _) = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()
    for W, out, inn, planted, want, got in cases:
        assert _call(F, W, out, inn, got) == F.FOCUS_OK
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == held and torch.cuda.mem_get_info()[0] == free, \
        "the calls took device memory"
    assert F.focus_get_error() == F.FOCUS_OK
    for W, out, inn, planted, want, got in cases:
        assert got.item() == want.item()
        assert got.item() == float(np.float32(planted) / np.float32(2688.0))


def test_noalloc_s2_of_an_empty_tensor_is_zero():
    from fp4_post_weight_b200 import focus as F
    W = torch.zeros((0, 4096), dtype=torch.bfloat16, device="cuda")
    got = torch.full((1,), -2.0, device="cuda")
    assert _call(F, W, 0, 4096, got) == F.FOCUS_OK
    assert F.focus_get_error() == F.FOCUS_OK
    assert got.item() == 0.0


def test_noalloc_s2_refuses_tensors_beyond_its_scratch():
    from fp4_post_weight_b200 import focus as F
    W = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    s2 = torch.zeros(1, device="cuda")
    # one row more than the scratch covers: refused by the host-side check, before any
    # kernel is enqueued (the 16-element buffer passed here is never read)
    too_many_rows = F.FOCUS_S2_NOALLOC_MAX_WEIGHTS // 4096 + 1
    assert _call(F, W, too_many_rows, 4096, s2) == 5          # FOCUS_ERR_WORKSPACE
    assert F.focus_get_error() == F.FOCUS_OK
