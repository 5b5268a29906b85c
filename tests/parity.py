"""Comparison helpers for the GPU parity tests (the oracle is the reference).

Bar (stated with the method): E4M3 scale bytes bit-exact; E2M1 codes
bit-exact except codes whose y lies within 2^-20 relative of a code boundary
or of +-6 (the oracle's band flag 1; exact midpoints, flag 2, must match), and
such mismatches below 1e-6 of the elements; w' bit-exact wherever the code
matches; gradients, parameters and moments within
|gpu - ref| <= 1e-7 + 1e-5 * |ref|.
"""
from __future__ import annotations

import numpy as np
import torch

RTOL = 1e-5
ATOL = 1e-7
MAX_MISMATCH_FRAC = 1e-6


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy()


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    out = np.empty((packed.shape[0], packed.shape[1] * 2), np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def check_codes(codes: np.ndarray, ref) -> np.ndarray:
    """Returns the boolean mismatch map after asserting the bar."""
    mism = codes != ref.codes
    n = int(mism.sum())
    if n:
        assert np.all(ref.band[mism] == 1), "code mismatch outside the 2^-20 band (or on an exact tie)"
        assert n <= MAX_MISMATCH_FRAC * codes.size, f"{n} code mismatches in {codes.size} elements"
    return mism


def check_forward(ref, Wq=None, codes=None, scales=None):
    """ref: oracle.Forward; Wq: uint16 bits; codes: unpacked uint8; scales: uint8."""
    mism = np.zeros(ref.codes.shape, bool)
    if scales is not None:
        np.testing.assert_array_equal(scales, ref.scales)
    if codes is not None:
        mism = check_codes(codes, ref)
    if Wq is not None:
        ok = ~mism
        bad = (Wq != ref.Wq) & ok
        assert not bad.any(), f"{int(bad.sum())} W' values differ where the codes agree"
    return mism


def block_mask(mism: np.ndarray) -> np.ndarray:
    """Blocks [out, in/16] that contain a tolerated code mismatch."""
    o, i = mism.shape
    return mism.reshape(o, i // 16, 16).any(-1)


def assert_close(gpu: np.ndarray, ref: np.ndarray, name: str, skip: np.ndarray | None = None):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (name, gpu.shape, ref.shape)
    err = np.abs(gpu - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    bad |= np.isnan(gpu) != np.isnan(ref)
    if skip is not None:
        bad &= ~skip
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{name}: {int(bad.sum())} of {gpu.size} outside tolerance; e.g. "
                             + ", ".join(f"{tuple(i)}: gpu {gpu[tuple(i)]!r} ref {ref[tuple(i)]!r}" for i in idx))
