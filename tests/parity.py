"""Comparison helpers for the GPU parity tests (the oracle is the reference).

Bar (stated with the method): E4M3 scale bytes bit-exact; E2M1 codes
bit-exact except codes whose y lies within 2^-20 relative of a code boundary
or of +-6 (the oracle's band flag 1; exact midpoints, flag 2, must match), and
such mismatches below 1e-6 of the elements; w' bit-exact wherever the code
matches; gradients, parameters and moments within
|gpu - ref| <= 1e-7 + 1e-5 * |ref|.

FourOverSix: the oracle's choice between the targets 6 and 4 is the exact
order of the two squared errors.  The kernels take it from binary32 sums and,
inside their certified screen band, from binary64 sums, which can order a
block otherwise only when |e4 - e6| <= 2^-47 (e4 + e6).  A block's outputs
(scale byte, codes, dequantized values) must therefore match bit for bit
except inside that band, and such blocks must stay below 1e-6 of the blocks.
"""
from __future__ import annotations

import numpy as np
import torch

RTOL = 1e-5
ATOL = 1e-7
MAX_MISMATCH_FRAC = 1e-6

# Counts the parity tests record (elements checked, band populations, mismatches),
# printed once at the end of the run by tests/conftest.py.
RECORD: dict[str, dict] = {}


def record(name: str, counts: dict) -> None:
    """Adds counts to the run's parity record under `name` (summed over calls)."""
    acc = RECORD.setdefault(name, {})
    for k, v in counts.items():
        acc[k] = acc.get(k, 0) + int(v)


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


def forward_counts(ref, mism: np.ndarray | None = None) -> dict:
    """Counts of an oracle forward (oracle.Forward.stats) with the code mismatches found."""
    st = ref.stats
    return {"elements": int(ref.codes.size), "band": st["band"], "exact_ties": st["exact_ties"],
            "code_mismatch": 0 if mism is None else int(mism.sum()), "zero_blocks": st["zero_blocks"],
            "clamp_low": st["clamp_low"], "clamp_high": st["clamp_high"], "out_of_range": st["out_of_range"]}


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


F46_SCREEN = 2.0 ** -19     # the kernels' binary32 screen: inside it the choice is taken from binary64 sums
F46_BAND = 2.0 ** -47       # the binary64 sums' bound: only inside it may a kernel's choice differ


def f46_counts(ref) -> dict:
    """Band populations of a FourOverSix oracle result (exact errors, reported as binary64 sums)."""
    e6, e4 = ref.errs[..., 0], ref.errs[..., 1]
    gap, tot = np.abs(e4 - e6), e4 + e6
    return {"blocks": int(e6.size), "target4": int(ref.four.sum()),
            "screen_band": int((gap <= F46_SCREEN * tot).sum()),
            "ties_nonzero": int(((gap == 0) & (tot > 0)).sum()),
            "band_2^-47": int((gap <= F46_BAND * tot).sum())}


def f46_tie_counts(ref, X_bits: np.ndarray, s) -> dict:
    """Of the blocks whose two exact errors tie (nonzero), how many have identical
    candidates (equal scale bytes S6 == S4: the block of the row's or tensor's maximum,
    where both scales clamp at 448) -- recomputed here from X and the scale(s)."""
    e6, e4 = ref.errs[..., 0], ref.errs[..., 1]
    tie = (e6 == e4) & (e6 + e4 > 0)
    rows, nb = ref.scales.shape
    A = ((X_bits.astype(np.uint32) & 0x7FFF) << 16).view(np.float32).reshape(rows, nb, 16).max(-1)
    s = np.broadcast_to(np.asarray(s, np.float32).reshape(-1, 1), (rows, nb))
    with np.errstate(divide="ignore", invalid="ignore"):      # a zero row (s = 0) has no tie
        x6 = (A / (np.float32(6) * s)).astype(np.float32)
        x4 = (A / (np.float32(4) * s)).astype(np.float32)
    same = (s > 0) & (x6 >= np.float32(432)) & (x4 >= np.float32(432))    # both E4M3 bytes round to 448
    return {"ties_same_candidate": int((tie & same).sum()), "ties_different_candidates": int((tie & ~same).sum())}


def check_fouroversix(ref, codes: np.ndarray, scales: np.ndarray, Xq: np.ndarray | None) -> dict:
    """ref: oracle.FourOverSix; codes unpacked uint8 [rows, cols]; scales uint8 [rows, cols/16];
    Xq uint16 bits or None.  Asserts the bar above and returns the counts with the mismatches."""
    rows, nb = ref.scales.shape
    bad = scales != ref.scales
    bad |= (codes != ref.codes).reshape(rows, nb, 16).any(-1)
    if Xq is not None:
        bad |= (Xq != ref.Xq).reshape(rows, nb, 16).any(-1)
    c = f46_counts(ref)
    c["mismatched_blocks"] = n = int(bad.sum())
    if n:
        e6, e4 = ref.errs[..., 0], ref.errs[..., 1]
        assert np.all(np.abs(e4 - e6)[bad] <= F46_BAND * (e4 + e6)[bad]), \
            f"{n} FourOverSix blocks differ outside the 2^-47 band of the exact errors"
        assert n <= MAX_MISMATCH_FRAC * bad.size, f"{n} FourOverSix blocks differ in {bad.size}"
    return c
