"""Exhaustive checks of the kernels' device arithmetic (focus_device.cuh).

* The quotient fl(w/D) from one reciprocal per sub-block with one Markstein
  correction (scalar and packed f32x2 forms) equals the IEEE division, bit
  for bit (signed zeros included),
  for every bf16 significand of w (both signs, and +-0) and every binary32
  significand of D, at several exponent pairs inside the range the kernels
  use it for; where the quotient is below 2^-100 (tiny w, large D) it is
  within one unit in the last place with the same sign and E2M1 code.
* fl(c*S) through the mixed-precision FMA equals the binary32 product for
  every E2M1 value and every normal E4M3 scale, and c - y likewise.
* The E2M1 conversion keeps the sign of negative values that round to zero
  (code 0x8), which the kernels rely on for the signed-zero reading; the
  four-pair form (codes packed by a byte move) equals four single pairs.
* The reciprocal from the hardware approximation and one Newton step equals
  __frcp_rn for every significand; the twice-corrected quotient used for the
  scaled block maximum equals __fdiv_rn (every divisor significand for 1024
  pseudo-random numerators, and 2^30 pseudo-random pairs).
* The pipeline's bounded wait gives up (and reports) on a barrier nothing
  completes, and succeeds on one that is completed.
* The forward's sigmoid (own e^x, a rounding-certainty test, sigmoid_rn where
  it cannot decide) equals sigmoid_rn for EVERY binary32 logit with
  |q| <= 100; the export's sigmoid of an updated logit (a Taylor step from the
  forward's binary64 sigmoid) equals sigmoid_rn on 2^29 pairs with steps of
  every magnitude.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cuda", "device_checks.cu")
LIB = os.path.join(HERE, "cuda", "libdevice_checks.so")
HDR = os.path.join(os.path.dirname(HERE), "fp4_post_weight_b200", "csrc", "focus_device.cuh")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(SRC), os.path.getmtime(HDR)):
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-Xcompiler",
                        "-fPIC", "-shared", SRC, "-o", LIB], check=True)
    L = ctypes.CDLL(LIB)
    L.check_div.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_ulonglong),
                            ctypes.POINTER(ctypes.c_float), ctypes.c_int]
    L.check_mixed.argtypes = [ctypes.POINTER(ctypes.c_ulonglong)]
    L.check_rcp.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_ulonglong)]
    L.check_div_full.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_ulonglong, ctypes.POINTER(ctypes.c_ulonglong),
                                 ctypes.POINTER(ctypes.c_float)]
    L.e2m1_raw_bytes.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
    L.check_wait.argtypes = [ctypes.c_ulonglong, ctypes.POINTER(ctypes.c_ulonglong)]
    L.check_quad.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_ulonglong, ctypes.c_int,
                             ctypes.POINTER(ctypes.c_ulonglong)]
    L.check_sigmoid_fast.argtypes = [ctypes.POINTER(ctypes.c_ulonglong), ctypes.POINTER(ctypes.c_float)]
    L.check_sigmoid_step.argtypes = [ctypes.c_ulonglong, ctypes.POINTER(ctypes.c_ulonglong),
                                     ctypes.POINTER(ctypes.c_float)]
    return L


@pytest.mark.parametrize("variant", [0, 2], ids=["scalar", "packed"])
@pytest.mark.parametrize("we,de", [(0, 0), (-7, 3), (-20, -13), (10, -40), (-40, 10), (59, 0), (0, 59), (0, -59),
                                   (-59, 0), (30, -30), (-30, 29)])
def test_division_exhaustive(lib, we, de, variant):
    n = ctypes.c_ulonglong(0)
    ex = (ctypes.c_float * 4)()
    assert lib.check_div(we, de, ctypes.byref(n), ex, variant) == 0
    assert n.value == 0, f"{n.value} quotients differ, e.g. w={ex[0]!r} D={ex[1]!r} got {ex[2]!r} want {ex[3]!r}"


@pytest.mark.parametrize("variant", [0, 2], ids=["scalar", "packed"])
@pytest.mark.parametrize("we,de", [(-126, 0), (-126, 5), (-133, 0), (-90, 40), (-110, 30), (-100, 59), (-126, 59),
                                   (-133, 59), (-120, -3)])
def test_division_tiny_quotients(lib, we, de, variant):
    """Tiny w over a large D (the kernels take the fast quotient whenever D lies in
    [2^-60, 2^60], whatever |w|): for quotients of at least 2^-100 the bits agree;
    below that the remainder of the correction need not be representable and the
    result may be one unit in the last place off, with the same sign, so its E2M1
    code is the same signed zero and its share of a gradient sum is below
    2^-123 |g|."""
    n = ctypes.c_ulonglong(0)
    ex = (ctypes.c_float * 4)()
    assert lib.check_div(we, de, ctypes.byref(n), ex, variant | 4) == 0
    assert n.value == 0, f"{n.value} quotients differ, e.g. w={ex[0]!r} D={ex[1]!r} got {ex[2]!r} want {ex[3]!r}"


def test_mixed_precision_helpers(lib):
    bad = ctypes.c_ulonglong(0)
    assert lib.check_mixed(ctypes.byref(bad)) == 0
    assert bad.value == 0


def test_e2m1_conversion_zero_sign(lib):
    lo = np.array([-0.1, -0.0, -0.25, 0.1, -1e-30, -0.2], np.float32)
    hi = np.array([0.0, -0.1, 0.2, -0.24, -0.0, -1e-20], np.float32)
    out = np.zeros(len(lo), np.uint32)
    assert lib.e2m1_raw_bytes(lo.ctypes.data, hi.ctypes.data, out.ctypes.data, len(lo)) == 0
    mags = out & 0x77
    assert np.all(mags == 0)            # every value rounds to a zero magnitude
    want = (np.signbit(lo).astype(np.uint32) << 3) | (np.signbit(hi).astype(np.uint32) << 7)
    np.testing.assert_array_equal(out, want)


def test_e2m1_quad_equals_pairs(lib):
    """The four-pair conversion (FourOverSix) gives the word and the binary16 values
    of four single-pair conversions, on 2^24 quadruples drawn from the E2M1 grid
    values, the midpoints and their binary32 neighbours, signed zeros, tiny and
    out-of-range values and random values."""
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, 6.5, 7], np.float32)
    near = np.concatenate([np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(10))])
    odd = np.array([1e-30, 1e-45, 6.0000005, 1e6, 3e38], np.float32)
    rng = np.random.default_rng(5)
    base = np.concatenate([grid, mids, near, odd, rng.uniform(-8, 8, 2000).astype(np.float32)])
    vals = np.ascontiguousarray(np.concatenate([base, -base, np.array([0.0, -0.0], np.float32)]))
    n = ctypes.c_ulonglong(0)
    assert lib.check_quad(vals.ctypes.data, len(vals), 99, 1 << 16, ctypes.byref(n)) == 0
    assert n.value == 0, f"{n.value} quadruples differ"


@pytest.mark.parametrize("e", [0, -20, 20, -59, 59, -100, 100])
def test_reciprocal_exhaustive(lib, e):
    n = ctypes.c_ulonglong(0)
    assert lib.check_rcp(e, ctypes.byref(n)) == 0
    assert n.value == 0


@pytest.mark.parametrize("mode,seed", [(0, 1), (0, 2), (1, 3), (1, 4)])
def test_full_quotient(lib, mode, seed):
    n = ctypes.c_ulonglong(0)
    ex = (ctypes.c_float * 4)()
    assert lib.check_div_full(mode, 512, seed, ctypes.byref(n), ex) == 0
    assert n.value == 0, f"{n.value} quotients differ, e.g. a={ex[0]!r} b={ex[1]!r} got {ex[2]!r} want {ex[3]!r}"


def test_sigmoid_fast_every_logit(lib):
    """Every binary32 logit with |q| <= 100: the forward's sigmoid equals sigmoid_rn
    bit for bit, its binary64 value is within 2^-49, and the fast path decides
    the rounding for nearly every logit."""
    c = (ctypes.c_ulonglong * 4)()
    ex = (ctypes.c_float * 4)()
    assert lib.check_sigmoid_fast(c, ex) == 0
    assert c[2] > 2_000_000_000
    assert c[0] == 0, f"{c[0]} sigmoids differ, e.g. q={ex[0]!r} got {ex[1]!r} want {ex[2]!r}"
    assert c[1] == 0, f"{c[1]} binary64 values outside 2^-49"
    assert c[3] > 0.999 * c[2] * 0.8


@pytest.mark.parametrize("seed", [21, 22])
def test_sigmoid_step_of_updated_logit(lib, seed):
    c = (ctypes.c_ulonglong * 4)()
    ex = (ctypes.c_float * 4)()
    assert lib.check_sigmoid_step(seed, c, ex) == 0
    assert c[1] == 1 << 28
    assert c[0] == 0, f"{c[0]} differ, e.g. q0={ex[0]!r} q1={ex[1]!r} got {ex[2]!r} want {ex[3]!r}"
    assert c[2] > 0.5 * c[1]            # the Taylor step decides most roundings


def test_bounded_wait_runs_out_and_reports(lib):
    """Failure detection without a GPU fault: a pipeline wait on a barrier that
    nothing completes gives up after its limit (2 ms here; 2 s in the kernels)
    and returns false -- the kernels then set the timeout flag, which
    focus_get_error reports as FOCUS_ERR_DEVICE_TIMEOUT -- while a wait on a
    completed barrier returns true.  Nothing hangs or traps."""
    res = (ctypes.c_ulonglong * 3)()
    assert lib.check_wait(2_000_000, res) == 0
    assert res[0] == 0, "the wait on a barrier nothing completes did not give up"
    assert 2_000_000 <= res[1] < 1_000_000_000, f"gave up after {res[1]} ns"
    assert res[2] == 1, "the wait on a completed barrier failed"
