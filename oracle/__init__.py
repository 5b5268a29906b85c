"""CPU oracle of the FOCUS NVFP4 weight fake-quantizer -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product (``fp4_post_weight_b200``) never
does, and this package never imports the product.  The arithmetic lives in
``focus_oracle.c`` (plain scalar C, one loop per equation of the FOCUS card);
this module only compiles it with gcc and marshals numpy arrays to it.

bf16 tensors travel as ``numpy.uint16`` arrays of their bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "focus_oracle.c")
_LIB = os.path.join(_HERE, "libfocus_oracle.so")

# -ffp-contract=off: one rounding per operation, as the forward's reading requires.
CFLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared",
          "-std=c11", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile focus_oracle.c into libfocus_oracle.so (when missing or stale)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


class Stats(ctypes.Structure):
    _fields_ = [("zero_blocks", ctypes.c_int64), ("clamp_low", ctypes.c_int64),
                ("clamp_high", ctypes.c_int64), ("out_of_range", ctypes.c_int64),
                ("band", ctypes.c_int64), ("exact_ties", ctypes.c_int64)]

    def as_dict(self):
        return {k: int(getattr(self, k)) for k, _ in self._fields_}


_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_F = ctypes.c_float
_D = ctypes.c_double


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.fo_bf16_to_f32.argtypes = [ctypes.c_uint16]; L.fo_bf16_to_f32.restype = _F
        L.fo_f32_to_bf16.argtypes = [_F]; L.fo_f32_to_bf16.restype = ctypes.c_uint16
        L.fo_e4m3_encode.argtypes = [_F]; L.fo_e4m3_encode.restype = ctypes.c_int
        L.fo_e4m3_decode.argtypes = [ctypes.c_int]; L.fo_e4m3_decode.restype = _D
        L.fo_e2m1_encode.argtypes = [_F]; L.fo_e2m1_encode.restype = ctypes.c_int
        L.fo_e2m1_decode.argtypes = [ctypes.c_int]; L.fo_e2m1_decode.restype = _D
        L.fo_sigmoid.argtypes = [_F]; L.fo_sigmoid.restype = _F
        L.fo_num_threads.argtypes = []; L.fo_num_threads.restype = ctypes.c_int
        L.fo_set_num_threads.argtypes = [ctypes.c_int]; L.fo_set_num_threads.restype = None
        L.fo_s2.argtypes = [_P, _I64, _P]; L.fo_s2.restype = ctypes.c_int
        L.fo_fwd.argtypes = [_P, _P, _P, _F, _I64, _I64, _P, _P, _P, _P, _P, _P]
        L.fo_fwd.restype = ctypes.c_int
        L.fo_ste_bwd.argtypes = [_P, _P, _P, _P, _F, _I64, _I64, _P, _P, ctypes.c_int]
        L.fo_ste_bwd.restype = ctypes.c_int
        L.fo_adamw.argtypes = [_P, _P, _P, _P, _I64, _D, _D, _D, _D, _D, _I64]
        L.fo_adamw.restype = ctypes.c_int
        L.fo_step.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _F, _I64, _I64, _D, _D, _D, _D, _D, _D,
                              _I64, _P, _P, _P, _P, _P]
        L.fo_step.restype = ctypes.c_int
        L.fo_pack.argtypes = [_P, _P, _P, _F, _I64, _I64, _P, _P, _P]
        L.fo_pack.restype = ctypes.c_int
        L.fo_f46.argtypes = [_P, _I64, _I64, _F, ctypes.c_int, _P, _P, _P, _P, _P, _P]
        L.fo_f46.restype = ctypes.c_int
        L.fo_f46_exact_sign.argtypes = [_P, _P, _P, ctypes.c_int]
        L.fo_f46_exact_sign.restype = ctypes.c_int
        L.fo_nvfp4_rows.argtypes = [_P, _I64, _I64, _P, _P, _P, _P]; L.fo_nvfp4_rows.restype = ctypes.c_int
        L.fo_mx_fwd.argtypes = [_P, _P, _P, _I64, _I64, _P, _P, _P]; L.fo_mx_fwd.restype = ctypes.c_int
        L.fo_mx_ste_bwd.argtypes = [_P, _P, _P, _P, _I64, _I64, _P, _P, ctypes.c_int]
        L.fo_mx_ste_bwd.restype = ctypes.c_int
        L.fo_swizzled_bytes.argtypes = [_I64, _I64]; L.fo_swizzled_bytes.restype = _I64
        L.fo_scales_swizzle.argtypes = [_P, _I64, _I64, _P]; L.fo_scales_swizzle.restype = ctypes.c_int
        _lib = L
    return _lib


class OracleError(RuntimeError):
    pass


_ERRS = {1: "shape", 2: "value", 3: "non-finite input"}


def _chk(rc):
    if rc != 0:
        raise OracleError(f"oracle error {rc}: {_ERRS.get(rc, '?')}")


def _p(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    if a.dtype != dtype:
        raise TypeError(f"expected {dtype}, got {a.dtype}")
    return a


def set_threads(n: int) -> None:
    lib().fo_set_num_threads(int(n))


def num_threads() -> int:
    return int(lib().fo_num_threads())


# --- scalar codecs -------------------------------------------------------------

def e2m1_encode(u: float) -> int:
    return int(lib().fo_e2m1_encode(float(u)))


def e2m1_decode(code: int) -> float:
    return float(lib().fo_e2m1_decode(int(code)))


def e4m3_encode(x: float) -> int:
    return int(lib().fo_e4m3_encode(float(x)))


def e4m3_decode(b: int) -> float:
    return float(lib().fo_e4m3_decode(int(b)))


def sigmoid(q: float) -> float:
    return float(lib().fo_sigmoid(float(q)))


def bf16_from_f32(f: float) -> int:
    return int(lib().fo_f32_to_bf16(float(f)))


def f32_from_bf16(h: int) -> float:
    return float(lib().fo_bf16_to_f32(int(h)))


# --- tensor entry points --------------------------------------------------------

def s2(W: np.ndarray) -> np.float32:
    """Per-tensor scale s2 = amax(|W|)/(6*448).  W: uint16 bf16 bits, any shape."""
    W = _c(W, np.uint16)
    out = np.zeros(1, np.float32)
    _chk(lib().fo_s2(_p(W), W.size, _p(out)))
    return out[0]


@dataclass
class Forward:
    Wq: np.ndarray       # uint16 bf16 bits [out, in]
    codes: np.ndarray    # uint8 [out, in], one E2M1 code per element
    scales: np.ndarray   # uint8 [out, in/16]
    band: np.ndarray     # uint8 [out, in]: 0, 1 near a boundary, 2 exactly on a midpoint
    y: np.ndarray        # float32 [out, in]
    stats: dict


def fwd(W, m, q, s2v, want_y: bool = True) -> Forward:
    W = _c(W, np.uint16); m = _c(m, np.float32); q = _c(q, np.float32)
    out, inn = W.shape
    if m.size != out * (inn // 16) or q.size != out * (inn // 8):
        raise ValueError("m/q size does not match W")
    Wq = np.empty((out, inn), np.uint16)
    codes = np.empty((out, inn), np.uint8)
    scales = np.empty((out, inn // 16), np.uint8)
    band = np.empty((out, inn), np.uint8)
    y = np.empty((out, inn), np.float32) if want_y else None
    st = Stats()
    _chk(lib().fo_fwd(_p(W), _p(m), _p(q), float(s2v), out, inn, _p(Wq), _p(codes), _p(scales),
                      _p(band), _p(y), ctypes.byref(st)))
    return Forward(Wq, codes, scales, band, y, st.as_dict())


def ste_bwd(W, dWq, m, q, s2v, dm=None, dq=None):
    """Straight-through gradients.  When dm/dq are given they are added to (in place)."""
    W = _c(W, np.uint16); dWq = _c(dWq, np.uint16)
    m = _c(m, np.float32); q = _c(q, np.float32)
    out, inn = W.shape
    acc = dm is not None
    if acc:
        dm = _c(dm, np.float32); dq = _c(dq, np.float32)
    else:
        dm = np.empty((out, inn // 16), np.float32)
        dq = np.empty((out, inn // 8), np.float32)
    _chk(lib().fo_ste_bwd(_p(W), _p(dWq), _p(m), _p(q), float(s2v), out, inn, _p(dm), _p(dq),
                          1 if acc else 0))
    return dm, dq


def adamw(p, g, v1, v2, lr, step, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0):
    """AdamW update in place on float32 arrays p, v1, v2."""
    for a in (p, v1, v2):
        if a.dtype != np.float32 or not a.flags.c_contiguous:
            raise TypeError("p, v1, v2 must be contiguous float32")
    g = _c(g, np.float32)
    _chk(lib().fo_adamw(_p(p), _p(g), _p(v1), _p(v2), p.size, lr, beta1, beta2, eps, weight_decay,
                        int(step)))


def step(W, dWq, m, q, m_v1, m_v2, q_v1, q_v2, s2v, step_t, lr_m=5e-3, lr_q=1e-3, beta1=0.9,
         beta2=0.999, eps=1e-8, weight_decay=0.0, want_wq=True, dm_acc=None, dq_acc=None):
    """One fused step in place on m, q and the four moment arrays.

    Returns (Wq or None, gm, gq): the forward's w' and the gradients used."""
    W = _c(W, np.uint16); dWq = _c(dWq, np.uint16)
    for a in (m, q, m_v1, m_v2, q_v1, q_v2):
        if a.dtype != np.float32 or not a.flags.c_contiguous:
            raise TypeError("parameters and moments must be contiguous float32")
    out, inn = W.shape
    Wq = np.empty((out, inn), np.uint16) if want_wq else None
    gm = np.empty((out, inn // 16), np.float32)
    gq = np.empty((out, inn // 8), np.float32)
    if dm_acc is not None:
        dm_acc = _c(dm_acc, np.float32); dq_acc = _c(dq_acc, np.float32)
    _chk(lib().fo_step(_p(W), _p(dWq), _p(m), _p(q), _p(m_v1), _p(m_v2), _p(q_v1), _p(q_v2),
                       float(s2v), out, inn, lr_m, lr_q, beta1, beta2, eps, weight_decay, int(step_t),
                       _p(Wq), _p(dm_acc), _p(dq_acc), _p(gm), _p(gq)))
    return Wq, gm, gq


def pack(W, m, q, s2v):
    """NVFP4 export: (codes u8 [out, in/2], scales u8 [out, in/16], tensor scale f32)."""
    W = _c(W, np.uint16); m = _c(m, np.float32); q = _c(q, np.float32)
    out, inn = W.shape
    codes = np.empty((out, inn // 2), np.uint8)
    scales = np.empty((out, inn // 16), np.uint8)
    ts = np.zeros(1, np.float32)
    _chk(lib().fo_pack(_p(W), _p(m), _p(q), float(s2v), out, inn, _p(codes), _p(scales), _p(ts)))
    return codes, scales, ts[0]


@dataclass
class FourOverSix:
    codes: np.ndarray       # uint8 [rows, cols], one E2M1 code per element
    scales: np.ndarray      # uint8 [rows, cols/16], E4M3 byte of the chosen block scale
    Xq: np.ndarray          # uint16 bf16 bits [rows, cols], dequantized values
    four: np.ndarray        # uint8 [rows, cols/16], 1 where the target 4 was chosen
    errs: np.ndarray        # float64 [rows, cols/16, 2], squared errors of the targets 6 and 4 (binary64 sums)
    row_scales: np.ndarray | None   # float32 [rows] with one scale per row, else None


def fouroversix(X, s=None) -> FourOverSix:
    """FourOverSix round to nearest.  s: the tensor scale (weights), or None for
    one scale per row (per-token activations), computed from each row."""
    X = _c(X, np.uint16)
    rows, cols = X.shape
    nb = cols // 16
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty((rows, nb), np.uint8)
    Xq = np.empty((rows, cols), np.uint16)
    four = np.empty((rows, nb), np.uint8)
    errs = np.empty((rows, nb, 2), np.float64)
    per_row = s is None
    rs = np.empty(rows, np.float32) if per_row else None
    _chk(lib().fo_f46(_p(X), rows, cols, 0.0 if per_row else float(s), 1 if per_row else 0, _p(codes),
                      _p(scales), _p(Xq), _p(four), _p(errs), _p(rs)))
    return FourOverSix(codes, scales, Xq, four, errs, rs)


def f46_exact_sign(w, v4, v6) -> int:
    """Sign of sum (w - v4)^2 - sum (w - v6)^2 over at most 16 binary64 values,
    evaluated exactly (the comparison behind the FourOverSix choice)."""
    w, v4, v6 = (_c(np.asarray(a, np.float64), np.float64) for a in (w, v4, v6))
    assert w.shape == v4.shape == v6.shape and w.size <= 16
    return int(lib().fo_f46_exact_sign(_p(w), _p(v4), _p(v6), w.size))


def nvfp4_rows(X) -> FourOverSix:
    """NVFP4 round to nearest with one scale per row (per-token activations): the
    card's block equations with m = 1, sigmoid = 1 and s_t = max_row|x|/2688.
    Returns the FourOverSix record with four = 0 and errs = None."""
    X = _c(X, np.uint16)
    rows, cols = X.shape
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty((rows, cols // 16), np.uint8)
    Xq = np.empty((rows, cols), np.uint16)
    rs = np.empty(rows, np.float32)
    _chk(lib().fo_nvfp4_rows(_p(X), rows, cols, _p(codes), _p(scales), _p(Xq), _p(rs)))
    return FourOverSix(codes, scales, Xq, np.zeros((rows, cols // 16), np.uint8), None, rs)


def scales_swizzle(scales: np.ndarray) -> np.ndarray:
    """E4M3 scale bytes [rows, cols] -> the 128x4-atom layout of the sm_100
    block-scaled GEMM (flat uint8, rows padded to 128 and cols to 4, zeros)."""
    scales = _c(scales, np.uint8)
    rows, cols = scales.shape
    out = np.empty(int(lib().fo_swizzled_bytes(rows, cols)), np.uint8)
    _chk(lib().fo_scales_swizzle(_p(scales), rows, cols, _p(out)))
    return out


@dataclass
class MXForward:
    Wq: np.ndarray       # uint16 bf16 bits [out, in]
    codes: np.ndarray    # uint8 [out, in], one E2M1 code per element
    scales: np.ndarray   # uint8 [out, in/32], E8M0 bytes


def mx_fwd(W, m, q) -> MXForward:
    """MXFP4 variant: m [out, in/32], q [out, in/8]."""
    W = _c(W, np.uint16); m = _c(m, np.float32); q = _c(q, np.float32)
    out, inn = W.shape
    if m.size != out * (inn // 32) or q.size != out * (inn // 8):
        raise ValueError("m/q size does not match W")
    Wq = np.empty((out, inn), np.uint16)
    codes = np.empty((out, inn), np.uint8)
    scales = np.empty((out, inn // 32), np.uint8)
    _chk(lib().fo_mx_fwd(_p(W), _p(m), _p(q), out, inn, _p(Wq), _p(codes), _p(scales)))
    return MXForward(Wq, codes, scales)


def mx_ste_bwd(W, dWq, m, q, dm=None, dq=None):
    """MXFP4 straight-through gradients (added to dm/dq in place when given)."""
    W = _c(W, np.uint16); dWq = _c(dWq, np.uint16)
    m = _c(m, np.float32); q = _c(q, np.float32)
    out, inn = W.shape
    acc = dm is not None
    if acc:
        dm = _c(dm, np.float32); dq = _c(dq, np.float32)
    else:
        dm = np.empty((out, inn // 32), np.float32)
        dq = np.empty((out, inn // 8), np.float32)
    _chk(lib().fo_mx_ste_bwd(_p(W), _p(dWq), _p(m), _p(q), out, inn, _p(dm), _p(dq), 1 if acc else 0))
    return dm, dq
