"""Thin ctypes binding of libfocus.so (include/focus.h): argument marshalling only.

Each function has the name of its C entry point, takes CUDA torch tensors (or
raw device addresses as ints), passes their addresses and the current CUDA
stream, and raises FocusError on a non-zero status.  Every computation runs in
the library's kernels; there is no fallback: a missing libfocus.so raises at
import time.
"""
from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfocus.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libfocus.so is not built ({_LIB_PATH}); run fp4_post_weight_b200.build.build()")
_lib = ctypes.CDLL(_LIB_PATH)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_F = ctypes.c_float
_SZ = ctypes.c_size_t

FOCUS_OK = 0
FOCUS_STEP_ACCUMULATE = 1
FOCUS_STEP_WRITE_GRAD = 2
FOCUS_STEP_PACK_UPDATED = 4
FOCUS_STEP_WQ_UPDATED = 8
FOCUS_PURPOSE_MX = 4
FOCUS_PURPOSE_ACT = 5
FOCUS_PURPOSE_ACT_SWIZZLED = 6
FOCUS_HOST_S2_FIRST = 16


class focus_tensor_desc(ctypes.Structure):
    _fields_ = [("W", _P), ("dWq", _P), ("Wq", _P), ("m", _P), ("q", _P),
                ("m_exp_avg", _P), ("m_exp_avg_sq", _P), ("q_exp_avg", _P), ("q_exp_avg_sq", _P),
                ("s2", _P), ("codes", _P), ("scales", _P), ("dm", _P), ("dq", _P),
                ("out", _I64), ("in_", _I64), ("block_begin", _I64), ("tile_begin", _I64)]


assert ctypes.sizeof(focus_tensor_desc) == 144


class focus_hparams(ctypes.Structure):
    _fields_ = [("lr_m", _F), ("lr_q", _F), ("beta1", _F), ("beta2", _F), ("eps", _F),
                ("weight_decay", _F)]


_SIGS = {
    "focus_status_string": ([_I], ctypes.c_char_p),
    "focus_version": ([], ctypes.c_char_p),
    "focus_s2_workspace_bytes": ([_I64, _I64], _SZ),
    "focus_s2": ([_P, _I64, _I64, _P, _P, _SZ, _P], _I),
    "focus_s2_noalloc": ([_P, _I64, _I64, _P, _P], _I),
    "focus_fwd": ([_P, _P, _P, _F, _I64, _I64, _P, _P], _I),
    "focus_ste_bwd": ([_P, _P, _P, _P, _F, _I64, _I64, _P, _P, _I, _P], _I),
    "focus_adamw_step": ([_P, _P, _P, _P, _I64, _F, _F, _F, _F, _F, _I64, _P], _I),
    "focus_pack_nvfp4": ([_P, _P, _P, _F, _I64, _I64, _P, _P, _P, _P], _I),
    "focus_table_prepare": ([ctypes.POINTER(focus_tensor_desc), _I, _I, ctypes.POINTER(_I64)], _I),
    "focus_s2_multi_workspace_bytes": ([_I64], _SZ),
    "focus_s2_multi": ([_P, _I, _I64, _P, _SZ, _P], _I),
    "focus_step_fused": ([_P, _I, _I64, ctypes.POINTER(focus_hparams), _I64, ctypes.c_uint, _P], _I),
    "focus_pack_multi": ([_P, _I, _I64, _P], _I),
    "focus_step_fused_amax": ([_P, _I, _I64, ctypes.POINTER(focus_hparams), _I64, ctypes.c_uint, _P, _P], _I),
    "focus_s2_from_amax": ([_P, _I, _P, _P], _I),
    "focus_fwd_multi": ([_P, _I, _I64, _P], _I),
    "focus_ste_bwd_multi": ([_P, _I, _I64, _I, _P], _I),
    "focus_fouroversix_weight": ([_P, _I64, _I64, _F, _P, _P, _P, _P], _I),
    "focus_fouroversix_multi": ([_P, _I, _I64, _P], _I),
    "focus_nvfp4_weight": ([_P, _I64, _I64, _F, _P, _P, _P, _P], _I),
    "focus_nvfp4_weight_multi": ([_P, _I, _I64, _P], _I),
    "focus_fouroversix_act": ([_P, _I64, _I64, _P, _P, _P, _P, _P], _I),
    "focus_fouroversix_act_swizzled": ([_P, _I64, _I64, _P, _P, _P, _SZ, _P, _P], _I),
    "focus_nvfp4_act": ([_P, _I64, _I64, _P, _P, _P, _P, _P], _I),
    "focus_nvfp4_act_swizzled": ([_P, _I64, _I64, _P, _P, _P, _SZ, _P, _P], _I),
    "focus_fouroversix_act_multi": ([_P, _I, _I64, _I64, _I, _P], _I),
    "focus_nvfp4_act_multi": ([_P, _I, _I64, _I64, _I, _P], _I),
    "focus_mx_fwd": ([_P, _P, _P, _I64, _I64, _P, _P, _P, _P], _I),
    "focus_mx_ste_bwd": ([_P, _P, _P, _P, _I64, _I64, _P, _P, _I, _P], _I),
    "focus_mx_step": ([_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, ctypes.POINTER(focus_hparams), _I64,
                       ctypes.c_uint, _P, _P, _P, _P], _I),
    "focus_mx_fwd_multi": ([_P, _I, _I64, _P], _I),
    "focus_mx_ste_bwd_multi": ([_P, _I, _I64, _I, _P], _I),
    "focus_mx_step_multi": ([_P, _I, _I64, ctypes.POINTER(focus_hparams), _I64, ctypes.c_uint, _P], _I),
    "focus_scales_swizzled_bytes": ([_I64, _I64], _SZ),
    "focus_scales_swizzle": ([_P, _I64, _I64, _P, _SZ, _P], _I),
    "focus_step_host_workspace_bytes": ([_P, _I], _SZ),
    "focus_step_host": ([_P, _I, ctypes.POINTER(focus_hparams), _I64, ctypes.c_uint, _P, _SZ, _P], _I),
    "focus_get_error": ([_P], _I),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res

EXPORTED = tuple(_SIGS)


class FocusError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_lib.focus_status_string(status).decode()}")


def _check(rc: int, where: str) -> None:
    if rc != FOCUS_OK:
        raise FocusError(rc, where)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if isinstance(x, torch.Tensor):
        if not x.is_cuda:
            raise ValueError("device tensors only (the library computes on the GPU)")
        if not x.is_contiguous():
            raise ValueError("tensors must be contiguous")
        return x.data_ptr()
    raise TypeError(f"cannot pass {type(x)} as a device pointer")


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _bf16(t, name):
    if isinstance(t, torch.Tensor) and t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16")


def _f32(t, name):
    if isinstance(t, torch.Tensor) and t.dtype != torch.float32:
        raise TypeError(f"{name} must be float32")


def _shape(W, out=None, in_=None):
    if out is not None:
        return int(out), int(in_)
    if W.dim() != 2:
        raise ValueError("W must be 2-D [out, in]")
    return int(W.shape[0]), int(W.shape[1])


def focus_version() -> str:
    return _lib.focus_version().decode()


def focus_status_string(status: int) -> str:
    return _lib.focus_status_string(int(status)).decode()


def focus_s2_workspace_bytes(out: int, in_: int) -> int:
    return int(_lib.focus_s2_workspace_bytes(int(out), int(in_)))


def focus_s2(W, s2_out, workspace, stream=None, out=None, in_=None):
    """s2 = amax(|W|)/(6*448) into the one-float device tensor s2_out."""
    _bf16(W, "W"); _f32(s2_out, "s2_out")
    o, i = _shape(W, out, in_)
    nbytes = workspace.numel() * workspace.element_size() if isinstance(workspace, torch.Tensor) else 1 << 62
    _check(_lib.focus_s2(_ptr(W), o, i, _ptr(s2_out), _ptr(workspace), nbytes, _stream(stream)), "focus_s2")


FOCUS_S2_NOALLOC_MAX_WEIGHTS = 268435456


def focus_s2_noalloc(W, s2_out, stream=None, out=None, in_=None):
    """s2 into the one-float device tensor s2_out, without a workspace: for callers
    that cannot hand the library device memory (the per-tile maxima live in a
    fixed array inside the library; tensors of up to FOCUS_S2_NOALLOC_MAX_WEIGHTS
    weights; calls that may overlap on the GPU must not be issued)."""
    _bf16(W, "W"); _f32(s2_out, "s2_out")
    o, i = _shape(W, out, in_)
    _check(_lib.focus_s2_noalloc(_ptr(W), o, i, _ptr(s2_out), _stream(stream)), "focus_s2_noalloc")


def focus_fwd(W, m, q, s2: float, Wq, stream=None, out=None, in_=None):
    _bf16(W, "W"); _bf16(Wq, "Wq"); _f32(m, "m"); _f32(q, "q")
    o, i = _shape(W, out, in_)
    _check(_lib.focus_fwd(_ptr(W), _ptr(m), _ptr(q), float(s2), o, i, _ptr(Wq), _stream(stream)), "focus_fwd")


def focus_ste_bwd(W, dWq, m, q, s2: float, dm, dq, accumulate: bool = False, stream=None, out=None, in_=None):
    _bf16(W, "W"); _bf16(dWq, "dWq"); _f32(m, "m"); _f32(q, "q"); _f32(dm, "dm"); _f32(dq, "dq")
    o, i = _shape(W, out, in_)
    _check(_lib.focus_ste_bwd(_ptr(W), _ptr(dWq), _ptr(m), _ptr(q), float(s2), o, i, _ptr(dm), _ptr(dq),
                              1 if accumulate else 0, _stream(stream)), "focus_ste_bwd")


def focus_adamw_step(p, g, exp_avg, exp_avg_sq, lr: float, step: int, beta1=0.9, beta2=0.999, eps=1e-8,
                     weight_decay=0.0, stream=None, n=None):
    for t, nm in ((p, "p"), (g, "g"), (exp_avg, "exp_avg"), (exp_avg_sq, "exp_avg_sq")):
        _f32(t, nm)
    n = int(p.numel()) if n is None else int(n)
    _check(_lib.focus_adamw_step(_ptr(p), _ptr(g), _ptr(exp_avg), _ptr(exp_avg_sq), n, float(lr), float(beta1),
                                 float(beta2), float(eps), float(weight_decay), int(step), _stream(stream)),
           "focus_adamw_step")


def focus_pack_nvfp4(W, m, q, s2: float, codes, scales, tensor_scale, stream=None, out=None, in_=None):
    _bf16(W, "W"); _f32(m, "m"); _f32(q, "q"); _f32(tensor_scale, "tensor_scale")
    o, i = _shape(W, out, in_)
    _check(_lib.focus_pack_nvfp4(_ptr(W), _ptr(m), _ptr(q), float(s2), o, i, _ptr(codes), _ptr(scales),
                                 _ptr(tensor_scale), _stream(stream)), "focus_pack_nvfp4")


def focus_table_prepare(descs, purpose: int) -> int:
    """Checks a ctypes array of focus_tensor_desc in place; returns total_tiles."""
    tiles = _I64(0)
    _check(_lib.focus_table_prepare(descs, len(descs), int(purpose), ctypes.byref(tiles)), "focus_table_prepare")
    return int(tiles.value)


def focus_s2_multi_workspace_bytes(total_tiles: int) -> int:
    return int(_lib.focus_s2_multi_workspace_bytes(int(total_tiles)))


def focus_s2_multi(table_dev, n: int, total_tiles: int, workspace, stream=None):
    nbytes = workspace.numel() * workspace.element_size()
    _check(_lib.focus_s2_multi(_ptr(table_dev), int(n), int(total_tiles), _ptr(workspace), nbytes,
                               _stream(stream)), "focus_s2_multi")


def focus_step_fused(table_dev, n: int, total_tiles: int, hp: focus_hparams, step: int, flags: int = 0,
                     stream=None):
    _check(_lib.focus_step_fused(_ptr(table_dev), int(n), int(total_tiles), ctypes.byref(hp), int(step),
                                 int(flags), _stream(stream)), "focus_step_fused")


def focus_step_fused_amax(table_dev, n: int, total_tiles: int, hp: focus_hparams, step: int, amax_ws, flags: int = 0,
                          stream=None):
    """focus_step_fused that also accumulates every tensor's max |w| into amax_ws (n int32 words)."""
    _check(_lib.focus_step_fused_amax(_ptr(table_dev), int(n), int(total_tiles), ctypes.byref(hp), int(step),
                                      int(flags), _ptr(amax_ws), _stream(stream)), "focus_step_fused_amax")


def focus_s2_from_amax(table_dev, n: int, amax_ws, stream=None):
    """desc.s2 = fl(max|w| / 2688) from a step's accumulated maxima; clears amax_ws."""
    _check(_lib.focus_s2_from_amax(_ptr(table_dev), int(n), _ptr(amax_ws), _stream(stream)), "focus_s2_from_amax")


def focus_fwd_multi(table_dev, n: int, total_tiles: int, stream=None):
    _check(_lib.focus_fwd_multi(_ptr(table_dev), int(n), int(total_tiles), _stream(stream)), "focus_fwd_multi")


def focus_ste_bwd_multi(table_dev, n: int, total_tiles: int, accumulate: bool = False, stream=None):
    _check(_lib.focus_ste_bwd_multi(_ptr(table_dev), int(n), int(total_tiles), 1 if accumulate else 0,
                                    _stream(stream)), "focus_ste_bwd_multi")


def focus_pack_multi(table_dev, n: int, total_tiles: int, stream=None):
    _check(_lib.focus_pack_multi(_ptr(table_dev), int(n), int(total_tiles), _stream(stream)), "focus_pack_multi")


def focus_fouroversix_weight(W, s2: float, codes, scales, Wq=None, stream=None, out=None, in_=None):
    """FourOverSix round to nearest of a weight with tensor scale s2: codes
    [out, in/2] u8, scales [out, in/16] u8 (both or neither), Wq bf16 (optional)."""
    _bf16(W, "W"); _bf16(Wq, "Wq")
    o, i = _shape(W, out, in_)
    _check(_lib.focus_fouroversix_weight(_ptr(W), o, i, float(s2), _ptr(codes), _ptr(scales), _ptr(Wq),
                                         _stream(stream)), "focus_fouroversix_weight")


def focus_fouroversix_act_multi(table_dev, n: int, total_rows: int, max_hidden: int, swizzled: bool = False,
                                stream=None):
    """FourOverSix with one scale per token over a table of activation tensors
    (prepared with FOCUS_PURPOSE_ACT, or FOCUS_PURPOSE_ACT_SWIZZLED and swizzled)."""
    _check(_lib.focus_fouroversix_act_multi(_ptr(table_dev), int(n), int(total_rows), int(max_hidden),
                                            1 if swizzled else 0, _stream(stream)), "focus_fouroversix_act_multi")


def focus_nvfp4_act_multi(table_dev, n: int, total_rows: int, max_hidden: int, swizzled: bool = False, stream=None):
    """NVFP4 round to nearest with one scale per token over a table of activation tensors."""
    _check(_lib.focus_nvfp4_act_multi(_ptr(table_dev), int(n), int(total_rows), int(max_hidden),
                                      1 if swizzled else 0, _stream(stream)), "focus_nvfp4_act_multi")


def focus_fouroversix_multi(table_dev, n: int, total_tiles: int, stream=None):
    _check(_lib.focus_fouroversix_multi(_ptr(table_dev), int(n), int(total_tiles), _stream(stream)),
           "focus_fouroversix_multi")


def focus_nvfp4_weight(W, s2: float, codes, scales, Wq=None, stream=None, out=None, in_=None):
    """Plain NVFP4 round to nearest of a weight with tensor scale s2 (outputs as
    focus_fouroversix_weight)."""
    _bf16(W, "W"); _bf16(Wq, "Wq")
    o, i = _shape(W, out, in_)
    _check(_lib.focus_nvfp4_weight(_ptr(W), o, i, float(s2), _ptr(codes), _ptr(scales), _ptr(Wq), _stream(stream)),
           "focus_nvfp4_weight")


def focus_nvfp4_weight_multi(table_dev, n: int, total_tiles: int, stream=None):
    _check(_lib.focus_nvfp4_weight_multi(_ptr(table_dev), int(n), int(total_tiles), _stream(stream)),
           "focus_nvfp4_weight_multi")


def focus_fouroversix_act(X, token_scales, codes, scales, Xq=None, stream=None, tokens=None, hidden=None):
    """FourOverSix with one scale per token: token_scales [tokens] f32, codes
    [tokens, hidden/2] u8, scales [tokens, hidden/16] u8, Xq bf16 (optional)."""
    _bf16(X, "X"); _bf16(Xq, "Xq"); _f32(token_scales, "token_scales")
    t, h = _shape(X, tokens, hidden)
    _check(_lib.focus_fouroversix_act(_ptr(X), t, h, _ptr(token_scales), _ptr(codes), _ptr(scales), _ptr(Xq),
                                      _stream(stream)), "focus_fouroversix_act")


def focus_fouroversix_act_swizzled(X, token_scales, codes, scales_swz, Xq=None, stream=None, tokens=None,
                                   hidden=None):
    """FourOverSix with one scale per token, the block scales written in the 128x4-atom
    layout of sm_100 block-scaled GEMMs (scales_swz: focus_scales_swizzled_bytes(tokens,
    hidden/16) bytes)."""
    _bf16(X, "X"); _bf16(Xq, "Xq"); _f32(token_scales, "token_scales")
    t, h = _shape(X, tokens, hidden)
    nbytes = scales_swz.numel() * scales_swz.element_size() if isinstance(scales_swz, torch.Tensor) else 1 << 62
    _check(_lib.focus_fouroversix_act_swizzled(_ptr(X), t, h, _ptr(token_scales), _ptr(codes), _ptr(scales_swz),
                                               nbytes, _ptr(Xq), _stream(stream)), "focus_fouroversix_act_swizzled")


def focus_nvfp4_act(X, token_scales, codes, scales, Xq=None, stream=None, tokens=None, hidden=None):
    """NVFP4 round to nearest with one scale per token (the target 6 alone); outputs
    as focus_fouroversix_act."""
    _bf16(X, "X"); _bf16(Xq, "Xq"); _f32(token_scales, "token_scales")
    t, h = _shape(X, tokens, hidden)
    _check(_lib.focus_nvfp4_act(_ptr(X), t, h, _ptr(token_scales), _ptr(codes), _ptr(scales), _ptr(Xq),
                                _stream(stream)), "focus_nvfp4_act")


def focus_nvfp4_act_swizzled(X, token_scales, codes, scales_swz, Xq=None, stream=None, tokens=None, hidden=None):
    """As focus_nvfp4_act, the block scales in the 128x4-atom layout."""
    _bf16(X, "X"); _bf16(Xq, "Xq"); _f32(token_scales, "token_scales")
    t, h = _shape(X, tokens, hidden)
    nbytes = scales_swz.numel() * scales_swz.element_size() if isinstance(scales_swz, torch.Tensor) else 1 << 62
    _check(_lib.focus_nvfp4_act_swizzled(_ptr(X), t, h, _ptr(token_scales), _ptr(codes), _ptr(scales_swz), nbytes,
                                         _ptr(Xq), _stream(stream)), "focus_nvfp4_act_swizzled")


def focus_mx_fwd(W, m, q, Wq=None, codes=None, scales=None, stream=None, out=None, in_=None):
    """MXFP4 variant forward: m [out, in/32], q [out, in/8]; Wq bf16 and/or codes+scales."""
    _bf16(W, "W"); _bf16(Wq, "Wq"); _f32(m, "m"); _f32(q, "q")
    o, i = _shape(W, out, in_)
    _check(_lib.focus_mx_fwd(_ptr(W), _ptr(m), _ptr(q), o, i, _ptr(Wq), _ptr(codes), _ptr(scales),
                             _stream(stream)), "focus_mx_fwd")


def focus_mx_ste_bwd(W, dWq, m, q, dm, dq, accumulate: bool = False, stream=None, out=None, in_=None):
    _bf16(W, "W"); _bf16(dWq, "dWq"); _f32(m, "m"); _f32(q, "q"); _f32(dm, "dm"); _f32(dq, "dq")
    o, i = _shape(W, out, in_)
    _check(_lib.focus_mx_ste_bwd(_ptr(W), _ptr(dWq), _ptr(m), _ptr(q), o, i, _ptr(dm), _ptr(dq),
                                 1 if accumulate else 0, _stream(stream)), "focus_mx_ste_bwd")


def focus_mx_step(W, dWq, m, q, m_exp_avg, m_exp_avg_sq, q_exp_avg, q_exp_avg_sq, hp: focus_hparams, step: int,
                  flags: int = 0, Wq=None, dm=None, dq=None, stream=None, out=None, in_=None):
    _bf16(W, "W"); _bf16(dWq, "dWq"); _bf16(Wq, "Wq")
    for t, nm in ((m, "m"), (q, "q"), (m_exp_avg, "m_exp_avg"), (m_exp_avg_sq, "m_exp_avg_sq"),
                  (q_exp_avg, "q_exp_avg"), (q_exp_avg_sq, "q_exp_avg_sq"), (dm, "dm"), (dq, "dq")):
        _f32(t, nm)
    o, i = _shape(W, out, in_)
    _check(_lib.focus_mx_step(_ptr(W), _ptr(dWq), _ptr(m), _ptr(q), _ptr(m_exp_avg), _ptr(m_exp_avg_sq),
                              _ptr(q_exp_avg), _ptr(q_exp_avg_sq), o, i, ctypes.byref(hp), int(step), int(flags),
                              _ptr(Wq), _ptr(dm), _ptr(dq), _stream(stream)), "focus_mx_step")


def focus_mx_fwd_multi(table_dev, n: int, total_tiles: int, stream=None):
    """MXFP4 forward over a table prepared with FOCUS_PURPOSE_MX, one launch."""
    _check(_lib.focus_mx_fwd_multi(_ptr(table_dev), int(n), int(total_tiles), _stream(stream)), "focus_mx_fwd_multi")


def focus_mx_ste_bwd_multi(table_dev, n: int, total_tiles: int, accumulate: bool = False, stream=None):
    _check(_lib.focus_mx_ste_bwd_multi(_ptr(table_dev), int(n), int(total_tiles), 1 if accumulate else 0,
                                       _stream(stream)), "focus_mx_ste_bwd_multi")


def focus_mx_step_multi(table_dev, n: int, total_tiles: int, hp: focus_hparams, step: int, flags: int = 0,
                        stream=None):
    _check(_lib.focus_mx_step_multi(_ptr(table_dev), int(n), int(total_tiles), ctypes.byref(hp), int(step),
                                    int(flags), _stream(stream)), "focus_mx_step_multi")


def focus_scales_swizzled_bytes(rows: int, cols: int) -> int:
    return int(_lib.focus_scales_swizzled_bytes(int(rows), int(cols)))


def focus_scales_swizzle(scales, out, stream=None, rows=None, cols=None):
    """E4M3 scales [rows, cols] -> the 128x4-atom layout of sm_100 block-scaled GEMMs (into out)."""
    r, c = _shape(scales, rows, cols)
    nbytes = out.numel() * out.element_size() if isinstance(out, torch.Tensor) else 1 << 62
    _check(_lib.focus_scales_swizzle(_ptr(scales), r, c, _ptr(out), nbytes, _stream(stream)), "focus_scales_swizzle")


def host_ptr(x):
    """Address of a contiguous CPU tensor (for focus_step_host), or None."""
    if x is None:
        return None
    if not isinstance(x, torch.Tensor) or x.is_cuda:
        raise ValueError("host tensors only")
    if not x.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return x.data_ptr() if x.numel() else None


def focus_step_host_workspace_bytes(descs_host, n: int) -> int:
    return int(_lib.focus_step_host_workspace_bytes(descs_host, int(n)))


def focus_step_host(descs_host, n: int, hp: focus_hparams, step: int, flags: int, ws, stream=None):
    """The fused step over tensors in host memory (descs_host: a focus_tensor_desc array
    holding host pointers); blocks until every result is back in host memory."""
    nbytes = ws.numel() * ws.element_size() if isinstance(ws, torch.Tensor) else 1 << 62
    _check(_lib.focus_step_host(descs_host, int(n), ctypes.byref(hp), int(step), int(flags), _ptr(ws), nbytes,
                                _stream(stream)), "focus_step_host")


def focus_get_error(stream=None) -> int:
    """Synchronizes the stream and returns (and clears) the sticky device status."""
    return int(_lib.focus_get_error(_stream(stream)))


def raw_call(name: str, *args):
    """Call an entry point with raw ctypes arguments (addresses as ints); returns the status."""
    return getattr(_lib, name)(*args)
