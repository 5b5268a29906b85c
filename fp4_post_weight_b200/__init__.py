"""FOCUS NVFP4 weight fake-quantizer on B200 (sm_100a).

The kernels live in libfocus.so (C ABI: include/focus.h); ``focus`` is its
ctypes binding and ``table`` the multi-tensor helper.  Importing this package
does not load the library; the first use of a binding name does, and raises
ImportError when libfocus.so has not been built (there is no CPU fallback).
"""
import importlib

__all__ = ["focus", "table", "build"]

_BINDING_NAMES = {"focus_s2", "focus_fwd", "focus_ste_bwd", "focus_adamw_step", "focus_pack_nvfp4",
                  "focus_table_prepare", "focus_s2_multi", "focus_step_fused", "focus_pack_multi",
                  "focus_fwd_multi", "focus_ste_bwd_multi", "focus_s2_noalloc",
                  "focus_fouroversix_weight", "focus_fouroversix_multi", "focus_fouroversix_act",
                  "focus_fouroversix_act_swizzled",
                  "focus_nvfp4_act", "focus_nvfp4_act_swizzled",
                  "focus_nvfp4_weight", "focus_nvfp4_weight_multi",
                  "focus_scales_swizzle", "focus_scales_swizzled_bytes", "focus_mx_fwd", "focus_mx_ste_bwd",
                  "focus_mx_step", "focus_mx_fwd_multi", "focus_mx_ste_bwd_multi", "focus_mx_step_multi",
                  "focus_step_host", "focus_step_host_workspace_bytes",
                  "focus_step_fused_amax", "focus_s2_from_amax",
                  "focus_get_error", "focus_s2_workspace_bytes", "focus_s2_multi_workspace_bytes",
                  "focus_status_string", "focus_version", "FocusError", "focus_tensor_desc", "focus_hparams"}


def __getattr__(name):
    if name in ("focus", "table", "build"):
        return importlib.import_module(f"{__name__}.{name}")
    if name in _BINDING_NAMES:
        return getattr(importlib.import_module(f"{__name__}.focus"), name)
    if name in ("FocusTable", "Entry", "hparams"):
        return getattr(importlib.import_module(f"{__name__}.table"), name)
    raise AttributeError(name)
