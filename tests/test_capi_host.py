"""The C-ABI library loads, exports every function include/focus.h declares,
and rejects bad arguments on the host before touching a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def F():
    from fp4_post_weight_b200 import build
    build.build()
    from fp4_post_weight_b200 import focus
    return focus


def declared_functions():
    src = open(os.path.join(ROOT, "include", "focus.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(focus_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_function(F):
    names = declared_functions()
    assert len(names) >= 14
    lib = ctypes.CDLL(F._LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(F.EXPORTED)


def test_status_strings(F):
    for s in range(9):
        assert F.focus_status_string(s).startswith("FOCUS_")
    assert F.focus_version() == "0.1.0"


P = 0x7f0000001000  # an aligned address that is never dereferenced: every call below fails its checks first
U = 0x7f0000001004  # misaligned
call = None


def _c(F, name, *a):
    return F.raw_call(name, *a)


def test_shape_and_value_checks(F):
    f32 = ctypes.c_float
    E = F
    assert _c(F, "focus_fwd", P, P, P, f32(1.0), 4, 15, P, None) == 2          # in % 16
    assert _c(F, "focus_fwd", P, P, P, f32(1.0), -1, 16, P, None) == 2         # out < 0
    assert _c(F, "focus_fwd", P, P, P, f32(0.0), 4, 16, P, None) == 4          # s2 <= 0
    assert _c(F, "focus_fwd", P, P, P, f32(float("inf")), 4, 16, P, None) == 4
    assert _c(F, "focus_fwd", P, P, P, f32(float("nan")), 4, 16, P, None) == 4
    assert _c(F, "focus_fwd", None, P, P, f32(1.0), 4, 16, P, None) == 1       # NULL
    assert _c(F, "focus_fwd", U, P, P, f32(1.0), 4, 16, P, None) == 3          # misaligned
    assert _c(F, "focus_fwd", P, P, P, f32(1.0), 0, 16, P, None) == 0          # empty: no-op
    assert _c(F, "focus_ste_bwd", P, P, P, P, f32(1.0), 4, 16, P, P, 2, None) == 4  # accumulate flag
    assert _c(F, "focus_ste_bwd", P, None, P, P, f32(1.0), 4, 16, P, P, 0, None) == 1
    assert _c(F, "focus_pack_nvfp4", P, P, P, f32(1.0), 4, 16, P, P, None, None) == 1
    assert _c(F, "focus_s2", P, 4, 16, P, P, 0, None) == 5                     # workspace too small
    assert _c(F, "focus_s2", P, 4, 24, P, P, 64, None) == 2
    assert F.focus_s2_workspace_bytes(4, 16) == 4
    assert F.focus_s2_workspace_bytes(2048, 2048) == 4 * (2048 * 128 // 256)


def test_adamw_checks(F):
    f = ctypes.c_float
    args = lambda lr, b1, b2, eps, wd, step: (P, P, P, P, 8, f(lr), f(b1), f(b2), f(eps), f(wd), step, None)
    assert _c(F, "focus_adamw_step", *args(1e-3, 0.9, 0.999, 1e-8, 0.0, 0)) == 4
    assert _c(F, "focus_adamw_step", *args(-1e-3, 0.9, 0.999, 1e-8, 0.0, 1)) == 4
    assert _c(F, "focus_adamw_step", *args(1e-3, 1.0, 0.999, 1e-8, 0.0, 1)) == 4
    assert _c(F, "focus_adamw_step", *args(1e-3, 0.9, 0.999, -1.0, 0.0, 1)) == 4
    assert _c(F, "focus_adamw_step", P, P, P, P, -1, f(1e-3), f(0.9), f(0.999), f(1e-8), f(0), 1, None) == 2
    assert _c(F, "focus_adamw_step", U, P, P, P, 8, f(1e-3), f(0.9), f(0.999), f(1e-8), f(0), 1, None) == 3


def test_table_prepare_on_host(F):
    n = 3
    shapes = [(4, 32), (1, 16), (300, 4096)]
    descs = (F.focus_tensor_desc * n)()
    for i, (o, k) in enumerate(shapes):
        d = descs[i]
        for name in ("W", "dWq", "Wq", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq", "s2"):
            setattr(d, name, P + 4096 * (i + 1))
        d.out, d.in_ = o, k
    tiles = F.focus_table_prepare(descs, 1)
    nblk = [o * k // 16 for o, k in shapes]
    assert [descs[i].block_begin for i in range(n)] == [0, nblk[0], nblk[0] + nblk[1]]
    t = [(b + 255) // 256 for b in nblk]
    assert [descs[i].tile_begin for i in range(n)] == [0, t[0], t[0] + t[1]]
    assert tiles == sum(t)
    # a step needs the moments and dW'
    descs[1].q_exp_avg = None
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, 1)
    assert e.value.status == 1
    assert F.focus_table_prepare(descs, 0) == tiles
    # a table backward needs dW', dm and dq; purposes beyond 6 do not exist
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, 2)
    assert e.value.status == 1
    for i in range(n):
        descs[i].dm = P + 65536 * (i + 1)
        descs[i].dq = P + 65536 * (i + 1) + 4096
    assert F.focus_table_prepare(descs, 2) == tiles
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, 7)
    assert e.value.status == 4
    with pytest.raises(F.FocusError) as e:      # MXFP4: in must be a multiple of 32
        F.focus_table_prepare(descs, F.FOCUS_PURPOSE_MX)
    assert e.value.status == 2
    descs[2].in_ = 40
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, 0)
    assert e.value.status == 2
    descs[2].in_ = 4096
    descs[2].m = U
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, 0)
    assert e.value.status == 3


def test_table_prepare_mx(F):
    """A table for the MXFP4 calls: 32-blocks, tiles of 128 of them (4096 weights),
    W, m and q required, s2 not needed, pointers both-or-neither as elsewhere."""
    shapes = [(4, 32), (3, 96), (300, 4096), (0, 64)]
    n = len(shapes)
    descs = (F.focus_tensor_desc * n)()
    for i, (o, k) in enumerate(shapes):
        d = descs[i]
        for name in ("W", "m", "q"):
            setattr(d, name, P + 4096 * (i + 1))
        d.out, d.in_ = o, k
    tiles = F.focus_table_prepare(descs, F.FOCUS_PURPOSE_MX)
    nblk = [o * k // 32 for o, k in shapes]
    t = [(b + 127) // 128 for b in nblk]
    assert [descs[i].block_begin for i in range(n)] == [sum(nblk[:i]) for i in range(n)]
    assert [descs[i].tile_begin for i in range(n)] == [sum(t[:i]) for i in range(n)]
    assert tiles == sum(t) == 1 + 1 + 300 + 0
    descs[1].codes = P                          # codes without scales
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, F.FOCUS_PURPOSE_MX)
    assert e.value.status == 1
    descs[1].scales = P
    descs[1].dm = P                             # dm without dq
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, F.FOCUS_PURPOSE_MX)
    assert e.value.status == 1
    descs[1].dq = U                             # misaligned
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, F.FOCUS_PURPOSE_MX)
    assert e.value.status == 3
    descs[1].dm = descs[1].dq = None
    descs[2].q = None
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, F.FOCUS_PURPOSE_MX)
    assert e.value.status == 1
    descs[2].q = P
    descs[0].in_ = 48
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, F.FOCUS_PURPOSE_MX)
    assert e.value.status == 2


def test_mx_multi_checks(F):
    hp = F.focus_hparams(5e-3, 1e-3, 0.9, 0.999, 1e-8, 0.0)
    assert F.raw_call("focus_mx_fwd_multi", P, -1, 1, None) == 4
    assert F.raw_call("focus_mx_fwd_multi", None, 1, 1, None) == 1
    assert F.raw_call("focus_mx_fwd_multi", U, 1, 1, None) == 3
    assert F.raw_call("focus_mx_fwd_multi", None, 0, 0, None) == 0            # nothing to do
    assert F.raw_call("focus_mx_ste_bwd_multi", P, 1, 1, 2, None) == 4        # accumulate must be 0 or 1
    assert F.raw_call("focus_mx_ste_bwd_multi", None, 1, 1, 0, None) == 1
    assert F.raw_call("focus_mx_step_multi", P, 1, 1, None, 1, 0, None) == 1
    assert F.raw_call("focus_mx_step_multi", P, 1, 1, ctypes.byref(hp), 0, 0, None) == 4    # step >= 1
    assert F.raw_call("focus_mx_step_multi", P, 1, 1, ctypes.byref(hp), 1, 16, None) == 4   # not a step flag
    assert F.raw_call("focus_mx_step_multi", U, 1, 1, ctypes.byref(hp), 1, 0, None) == 3


def test_step_host_checks(F):
    """focus_step_host checks every entry on the host before it enqueues anything."""
    hp = F.focus_hparams(5e-3, 1e-3, 0.9, 0.999, 1e-8, 0.0)
    S = ctypes.c_size_t
    s2 = (ctypes.c_float * 2)(0.01, 0.0)
    descs = (F.focus_tensor_desc * 2)()
    for i, (o, k) in enumerate([(4, 32), (3, 16)]):
        d = descs[i]
        for name in ("W", "dWq", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq"):
            setattr(d, name, P)
        d.s2 = ctypes.addressof(s2) + 4 * i
        d.out, d.in_ = o, k
    need = F.focus_step_host_workspace_bytes(descs, 2)
    # three slots of the largest tensor (128 weights): about 8.8 bytes per weight plus fields
    assert 3 * 8.8125 * 128 <= need <= 3 * (8.8125 * 128 + 16 * 256)
    W = 1 << 40                                   # a 256-byte aligned address, never dereferenced
    call = lambda *a: F.raw_call("focus_step_host", *a)
    assert call(descs, -1, ctypes.byref(hp), 1, 0, W, S(need), None) == 4
    assert call(descs, 2, None, 1, 0, W, S(need), None) == 1
    assert call(descs, 2, ctypes.byref(hp), 1, 1, W, S(need), None) == 4          # ACCUMULATE: not on this path
    assert call(descs, 0, ctypes.byref(hp), 1, 0, None, S(0), None) == 0
    assert call(None, 2, ctypes.byref(hp), 1, 0, W, S(need), None) == 1
    assert call(descs, 2, ctypes.byref(hp), 1, 0, W, S(need), None) == 4          # entry 1: s2 = 0
    assert call(descs, 1, ctypes.byref(hp), 1, 0, None, S(need), None) == 1       # no workspace
    assert call(descs, 1, ctypes.byref(hp), 1, 0, W + 16, S(need), None) == 3     # not 256-byte aligned
    assert call(descs, 1, ctypes.byref(hp), 1, 0, W, S(need - 1), None) == 5
    s2[1] = 0.02
    descs[1].in_ = 24
    assert call(descs, 2, ctypes.byref(hp), 1, 0, W, S(need), None) == 2
    assert F.focus_step_host_workspace_bytes(descs, 2) == 0
    descs[1].in_ = 16
    descs[1].q_exp_avg = None
    assert call(descs, 2, ctypes.byref(hp), 1, 0, W, S(need), None) == 1
    descs[1].q_exp_avg = P
    descs[1].dm = P
    assert call(descs, 2, ctypes.byref(hp), 1, 0, W, S(need), None) == 4          # no gradient buffers
    descs[1].dm = None
    descs[1].codes = P                                                             # codes without scales
    assert call(descs, 2, ctypes.byref(hp), 1, 0, W, S(need), None) == 1


def test_multi_entry_checks(F):
    assert F.raw_call("focus_ste_bwd_multi", P, 1, 1, 2, None) == 4        # accumulate must be 0 or 1
    assert F.raw_call("focus_ste_bwd_multi", None, 1, 1, 0, None) == 1
    assert F.raw_call("focus_fwd_multi", U, 1, 1, None) == 3
    assert F.raw_call("focus_fwd_multi", P, -1, 1, None) == 4
    assert F.raw_call("focus_fwd_multi", P, 0, 0, None) == 0                  # empty table: nothing to do


def test_step_hparam_checks(F):
    hp = F.focus_hparams(5e-3, 1e-3, 0.9, 0.999, 1e-8, 0.0)
    assert F.raw_call("focus_step_fused", P, 1, 1, ctypes.byref(hp), 0, 0, None) == 4
    # unknown flag bits (every call here fails its host checks: nothing is launched)
    assert F.raw_call("focus_step_fused", P, 1, 1, ctypes.byref(hp), 1, 16, None) == 4
    assert F.raw_call("focus_step_fused", P, 1, 1, ctypes.byref(hp), 1, 32 | 1, None) == 4
    assert F.raw_call("focus_step_fused", P, 1, 1, None, 1, 0, None) == 1
    bad = F.focus_hparams(5e-3, -1e-3, 0.9, 0.999, 1e-8, 0.0)
    assert F.raw_call("focus_step_fused", P, 1, 1, ctypes.byref(bad), 1, 0, None) == 4


def test_fouroversix_checks(F):
    f32 = ctypes.c_float
    # weights: shape, tensor scale, outputs (codes and scales together; codes or Wq), alignment
    assert F.raw_call("focus_fouroversix_weight", P, 4, 24, f32(1.0), P, P, None, None) == 2
    assert F.raw_call("focus_fouroversix_weight", P, 4, 16, f32(0.0), P, P, None, None) == 4
    assert F.raw_call("focus_fouroversix_weight", P, 4, 16, f32(float("nan")), P, P, None, None) == 4
    assert F.raw_call("focus_fouroversix_weight", P, 4, 16, f32(1.0), P, None, None, None) == 1
    assert F.raw_call("focus_fouroversix_weight", P, 4, 16, f32(1.0), None, None, None, None) == 1
    assert F.raw_call("focus_fouroversix_weight", None, 4, 16, f32(1.0), P, P, None, None) == 1
    assert F.raw_call("focus_fouroversix_weight", U, 4, 16, f32(1.0), P, P, None, None) == 3
    assert F.raw_call("focus_fouroversix_weight", P, 4, 16, f32(1.0), None, None, U, None) == 3
    assert F.raw_call("focus_fouroversix_weight", P, 0, 16, f32(1.0), P, P, None, None) == 0   # empty
    assert F.raw_call("focus_fouroversix_multi", P, -1, 1, None) == 4
    assert F.raw_call("focus_fouroversix_multi", None, 1, 1, None) == 1
    assert F.raw_call("focus_fouroversix_multi", U, 1, 1, None) == 3
    # plain NVFP4 weights: the same checks
    assert F.raw_call("focus_nvfp4_weight", P, 4, 24, f32(1.0), P, P, None, None) == 2
    assert F.raw_call("focus_nvfp4_weight", P, 4, 16, f32(0.0), P, P, None, None) == 4
    assert F.raw_call("focus_nvfp4_weight", P, 4, 16, f32(1.0), None, None, None, None) == 1
    assert F.raw_call("focus_nvfp4_weight", U, 4, 16, f32(1.0), P, P, None, None) == 3
    assert F.raw_call("focus_nvfp4_weight_multi", P, -1, 1, None) == 4
    assert F.raw_call("focus_nvfp4_weight_multi", None, 1, 1, None) == 1
    # activations: per-token scales, codes and scales are required
    assert F.raw_call("focus_fouroversix_act", P, 4, 40, P, P, P, None, None) == 2
    assert F.raw_call("focus_fouroversix_act", P, 4, 32, None, P, P, None, None) == 1
    assert F.raw_call("focus_fouroversix_act", P, 4, 32, P, None, P, None, None) == 1
    assert F.raw_call("focus_fouroversix_act", P, 4, 32, P, P, P, U, None) == 3
    assert F.raw_call("focus_fouroversix_act", P, 0, 32, P, P, P, None, None) == 0             # no tokens
    # the same with the scales in the 128x4 layout: its size is checked too
    S = ctypes.c_size_t
    need = F.focus_scales_swizzled_bytes(4, 2)           # 128 rows x 4 columns
    assert need == 512
    sw = "focus_fouroversix_act_swizzled"
    assert F.raw_call(sw, P, 4, 40, P, P, P, S(need), None, None) == 2
    assert F.raw_call(sw, P, 4, 32, None, P, P, S(need), None, None) == 1
    assert F.raw_call(sw, P, 4, 32, P, None, P, S(need), None, None) == 1
    assert F.raw_call(sw, P, 4, 32, P, P, None, S(need), None, None) == 1
    assert F.raw_call(sw, P, 4, 32, P, P, U, S(need), None, None) == 3
    assert F.raw_call(sw, P, 4, 32, P, P, P, S(need), U, None) == 3
    assert F.raw_call(sw, P, 4, 32, P, P, P, S(need - 1), None, None) == 5
    assert F.raw_call(sw, P, 0, 32, P, P, P, S(0), None, None) == 0                # no tokens
    # plain NVFP4 per token: the same checks
    assert F.raw_call("focus_nvfp4_act", P, 4, 40, P, P, P, None, None) == 2
    assert F.raw_call("focus_nvfp4_act", P, 4, 32, None, P, P, None, None) == 1
    assert F.raw_call("focus_nvfp4_act", P, 4, 32, P, P, P, U, None) == 3
    assert F.raw_call("focus_nvfp4_act", P, 0, 32, P, P, P, None, None) == 0
    assert F.raw_call("focus_nvfp4_act_swizzled", P, 4, 32, P, P, P, S(need - 1), None, None) == 5
    assert F.raw_call("focus_nvfp4_act_swizzled", P, 4, 32, P, P, None, S(need), None, None) == 1


def test_table_prepare_fouroversix(F):
    descs = (F.focus_tensor_desc * 2)()
    for i, (o, k) in enumerate([(8, 64), (3, 32)]):
        d = descs[i]
        d.W = P + 4096 * i; d.s2 = P + 65536 + 16 * i
        d.out, d.in_ = o, k
    with pytest.raises(F.FocusError) as e:          # nothing to write
        F.focus_table_prepare(descs, 3)
    assert e.value.status == 1
    for i in range(2):
        descs[i].Wq = P + 131072 + 4096 * i
    assert F.focus_table_prepare(descs, 3) == 2     # m and q are not needed
    with pytest.raises(F.FocusError) as e:          # the FOCUS purposes still need m and q
        F.focus_table_prepare(descs, 0)
    assert e.value.status == 1


def test_swizzle_checks(F):
    assert F.focus_scales_swizzled_bytes(1, 1) == 512
    assert F.focus_scales_swizzled_bytes(130, 6) == 256 * 8
    assert F.focus_scales_swizzled_bytes(0, 7) == 0
    assert F.raw_call("focus_scales_swizzle", P, -1, 4, P, 4096, None) == 2
    assert F.raw_call("focus_scales_swizzle", P, 0, 4, P, 0, None) == 0          # nothing to write
    assert F.raw_call("focus_scales_swizzle", P, 4, 4, None, 4096, None) == 1
    assert F.raw_call("focus_scales_swizzle", None, 4, 4, P, 4096, None) == 1
    assert F.raw_call("focus_scales_swizzle", P, 4, 4, U, 4096, None) == 3
    assert F.raw_call("focus_scales_swizzle", P, 4, 4, P, 511, None) == 5        # output too small


def test_mx_checks(F):
    f32 = ctypes.c_float
    hp = F.focus_hparams(5e-3, 1e-3, 0.9, 0.999, 1e-8, 0.0)
    assert F.raw_call("focus_mx_fwd", P, P, P, 4, 48, P, None, None, None) == 2      # in % 32
    assert F.raw_call("focus_mx_fwd", P, P, P, 4, 32, None, None, None, None) == 1   # no output
    assert F.raw_call("focus_mx_fwd", P, P, P, 4, 32, None, P, None, None) == 1      # codes without scales
    assert F.raw_call("focus_mx_fwd", U, P, P, 4, 32, P, None, None, None) == 3
    assert F.raw_call("focus_mx_fwd", P, P, P, 0, 32, P, None, None, None) == 0      # empty
    assert F.raw_call("focus_mx_ste_bwd", P, P, P, P, 4, 32, P, P, 2, None) == 4     # accumulate flag
    assert F.raw_call("focus_mx_ste_bwd", P, None, P, P, 4, 32, P, P, 0, None) == 1
    args = lambda step, flags, dm: (P, P, P, P, P, P, P, P, 4, 32, ctypes.byref(hp), step, flags, None, dm, dm, None)
    assert F.raw_call("focus_mx_step", *args(0, 0, None)) == 4                       # step < 1
    assert F.raw_call("focus_mx_step", *args(1, 4, None)) == 4                       # no codes buffer: no pack flag
    assert F.raw_call("focus_mx_step", *args(1, 16, None)) == 4                      # not a step flag
    assert F.raw_call("focus_mx_step", *args(1, 1, None)) == 1                       # accumulate needs dm, dq
    assert F.raw_call("focus_mx_step", P, P, P, P, P, P, P, P, 4, 32, None, 1, 0, None, None, None, None) == 1


def test_maximum_tensor_size(F):
    """A tensor of more than 2^31 - 2^16 blocks is rejected on the host (block
    indices inside a tensor stay 32-bit in the kernels); nothing is launched."""
    f32 = ctypes.c_float
    rows = 32768
    in16 = 16 * 65536                 # 65,536 16-blocks per row: 2^31 blocks in all
    assert _c(F, "focus_fwd", P, P, P, f32(1.0), rows, in16, P, None) == 2
    assert _c(F, "focus_ste_bwd", P, P, P, P, f32(1.0), rows, in16, P, P, 0, None) == 2
    assert _c(F, "focus_pack_nvfp4", P, P, P, f32(1.0), rows, in16, P, P, P, None) == 2
    assert _c(F, "focus_s2", P, rows, in16, P, P, 1 << 40, None) == 2
    assert F.focus_s2_workspace_bytes(rows, in16) == 0
    assert F.raw_call("focus_fouroversix_weight", P, rows, in16, f32(1.0), P, P, None, None) == 2
    assert F.raw_call("focus_fouroversix_act", P, rows, in16, P, P, P, None, None) == 2
    assert F.raw_call("focus_fouroversix_act_swizzled", P, rows, in16, P, P, P, ctypes.c_size_t(1 << 40), None,
                      None) == 2
    assert F.raw_call("focus_nvfp4_act", P, rows, in16, P, P, P, None, None) == 2
    in32 = 32 * 65536                 # MXFP4: 65,536 32-blocks per row
    assert F.raw_call("focus_mx_fwd", P, P, P, rows, in32, P, None, None, None) == 2
    descs = (F.focus_tensor_desc * 1)()
    descs[0].W = descs[0].m = descs[0].q = descs[0].s2 = P
    descs[0].out, descs[0].in_ = rows, in16
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, 0)
    assert e.value.status == 2


def test_step_amax_checks(F):
    hp = F.focus_hparams(5e-3, 1e-3, 0.9, 0.999, 1e-8, 0.0)
    assert F.raw_call("focus_step_fused_amax", P, 1, 1, ctypes.byref(hp), 1, 0, None, None) == 1   # no workspace
    assert F.raw_call("focus_step_fused_amax", P, 1, 1, ctypes.byref(hp), 1, 0, U, None) == 3
    assert F.raw_call("focus_step_fused_amax", P, 1, 1, ctypes.byref(hp), 0, 0, P, None) == 4      # step < 1
    assert F.raw_call("focus_s2_from_amax", P, -1, P, None) == 4
    assert F.raw_call("focus_s2_from_amax", P, 1, None, None) == 1
    assert F.raw_call("focus_s2_from_amax", U, 1, P, None) == 3
    assert F.raw_call("focus_s2_from_amax", P, 0, P, None) == 0


def test_activation_table_prepare_on_host():
    """Purposes 5 and 6 (activation tables for the per-token calls): tile_begin is
    each entry's first bundle of rows (rows padded to 128 for the 128x4 layout),
    the total is the bundle count, an empty entry adds none, rows above 16384
    values and entries without codes, scales or token scales are refused."""
    from fp4_post_weight_b200 import focus as F
    P = 1 << 20
    shapes = [(33, 4096), (0, 64), (130, 1040), (5, 16384)]
    descs = (F.focus_tensor_desc * len(shapes))()
    for i, (t, h) in enumerate(shapes):
        d = descs[i]
        d.W, d.s2, d.codes, d.scales = P + (i << 24), P + (i << 24) + 4096, P + (i << 24) + 8192, P + (i << 24) + 16384
        d.out, d.in_ = t, h
    # work units are bundles of rows: 4 rows of 4096 values (64 threads each), 8 of 1040
    # (32 threads each, at most 4 blocks per thread), 1 of 16384
    assert F.focus_table_prepare(descs, F.FOCUS_PURPOSE_ACT) == 9 + 17 + 5
    assert [descs[i].tile_begin for i in range(4)] == [0, 9, 9, 26]
    assert F.focus_table_prepare(descs, F.FOCUS_PURPOSE_ACT_SWIZZLED) == 32 + 32 + 128
    assert [descs[i].tile_begin for i in range(4)] == [0, 32, 32, 64]
    descs[2].codes = None
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, F.FOCUS_PURPOSE_ACT)
    assert e.value.status == 1
    descs[2].codes = P + (2 << 24) + 8192
    descs[3].in_ = 16400
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, F.FOCUS_PURPOSE_ACT)
    assert e.value.status == 2
    descs[3].in_ = 16384
    descs[0].s2 = P + 2                                # token scales not 16-byte aligned
    with pytest.raises(F.FocusError) as e:
        F.focus_table_prepare(descs, F.FOCUS_PURPOSE_ACT)
    assert e.value.status == 3
