"""The 128x4-atom scale layout on the GPU: the relayout kernel against the
oracle (bit for bit), and both against a real consumer -- PyTorch's NVFP4
scaled_mm, i.e. cuBLASLt's block-scaled GEMM on sm_100 -- fed with the
library's NVFP4 export of weights (codes, swizzled scales, tensor scale) and
its FourOverSix activations (codes, swizzled scales, one scale per token).
The GEMM result, times the tensor and token scales, must match the product of
the dequantized operands; with the scales left in row-major order it must not
(the negative control shows the test can see a wrong layout)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity import host, host_bits, unpack_codes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    from fp4_post_weight_b200 import focus
    return focus


def swizzle_gpu(F, scales):
    out = torch.full((F.focus_scales_swizzled_bytes(*scales.shape),), 0xAB, dtype=torch.uint8, device="cuda")
    F.focus_scales_swizzle(scales, out)
    return out


@pytest.mark.parametrize("rows,cols", [(1, 1), (128, 4), (130, 6), (300, 64), (37, 9), (1024, 256)])
def test_swizzle_matches_oracle(F, rows, cols):
    g = torch.Generator(device="cuda").manual_seed(rows * 1000 + cols)
    sc = torch.randint(1, 255, (rows, cols), generator=g, device="cuda", dtype=torch.int32).to(torch.uint8)
    out = swizzle_gpu(F, sc)
    assert F.focus_get_error() == 0
    np.testing.assert_array_equal(host(out), oracle.scales_swizzle(host(sc)))


@pytest.mark.parametrize("tokens,hidden", [(1, 16), (5, 96), (128, 64), (130, 1040), (300, 4096), (33, 14336)])
def test_fouroversix_act_swizzled_matches_oracle(F, tokens, hidden):
    """Per-token FourOverSix writing its scales straight into the 128x4 layout: the
    oracle's quantization followed by the oracle's relayout, bit for bit, padding
    included (the buffer starts filled with 0xAB)."""
    X = synth.activations(tokens, hidden, "cuda", seed=7 * tokens + hidden, zero_tokens=1 if tokens > 2 else 0)
    ts = torch.full((tokens,), -1.0, device="cuda")
    codes = torch.empty((tokens, hidden // 2), dtype=torch.uint8, device="cuda")
    Xq = torch.empty_like(X)
    sw = torch.full((F.focus_scales_swizzled_bytes(tokens, hidden // 16),), 0xAB, dtype=torch.uint8, device="cuda")
    F.focus_fouroversix_act_swizzled(X, ts, codes, sw, Xq)
    assert F.focus_get_error() == 0
    ref = oracle.fouroversix(host_bits(X))
    np.testing.assert_array_equal(host(ts), ref.row_scales)
    np.testing.assert_array_equal(unpack_codes(host(codes)), ref.codes)
    np.testing.assert_array_equal(host_bits(Xq), ref.Xq)
    np.testing.assert_array_equal(host(sw), oracle.scales_swizzle(ref.scales))


def test_fouroversix_act_swizzled_nonfinite_row(F):
    """A row holding infinity sets the device flag and leaves its outputs unwritten
    (its scale bytes, padding columns included, keep the fill); the other rows match
    the oracle."""
    tokens, hidden = 6, 96                                 # 6 scale columns: 2 padding columns per row
    X = synth.activations(tokens, hidden, "cuda", seed=3, zero_tokens=0)
    X[2, 17] = float("inf")
    ts = torch.zeros(tokens, device="cuda")
    codes = torch.zeros((tokens, hidden // 2), dtype=torch.uint8, device="cuda")
    sw = torch.full((F.focus_scales_swizzled_bytes(tokens, hidden // 16),), 0xAB, dtype=torch.uint8, device="cuda")
    assert F.focus_get_error() == 0
    F.focus_fouroversix_act_swizzled(X, ts, codes, sw)
    assert F.focus_get_error() == 7
    Xh = host_bits(X)
    good = [r for r in range(tokens) if r != 2]
    ref = oracle.fouroversix(Xh[good])
    lin = np.zeros((tokens, hidden // 16), np.uint8)
    lin[good] = ref.scales
    want = oracle.scales_swizzle(lin)
    got = host(sw)
    # the bytes of row 2 in the layout: a 1-row marker pushed through the oracle's relayout
    mark = np.zeros((tokens, hidden // 16), np.uint8)
    mark[2] = 1
    row2 = oracle.scales_swizzle(mark) == 1
    mark_pad = np.zeros((tokens, 8), np.uint8)
    mark_pad[2, 6:] = 1
    row2_pad = oracle.scales_swizzle(mark_pad) == 1
    assert np.all(got[row2] == 0xAB) and np.all(got[row2_pad] == 0xAB)
    rest = ~(row2 | row2_pad)
    np.testing.assert_array_equal(got[rest], want[rest])
    np.testing.assert_array_equal(unpack_codes(host(codes))[good], ref.codes)
    assert np.all(host(codes)[2] == 0)


E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)


def e4m3_values(b):
    b = np.asarray(b, np.int64)
    e, m = (b >> 3) & 15, b & 7
    return np.where(e == 0, m * 2.0 ** -9, (1 + m / 8) * 2.0 ** (e - 7))


def dequant(codes_packed, scales):
    """c * S per element, binary64 (the tensor / token scale applied by the caller)."""
    c = E2M1[unpack_codes(codes_packed)]
    S = np.repeat(e4m3_values(scales), 16, axis=1)
    return c * S


def nvfp4_gemm(a_codes, a_sc, b_codes, b_sc, M, N, K):
    """sum_k (c_a S_a)(c_b S_b) through PyTorch's block-scaled NVFP4 GEMM; the scale
    arguments are the flat 128x4-atom buffers."""
    import torch.nn.functional as Fn
    a = a_codes.view(torch.float4_e2m1fn_x2)                      # [M, K/2]
    b = b_codes.view(torch.float4_e2m1fn_x2).t()                  # [K/2, N], column-major
    sa = a_sc.view(torch.float8_e4m3fn).view(-(-M // 128) * 128, -(-(K // 16) // 4) * 4)
    sb = b_sc.view(torch.float8_e4m3fn).view(-(-N // 128) * 128, -(-(K // 16) // 4) * 4)
    return Fn.scaled_mm(a, b, sa, Fn.ScalingType.BlockWise1x16, sb, Fn.ScalingType.BlockWise1x16,
                        swizzle_a=Fn.SwizzleType.SWIZZLE_32_4_4, swizzle_b=Fn.SwizzleType.SWIZZLE_32_4_4,
                        output_dtype=torch.bfloat16).float()


def check_product(Y, ref, bound, what):
    err = np.abs(host(Y).astype(np.float64) - ref)
    # bf16 output (2^-9 relative) plus fp32 accumulation over K terms
    ok = err <= 2.0 ** -7 * bound + 1e-30
    assert ok.all(), f"{what}: {int((~ok).sum())} of {ok.size} outputs off; max err/bound {np.max(err / (bound + 1e-30)):.3g}"


def test_export_feeds_sm100_block_scaled_gemm(F):
    M, N, K = 256, 384, 1024
    X = synth.activations(M, K, "cuda", seed=11, zero_tokens=0)
    g = torch.Generator(device="cuda").manual_seed(12)
    W = synth.normal_bf16((N, K), 0.02, g, "cuda")
    m = synth.uniform((N, K // 16), 0.8, 1.2, g, "cuda")
    q = synth.normal((N, K // 8), 6.0, 2.0, g, "cuda")
    # activations: FourOverSix, one scale per token; weights: the FOCUS NVFP4 export
    ts = torch.empty(M, device="cuda")
    xc = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    xs = torch.empty((M, K // 16), dtype=torch.uint8, device="cuda")
    F.focus_fouroversix_act(X, ts, xc, xs)
    ws = torch.empty(F.focus_s2_workspace_bytes(N, K), dtype=torch.uint8, device="cuda")
    s2d = torch.zeros(1, device="cuda")
    F.focus_s2(W, s2d, ws)
    s2 = float(host(s2d)[0])
    wc = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    wsc = torch.empty((N, K // 16), dtype=torch.uint8, device="cuda")
    F.focus_pack_nvfp4(W, m, q, s2, wc, wsc, torch.zeros(1, device="cuda"))
    xs_sw, ws_sw = swizzle_gpu(F, xs), swizzle_gpu(F, wsc)
    # the per-token quantizer that writes the 128x4 layout itself gives the same bytes
    xs_fused = torch.empty_like(xs_sw)
    xc_fused = torch.empty_like(xc)
    F.focus_fouroversix_act_swizzled(X, torch.empty_like(ts), xc_fused, xs_fused)
    assert F.focus_get_error() == 0
    assert torch.equal(xs_fused, xs_sw) and torch.equal(xc_fused, xc)

    Xd, Wd = dequant(host(xc), host(xs)), dequant(host(wc), host(wsc))
    tsh = host(ts).astype(np.float64)[:, None]
    ref = (Xd @ Wd.T) * tsh * s2
    bound = (np.abs(Xd) @ np.abs(Wd).T) * tsh * s2
    Y = nvfp4_gemm(xc, xs_sw, wc, ws_sw, M, N, K) * ts[:, None] * s2
    check_product(Y, ref, bound, "library export, library swizzle")

    # the oracle's layout, from the oracle's own quantization of the same inputs, pinned by the same consumer
    ro = oracle.fouroversix(host_bits(X))
    codes_o, scales_o, _ = oracle.pack(host_bits(W), host(m), host(q), np.float32(s2))
    xs_o = torch.from_numpy(oracle.scales_swizzle(ro.scales)).cuda()
    ws_o = torch.from_numpy(oracle.scales_swizzle(scales_o)).cuda()
    xc_o = torch.from_numpy(np.ascontiguousarray(ro.codes[:, 0::2] | (ro.codes[:, 1::2] << 4))).cuda()
    wc_o = torch.from_numpy(codes_o).cuda()
    Xo, Wo = dequant(host(xc_o), ro.scales), dequant(codes_o, scales_o)
    tso = ro.row_scales.astype(np.float64)[:, None]
    Yo = nvfp4_gemm(xc_o, xs_o, wc_o, ws_o, M, N, K) * torch.from_numpy(ro.row_scales).cuda()[:, None] * s2
    check_product(Yo, (Xo @ Wo.T) * tso * s2, (np.abs(Xo) @ np.abs(Wo).T) * tso * s2, "oracle export, oracle swizzle")

    # negative control: row-major scales passed as if they were in the 128x4 layout
    lin_x = torch.zeros_like(xs_sw); lin_x[:xs.numel()] = xs.view(-1)
    lin_w = torch.zeros_like(ws_sw); lin_w[:wsc.numel()] = wsc.view(-1)
    Yb = nvfp4_gemm(xc, lin_x, wc, lin_w, M, N, K) * ts[:, None] * s2
    err = np.abs(host(Yb).astype(np.float64) - ref)
    assert np.mean(err > 2.0 ** -7 * bound) > 0.5, "a wrong scale layout went unnoticed"
