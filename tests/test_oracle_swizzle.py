"""The oracle's relayout of E4M3 scale factors into the 128x4-atom layout of
sm_100 block-scaled GEMMs.  The pages do not describe this layout (it is
NVIDIA's published format for NVFP4 GEMM operands); the CPU tests below check
its structure -- a bijection onto the padded buffer, zero padding, the atom
and in-atom strides -- and tests/test_gpu_swizzle.py pins it against a real
consumer, PyTorch's NVFP4 scaled_mm (cuBLASLt's block-scaled GEMM) on a B200."""
import numpy as np
import pytest

import oracle


def positions(rows, cols):
    """Output position of every scale (r, c), found by relaying out unique markers."""
    idx = np.arange(rows * cols, dtype=np.int64).reshape(rows, cols) + 1
    lo = oracle.scales_swizzle((idx & 0xFF).astype(np.uint8)).astype(np.int64)
    mid = oracle.scales_swizzle(((idx >> 8) & 0xFF).astype(np.uint8)).astype(np.int64)
    hi = oracle.scales_swizzle(((idx >> 16) & 0xFF).astype(np.uint8)).astype(np.int64)
    tag = lo | (mid << 8) | (hi << 16)
    pos = np.full(rows * cols, -1, np.int64)
    nz = np.nonzero(tag)[0]
    pos[tag[nz] - 1] = nz
    return pos.reshape(rows, cols), tag


@pytest.mark.parametrize("rows,cols", [(1, 1), (128, 4), (130, 6), (300, 64), (37, 9)])
def test_bijection_and_padding(rows, cols):
    pos, tag = positions(rows, cols)
    R, C = -(-rows // 128) * 128, -(-cols // 4) * 4
    assert tag.size == R * C
    assert np.all(pos >= 0) and len(np.unique(pos)) == rows * cols      # every scale lands once
    assert np.count_nonzero(tag) == rows * cols                          # the rest is padding, 0


def test_atom_structure():
    rows, cols = 384, 12
    pos, _ = positions(rows, cols)
    groups = cols // 4
    for r in range(0, rows, 7):
        for c in range(cols):
            atom, off = divmod(int(pos[r, c]), 512)
            assert atom == (r // 128) * groups + c // 4                 # band-major, column groups inner
            assert off % 4 == c % 4                                      # 4 scales of a row are contiguous
            assert (off // 4) % 4 == (r % 128) // 32                     # 32-row groups 4 bytes apart
            assert off // 16 == r % 32                                   # rows 16 bytes apart within a group
