"""Multi-tensor table: every linear weight of a model, stepped in one launch.

Builds the focus_tensor_desc array (include/focus.h) from torch tensors, lets
the library check it (focus_table_prepare), keeps the device copy, and calls
the multi-tensor entry points.  Marshalling only: all arithmetic is in the
library's kernels.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

from . import focus as F

_FIELDS = ("W", "dWq", "Wq", "m", "q", "m_exp_avg", "m_exp_avg_sq", "q_exp_avg", "q_exp_avg_sq", "s2",
           "codes", "scales", "dm", "dq")

PURPOSE_FORWARD = 0
PURPOSE_STEP = 1
PURPOSE_BACKWARD = 2
PURPOSE_FOUROVERSIX = 3
PURPOSE_MX = 4                                # the MXFP4 calls (focus_mx_*_multi): in % 32 == 0, no s2
PURPOSE_ACT = 5                               # activations for the per-token calls, scales row-major
PURPOSE_ACT_SWIZZLED = 6                      # the same, scales in the 128x4-atom layout


@dataclass
class Entry:
    """One weight: W [out, in] bf16 plus whatever the calls in use need."""
    W: torch.Tensor
    m: torch.Tensor
    q: torch.Tensor
    s2: torch.Tensor | None                   # one float32 on the device (None for an MXFP4 table)
    dWq: torch.Tensor | None = None
    Wq: torch.Tensor | None = None
    m_exp_avg: torch.Tensor | None = None
    m_exp_avg_sq: torch.Tensor | None = None
    q_exp_avg: torch.Tensor | None = None
    q_exp_avg_sq: torch.Tensor | None = None
    codes: torch.Tensor | None = None
    scales: torch.Tensor | None = None
    dm: torch.Tensor | None = None
    dq: torch.Tensor | None = None
    extra: dict = field(default_factory=dict)


class FocusTable:
    def __init__(self, entries: list[Entry], purpose: int = PURPOSE_STEP):
        self.entries = list(entries)
        n = len(self.entries)
        self.n = n
        descs = (F.focus_tensor_desc * max(n, 1))()
        for i, e in enumerate(self.entries):
            d = descs[i]
            for name in _FIELDS:
                t = getattr(e, name)
                setattr(d, name, None if t is None else F._ptr(t))
            d.out, d.in_ = int(e.W.shape[0]), int(e.W.shape[1])
        self.total_tiles = F.focus_table_prepare((F.focus_tensor_desc * n).from_buffer(descs), purpose) if n else 0
        self.descs = descs
        dev = self.entries[0].W.device if n else torch.device("cuda")
        raw = torch.frombuffer(bytearray(bytes(descs)), dtype=torch.uint8)
        self.dev = raw.to(dev)                  # 256-byte aligned device copy
        self._ws = None
        self._amax = None

    def s2(self, stream=None):
        need = F.focus_s2_multi_workspace_bytes(self.total_tiles)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.dev.device)
        F.focus_s2_multi(self.dev, self.n, self.total_tiles, self._ws, stream)

    def step(self, step: int, hp: F.focus_hparams | None = None, flags: int = 0, stream=None):
        hp = hp or hparams()
        F.focus_step_fused(self.dev, self.n, self.total_tiles, hp, step, flags, stream)

    def step_s2(self, step: int, hp: F.focus_hparams | None = None, flags: int = 0, stream=None):
        """The fused step that also leaves each tensor's s2 for the next step (two launches:
        the step, which reduces the block maxima it computes into the tensor maxima, and
        the one that turns them into s2).  The step reads the current desc.s2."""
        hp = hp or hparams()
        if self._amax is None:
            self._amax = torch.zeros(max(self.n, 4), dtype=torch.int32, device=self.dev.device)
        F.focus_step_fused_amax(self.dev, self.n, self.total_tiles, hp, step, self._amax, flags, stream)
        F.focus_s2_from_amax(self.dev, self.n, self._amax, stream)

    def pack(self, stream=None):
        F.focus_pack_multi(self.dev, self.n, self.total_tiles, stream)

    def fwd(self, stream=None):
        F.focus_fwd_multi(self.dev, self.n, self.total_tiles, stream)

    def bwd(self, accumulate: bool = False, stream=None):
        F.focus_ste_bwd_multi(self.dev, self.n, self.total_tiles, accumulate, stream)

    def fouroversix(self, stream=None):
        F.focus_fouroversix_multi(self.dev, self.n, self.total_tiles, stream)

    def nvfp4_rtn(self, stream=None):
        """Plain NVFP4 round to nearest of every entry (a table as for fouroversix)."""
        F.focus_nvfp4_weight_multi(self.dev, self.n, self.total_tiles, stream)

    # MXFP4 (a table built with PURPOSE_MX)
    def mx_fwd(self, stream=None):
        F.focus_mx_fwd_multi(self.dev, self.n, self.total_tiles, stream)

    def mx_bwd(self, accumulate: bool = False, stream=None):
        F.focus_mx_ste_bwd_multi(self.dev, self.n, self.total_tiles, accumulate, stream)

    def mx_step(self, step: int, hp: F.focus_hparams | None = None, flags: int = 0, stream=None):
        F.focus_mx_step_multi(self.dev, self.n, self.total_tiles, hp or hparams(), step, flags, stream)


def hparams(lr_m=5e-3, lr_q=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0) -> F.focus_hparams:
    """The card's calibration setting: AdamW, lr 5e-3 for m and 1e-3 for q, betas 0.9/0.999, wd 0."""
    return F.focus_hparams(lr_m, lr_q, beta1, beta2, eps, weight_decay)


class HostTable:
    """Tensors held in host memory, stepped through focus_step_host: every call uploads
    the step's inputs, steps each tensor on the device and reads the updated parameters
    and outputs back (blocking).  Entries use host tensors (pinned for overlap): W,
    dWq, m, q, the moments, s2 (one float32) and optionally Wq, codes, scales."""

    def __init__(self, entries: list[Entry], device=None):
        self.entries = list(entries)
        n = len(self.entries)
        self.n = n
        descs = (F.focus_tensor_desc * max(n, 1))()
        for i, e in enumerate(self.entries):
            d = descs[i]
            for name in _FIELDS:
                setattr(d, name, F.host_ptr(getattr(e, name)))
            d.out, d.in_ = int(e.W.shape[0]), int(e.W.shape[1])
        self.descs = descs
        need = F.focus_step_host_workspace_bytes(descs, n) if n else 0
        self.ws = torch.empty(max(need, 256), dtype=torch.uint8, device=device or "cuda")

    def step(self, step: int, hp: F.focus_hparams | None = None, flags: int = 0, stream=None):
        F.focus_step_host(self.descs, self.n, hp or hparams(), step, flags, self.ws, stream)


def act_entry(X: torch.Tensor, token_scales: torch.Tensor, codes: torch.Tensor, scales: torch.Tensor,
              Xq: torch.Tensor | None = None) -> Entry:
    """An activation tensor X [tokens, hidden] bf16 for an ActTable: token_scales [tokens]
    f32, codes [tokens, hidden/2] u8, scales (row-major [tokens, hidden/16] u8, or the
    128x4-atom buffer), Xq bf16 (optional)."""
    return Entry(W=X, m=None, q=None, s2=token_scales, codes=codes, scales=scales, Wq=Xq)


class ActTable(FocusTable):
    """Activation tensors (act_entry) quantized per token in one launch: FourOverSix or
    plain NVFP4, the block scales row-major or (swizzled) in the 128x4-atom layout."""

    def __init__(self, entries: list[Entry], swizzled: bool = False):
        self.swizzled = bool(swizzled)
        super().__init__(entries, PURPOSE_ACT_SWIZZLED if swizzled else PURPOSE_ACT)
        self.total_rows = self.total_tiles
        self.max_hidden = max([int(e.W.shape[1]) for e in self.entries] + [16])

    def fouroversix(self, stream=None):
        F.focus_fouroversix_act_multi(self.dev, self.n, self.total_rows, self.max_hidden, self.swizzled, stream)

    def nvfp4(self, stream=None):
        F.focus_nvfp4_act_multi(self.dev, self.n, self.total_rows, self.max_hidden, self.swizzled, stream)
