"""Seeded synthetic inputs for the FOCUS quantizer: shapes and value recipes.

This module serves both the CUDA path's tests and benchmark and the CPU
oracle's tests; it holds none of the quantizer's arithmetic (no scale, no
encoder, no gradient).  Every generator draws from a ``torch.Generator``
seeded explicitly, on the device it is given, so a run is reproducible on that
device (CPU and CUDA streams differ, so parity tests generate on one device and
copy the same values to the other side).

Shapes follow the model cards: every linear layer except the LM head.
 * Llama-3.2-1B: 16 layers, hidden 2048, KV width 512, MLP 8192 -- the card
   "FOCUS NVFP4 scales for Llama-3.2-1B-Instruct", "What this is" (112 layers,
   60,817,408 blocks, 121,634,816 sub-blocks).
 * Llama-3.1-8B: 32 layers, hidden 4096, KV width 1024, MLP 14336 -- the card
   "Llama-3.1-8B-Instruct FlipQuant MixFP4 maps", tile table (13,631,488 8x64
   tiles).
 * Llama-3.1-70B: 80 layers, hidden 8192, KV width 1024, MLP 28672 -- the card
   "Llama-3.1-70B-Instruct-NVFP4-W4A4" (group size 16, lm_head ignored).
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

PROJ = ("q_proj", "k_proj", "v_proj", "o_proj", "gate_proj", "up_proj", "down_proj")


@dataclass(frozen=True)
class ModelShapes:
    name: str
    layers: int
    hidden: int
    kv: int
    mlp: int

    def layer_shapes(self):
        h, kv, f = self.hidden, self.kv, self.mlp
        return [("q_proj", (h, h)), ("k_proj", (kv, h)), ("v_proj", (kv, h)), ("o_proj", (h, h)),
                ("gate_proj", (f, h)), ("up_proj", (f, h)), ("down_proj", (h, f))]

    def tensors(self):
        """[(name, (out, in))] for every quantized linear, layer-major."""
        return [(f"model.layers.{l}.mlp.{p}" if p in ("gate_proj", "up_proj", "down_proj")
                 else f"model.layers.{l}.self_attn.{p}", s)
                for l in range(self.layers) for p, s in self.layer_shapes()]

    def n_elements(self) -> int:
        return sum(o * i for _, (o, i) in self.tensors())


LLAMA_1B = ModelShapes("Llama-3.2-1B", 16, 2048, 512, 8192)
LLAMA_8B = ModelShapes("Llama-3.1-8B", 32, 4096, 1024, 14336)
LLAMA_70B = ModelShapes("Llama-3.1-70B", 80, 8192, 1024, 28672)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def normal_bf16(shape, std: float, g: torch.Generator, device) -> torch.Tensor:
    """N(0, std) rounded to bf16 (std is the standard deviation)."""
    return (torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std).to(torch.bfloat16)


def add_outliers(W: torch.Tensor, frac: float, factor: float, g: torch.Generator) -> torch.Tensor:
    """Multiply a uniformly chosen fraction of the elements by `factor`."""
    n = W.numel()
    k = max(1, int(round(n * frac)))
    idx = torch.randint(0, n, (k,), generator=g, device=W.device)
    flat = W.view(-1)
    flat[idx] = (flat[idx].float() * factor).to(torch.bfloat16)
    return W


def uniform(shape, lo: float, hi: float, g, device) -> torch.Tensor:
    return torch.rand(shape, generator=g, device=device, dtype=torch.float32) * (hi - lo) + lo


def normal(shape, mean: float, std: float, g, device) -> torch.Tensor:
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std + mean


@dataclass
class Tensors:
    """One weight with everything a step reads; tensors on one device."""
    W: torch.Tensor            # bf16 [out, in]
    m: torch.Tensor            # f32 [out, in/16]
    q: torch.Tensor            # f32 [out, in/8]
    dWq: torch.Tensor | None   # bf16 [out, in]
    m_v1: torch.Tensor | None = None
    m_v2: torch.Tensor | None = None
    q_v1: torch.Tensor | None = None
    q_v2: torch.Tensor | None = None


def adam_states(t: Tensors, g: torch.Generator | None = None, warm: bool = False) -> Tensors:
    """Zero AdamW moments (step 1), or warm ones as a run leaves them (a later
    step): first moments v1 ~ N(0, sigma), second moments v2 = v1^2 + N(0, sigma)^2,
    random, non-negative and at least v1^2 (an EMA of squares bounds the EMA of
    the values), with sigma = 1e-4 for m and 1e-6 for q."""
    dev = t.m.device
    if not warm:
        t.m_v1 = torch.zeros_like(t.m); t.m_v2 = torch.zeros_like(t.m)
        t.q_v1 = torch.zeros_like(t.q); t.q_v2 = torch.zeros_like(t.q)
    else:
        t.m_v1 = normal(t.m.shape, 0.0, 1e-4, g, dev)
        t.m_v2 = t.m_v1 ** 2 + normal(t.m.shape, 0.0, 1e-4, g, dev) ** 2
        t.q_v1 = normal(t.q.shape, 0.0, 1e-6, g, dev)
        t.q_v2 = t.q_v1 ** 2 + normal(t.q.shape, 0.0, 1e-6, g, dev) ** 2
    return t


# --- the five workloads ------------------------------------------------------------

def single_2048(device, seed: int = 0) -> Tensors:
    """W[2048, 2048] ~ N(0, 0.02), m = 1, q = 6 (forward + pack)."""
    g = _gen(seed, device)
    W = normal_bf16((2048, 2048), 0.02, g, device)
    m = torch.ones((2048, 2048 // 16), device=device)
    q = torch.full((2048, 2048 // 8), 6.0, device=device)
    return Tensors(W, m, q, None)


def llama_1b_tensor(index: int, shape, device, with_grad: bool = True) -> Tensors:
    """A Llama-3.2-1B-shaped weight: N(0, 0.02) plus 0.1% outliers x20;
    m ~ U(0.8, 1.2), q ~ N(6, 2), dW' ~ N(0, 1e-3).  Seed 1 + index."""
    g = _gen(1 + index, device)
    out, inn = shape
    W = add_outliers(normal_bf16(shape, 0.02, g, device), 1e-3, 20.0, g)
    m = uniform((out, inn // 16), 0.8, 1.2, g, device)
    q = normal((out, inn // 8), 6.0, 2.0, g, device)
    dWq = normal_bf16(shape, 1e-3, g, device) if with_grad else None
    return Tensors(W, m, q, dWq)


def llama_8b_tensor(index: int, shape, device, with_grad: bool = True, seed_base: int = 2) -> Tensors:
    """A Llama-3.1-8B-shaped weight: N(0, 0.02), m = 1, q = 6, dW' ~ N(0, 1e-3).
    Seed seed_base + index."""
    g = _gen(seed_base + index, device)
    out, inn = shape
    W = normal_bf16(shape, 0.02, g, device)
    m = torch.ones((out, inn // 16), device=device)
    q = torch.full((out, inn // 8), 6.0, device=device)
    dWq = normal_bf16(shape, 1e-3, g, device) if with_grad else None
    return Tensors(W, m, q, dWq)


def llama_70b_layer(layer: int, device, with_grad: bool = True) -> list[Tensors]:
    """The seven weights of one Llama-3.1-70B layer: N(0, 0.015),
    m ~ U(0.9, 1.1), q ~ N(6, 1), dW' ~ N(0, 1e-3).  One generator seeded
    3 + layer draws the projections in order."""
    g = _gen(3 + layer, device)
    res = []
    for _, (out, inn) in LLAMA_70B.layer_shapes():
        W = normal_bf16((out, inn), 0.015, g, device)
        m = uniform((out, inn // 16), 0.9, 1.1, g, device)
        q = normal((out, inn // 8), 6.0, 1.0, g, device)
        dWq = normal_bf16((out, inn), 1e-3, g, device) if with_grad else None
        res.append(Tensors(W, m, q, dWq))
    return res


# E4M3 values used as planted block scales: powers of two times 1, 1.25, 1.5, 1.75.
_PLANT_SCALES = [2.0 ** e * f for e in range(-4, 8) for f in (1.0, 1.25, 1.5, 1.75)]
_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def stress(out: int, inn: int, device, seed: int = 4, frac_zero: float = 0.01, frac_tie: float = 0.01,
           n_high: int = 2000, n_low: int = 2000) -> tuple[Tensors, dict]:
    """The stress tensor: Student-t (nu = 3) x 0.02 with planted structure.

    * Student-t from normals: z / sqrt((n1^2 + n2^2 + n3^2) / 3).
    * The tensor max is raised to A = 21 * 2^e (the smallest such value >= the
      drawn max), planted at one element, so that s2 = A / 2688 = 2^(e-7) is a
      power of two.
    * frac_zero of the blocks are all zero.
    * frac_tie of the blocks are "tie blocks": m = 1, q = 0 for both
      sub-blocks, element 0 = 6 * S * s2 for a planted E4M3 value S and the
      other 15 elements +-t * S * s2 / 2 with t drawn from the seven E2M1
      midpoints.  Every value is exact in bf16.
    * n_high blocks are scaled so their max is near A and get m in [2, 4]
      (scaled max above 448); n_low blocks are scaled by 2^-14 (below 2^-6).
    * m ~ U(0.01, 4) and q per sub-block uniform from {-8, 0, 6, 12} elsewhere.
    Returns the tensors and the index sets of the planted blocks."""
    assert inn % 16 == 0
    g = _gen(seed, device)
    nb = out * inn // 16
    z = torch.randn((out, inn), generator=g, device=device)
    chi = torch.randn((3, out, inn), generator=g, device=device).pow(2).sum(0) / 3.0
    Wf = z / chi.sqrt() * 0.02
    amax = float(Wf.abs().max())
    e = math.ceil(math.log2(amax / 21.0))
    A = 21.0 * 2.0 ** e
    s2 = 2.0 ** (e - 7)
    Wf = Wf.to(torch.bfloat16).float()
    blocks = Wf.view(nb, 16)

    perm = torch.randperm(nb, generator=g, device=device)
    n_zero = int(nb * frac_zero)
    n_tie = int(nb * frac_tie)
    zero_idx = perm[:n_zero]
    tie_idx = perm[n_zero:n_zero + n_tie]
    high_idx = perm[n_zero + n_tie:n_zero + n_tie + n_high]
    low_idx = perm[n_zero + n_tie + n_high:n_zero + n_tie + n_high + n_low]
    max_idx = int(perm[n_zero + n_tie + n_high + n_low])

    m = uniform((nb,), 0.01, 4.0, g, device)
    qchoice = torch.tensor([-8.0, 0.0, 6.0, 12.0], device=device)
    q = qchoice[torch.randint(0, 4, (nb, 2), generator=g, device=device)]

    blocks[zero_idx] = 0.0
    # high clamp: rescale the block so its max is A * u, u in [0.5, 1], and m in [2, 4]
    hb = blocks[high_idx]
    hmax = hb.abs().amax(1, keepdim=True).clamp_min(1e-30)
    u = uniform((len(high_idx), 1), 0.5, 1.0, g, device)
    blocks[high_idx] = (hb / hmax * A * u).to(torch.bfloat16).float()
    m[high_idx] = uniform((len(high_idx),), 2.0, 4.0, g, device)
    # low clamp: shrink by 2^-14
    blocks[low_idx] = (blocks[low_idx] * 2.0 ** -14).to(torch.bfloat16).float()
    # tie blocks
    sc = torch.tensor(_PLANT_SCALES, device=device)
    S = sc[torch.randint(0, len(_PLANT_SCALES), (n_tie,), generator=g, device=device)]
    mids = torch.tensor(_MIDPOINTS, device=device)
    t = mids[torch.randint(0, 7, (n_tie, 15), generator=g, device=device)]
    sgn = torch.where(torch.rand((n_tie, 15), generator=g, device=device) < 0.5, -1.0, 1.0)
    tb = torch.empty((n_tie, 16), device=device)
    tb[:, 0] = 6.0 * S * s2
    tb[:, 1:] = sgn * t * (S * s2 * 0.5)[:, None]
    blocks[tie_idx] = tb
    m[tie_idx] = 1.0
    q[tie_idx] = 0.0
    # the tensor max
    blocks[max_idx] = 0.0
    blocks[max_idx, 0] = A
    m[max_idx] = 1.0

    W = blocks.view(out, inn).to(torch.bfloat16)
    assert float(W.float().abs().max()) == A
    dWq = normal_bf16((out, inn), 1e-3, g, device)
    info = {"A": A, "s2": s2, "zero": zero_idx, "tie": tie_idx, "high": high_idx, "low": low_idx,
            "max_block": max_idx}
    return Tensors(W, m.view(out, inn // 16), q.view(out, inn // 8).contiguous(), dWq), info


def bits(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (on the host)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view("uint16")


def from_bits(a, device="cpu") -> torch.Tensor:
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def activations(tokens: int, hidden: int, device, seed: int = 5, outlier_channels: float = 0.005,
                outlier_factor: float = 30.0, zero_tokens: int = 1) -> torch.Tensor:
    """Activations X [tokens, hidden] bf16 with the structure of a decoder's
    linear inputs: N(0, 1) per element, a fixed set of outlier channels
    (``outlier_channels`` of the columns, scaled by ``outlier_factor``, as
    hidden states of large language models show) and ``zero_tokens`` all-zero
    rows at the end (padding).  The card's calibration runs micro-batches of
    8 windows of 512 tokens (4096 tokens per forward pass)."""
    g = _gen(seed, device)
    X = torch.randn((tokens, hidden), generator=g, device=device, dtype=torch.float32)
    n_out = max(1, int(round(outlier_channels * hidden)))
    cols = torch.randperm(hidden, generator=g, device=device)[:n_out]
    X[:, cols] *= outlier_factor
    if zero_tokens:
        X[tokens - zero_tokens:] = 0.0
    return X.to(torch.bfloat16)
