"""Seeded synthetic workloads for the Muon step.

This module only *draws* inputs: shapes, hyperparameters and random tensors.
It holds none of the method's arithmetic (no momentum, normalisation,
Newton-Schulz or update), so that the oracle and the CUDA path can both take
their inputs from here without sharing any of the computation.

Workloads (projection-matrix sets named after the models whose layer shapes
they copy; PyTorch ``nn.Linear`` weight layout, i.e. ``(out, in)``):

* ``single_256x512_f32``  - one 256x512 fp32 matrix, N(0,1) gradient,
  zero momentum buffer, N(0,0.02) parameter.
* ``small_layer_bf16``    - one small transformer layer (hidden 1024,
  intermediate 2816, 16x64 heads, 4 KV heads): q/o 1024x1024, k/v 256x1024,
  gate/up 2816x1024, down 1024x2816.  Gradient = rank-64 ``U diag(1/i) V^T``
  plus N(0,1e-3) noise; buffers N(0,0.01).
* ``llama3_2_3b_bf16``    - 28 layers x 7 projections (hidden 3072,
  intermediate 8192, 24x128 heads, 8 KV heads), wd=0.1.
* ``llama_7b_bf16``       - 32 layers x 7 projections (hidden 4096,
  intermediate 11008).
* ``moe_skewed_bf16``     - 64 experts x (gate, up 1408x2048, down
  2048x1408), 48 GateDelta-style 32x4096 projections and 8 tall 16384x2048
  matrices; N(0,1) gradients with 5% of the matrices scaled by 1e-4.

For the two Llama-shaped sets the gradient is N(0,1e-2) noise plus a
decaying-spectrum low-rank term ``U diag(1/i) V^T`` (rank 64 / 128) scaled to
the same Frobenius energy as the noise.  "N(0, s)" always means standard
deviation ``s``.

Every matrix ``idx`` of workload number ``k`` (1-based, in the order above)
is drawn from its own generator seeded with ``1234 + 1000*k + idx``: first the
gradient, then the momentum buffer, then the parameter.  A single matrix can
therefore be regenerated on its own (used for sampled parity checks at full
size).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence, Tuple

import numpy as np
import torch

F32 = "f32"
BF16 = "bf16"

_TORCH_DTYPE = {F32: torch.float32, BF16: torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    number: int                       # 1-based position in the list below
    shapes: Tuple[Tuple[int, int], ...]
    names: Tuple[str, ...]
    dtype: str
    lr: float = 0.02
    momentum: float = 0.95
    nesterov: bool = True
    ns_steps: int = 5
    wd: float = 0.0
    grad_kind: str = "gaussian"       # gaussian | lowrank_noise | noise_lowrank | gaussian_skewed
    grad_std: float = 1.0
    lowrank_rank: int = 0
    buf_kind: str = "zero"            # zero | gaussian
    buf_std: float = 0.0
    param_std: float = 0.02
    skew_fraction: float = 0.0        # fraction of matrices whose gradient is scaled
    skew_scale: float = 1.0

    @property
    def count(self) -> int:
        return len(self.shapes)

    def torch_dtype(self) -> torch.dtype:
        return _TORCH_DTYPE[self.dtype]

    def elements(self) -> int:
        return sum(r * c for r, c in self.shapes)

    def ns_flops(self) -> float:
        """Algorithmic flops of the Gram Newton-Schulz chain for one step.

        Per matrix and iteration with m = min(R, C), n = max(R, C):
        one triangle of X X^T (m^2 n), one triangle of G G (m^3) and the
        full p(G) X product (2 m^2 n).
        """
        tot = 0.0
        for r, c in self.shapes:
            m, n = min(r, c), max(r, c)
            tot += 3.0 * m * m * n + float(m) ** 3
        return tot * self.ns_steps

    def dense_ns_flops(self) -> float:
        """Dense-equivalent flops (no symmetry saving): 4 m^2 n + 2 m^3."""
        tot = 0.0
        for r, c in self.shapes:
            m, n = min(r, c), max(r, c)
            tot += 4.0 * m * m * n + 2.0 * float(m) ** 3
        return tot * self.ns_steps


def _layer_set(layers: int, hidden: int, inter: int, q_out: int, kv_out: int):
    shapes, names = [], []
    for layer in range(layers):
        for nm, shp in (("q_proj", (q_out, hidden)), ("k_proj", (kv_out, hidden)),
                        ("v_proj", (kv_out, hidden)), ("o_proj", (hidden, q_out)),
                        ("gate_proj", (inter, hidden)), ("up_proj", (inter, hidden)),
                        ("down_proj", (hidden, inter))):
            shapes.append(shp)
            names.append(f"layers.{layer}.{nm}")
    return tuple(shapes), tuple(names)


def _moe_set():
    shapes, names = [], []
    for e in range(64):
        for nm, shp in (("gate_proj", (1408, 2048)), ("up_proj", (1408, 2048)),
                        ("down_proj", (2048, 1408))):
            shapes.append(shp)
            names.append(f"experts.{e}.{nm}")
    for i in range(48):
        shapes.append((32, 4096))
        names.append(f"gatedelta.{i}.a_proj")
    for i in range(8):
        shapes.append((16384, 2048))
        names.append(f"tall.{i}.proj")
    return tuple(shapes), tuple(names)


def _build() -> List[Workload]:
    out = []
    out.append(Workload("single_256x512_f32", 1, ((256, 512),), ("proj",), F32,
                        grad_kind="gaussian", grad_std=1.0, buf_kind="zero"))
    s, n = _layer_set(1, 1024, 2816, 16 * 64, 4 * 64)
    out.append(Workload("small_layer_bf16", 2, s, n, BF16, grad_kind="lowrank_noise",
                        grad_std=1e-3, lowrank_rank=64, buf_kind="gaussian", buf_std=0.01))
    s, n = _layer_set(28, 3072, 8192, 24 * 128, 8 * 128)
    out.append(Workload("llama3_2_3b_bf16", 3, s, n, BF16, grad_kind="noise_lowrank",
                        grad_std=1e-2, lowrank_rank=64, buf_kind="gaussian", buf_std=0.01,
                        wd=0.1))
    s, n = _layer_set(32, 4096, 11008, 4096, 4096)
    out.append(Workload("llama_7b_bf16", 4, s, n, BF16, grad_kind="noise_lowrank",
                        grad_std=1e-2, lowrank_rank=128, buf_kind="gaussian", buf_std=0.01))
    s, n = _moe_set()
    out.append(Workload("moe_skewed_bf16", 5, s, n, BF16, grad_kind="gaussian_skewed",
                        grad_std=1.0, buf_kind="zero", skew_fraction=0.05, skew_scale=1e-4))
    return out


WORKLOADS: List[Workload] = _build()
BY_NAME = {w.name: w for w in WORKLOADS}


def get(name_or_number) -> Workload:
    if isinstance(name_or_number, int):
        return WORKLOADS[name_or_number - 1]
    return BY_NAME[name_or_number]


def matrix_seed(w: Workload, idx: int) -> int:
    return 1234 + 1000 * w.number + idx


def skewed_indices(w: Workload) -> List[int]:
    """Indices whose gradient is scaled by ``skew_scale`` (chosen by seed)."""
    if w.skew_fraction <= 0.0:
        return []
    k = int(round(w.skew_fraction * w.count))
    rs = np.random.RandomState(1234 + 1000 * w.number)
    return sorted(int(i) for i in rs.choice(w.count, size=k, replace=False))


def _orthonormal(gen: torch.Generator, rows: int, rank: int, device) -> torch.Tensor:
    g = torch.randn(rows, rank, generator=gen, device=device, dtype=torch.float32)
    q, _ = torch.linalg.qr(g)
    return q


def _lowrank(gen, r: int, c: int, rank: int, device) -> torch.Tensor:
    rank = min(rank, r, c)
    u = _orthonormal(gen, r, rank, device)
    v = _orthonormal(gen, c, rank, device)
    s = 1.0 / torch.arange(1, rank + 1, device=device, dtype=torch.float32)
    return (u * s) @ v.T


def make_matrix(w: Workload, idx: int, device="cpu",
                skewed: Optional[Sequence[int]] = None):
    """(param, grad, buf) for matrix ``idx`` of workload ``w`` on ``device``."""
    r, c = w.shapes[idx]
    dt = w.torch_dtype()
    gen = torch.Generator(device=device)
    gen.manual_seed(matrix_seed(w, idx))
    if w.grad_kind in ("gaussian", "gaussian_skewed"):
        g = torch.randn(r, c, generator=gen, device=device) * w.grad_std
        if w.grad_kind == "gaussian_skewed":
            if skewed is None:
                skewed = skewed_indices(w)
            if idx in skewed:
                g = g * w.skew_scale
    elif w.grad_kind == "lowrank_noise":
        g = _lowrank(gen, r, c, w.lowrank_rank, device)
        g = g + torch.randn(r, c, generator=gen, device=device) * w.grad_std
    elif w.grad_kind == "noise_lowrank":
        noise = torch.randn(r, c, generator=gen, device=device) * w.grad_std
        lr_part = _lowrank(gen, r, c, w.lowrank_rank, device)
        target = w.grad_std * math.sqrt(r * c)
        lr_part = lr_part * (target / float(lr_part.norm()))
        g = noise + lr_part
    else:
        raise ValueError(w.grad_kind)
    if w.buf_kind == "zero":
        b = torch.zeros(r, c, device=device)
    else:
        b = torch.randn(r, c, generator=gen, device=device) * w.buf_std
    p = torch.randn(r, c, generator=gen, device=device) * w.param_std
    return p.to(dt).contiguous(), g.to(dt).contiguous(), b.to(dt).contiguous()


def make_all(w: Workload, device="cpu"):
    """Lists (params, grads, bufs) for the whole workload."""
    sk = skewed_indices(w)
    ps, gs, bs = [], [], []
    for i in range(w.count):
        p, g, b = make_matrix(w, i, device, sk)
        ps.append(p)
        gs.append(g)
        bs.append(b)
    return ps, gs, bs


def gaussian(shape, seed: int, dtype=torch.float32, std: float = 1.0, device="cpu"):
    """Plain seeded N(0, std) tensor (test helper)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return (torch.randn(*shape, generator=gen, device=device) * std).to(dtype)
