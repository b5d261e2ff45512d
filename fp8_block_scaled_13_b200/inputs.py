"""Seeded synthetic inputs for the block-scaled FP8 linear layer.

This module only draws random tensors; it holds none of the method's
arithmetic, and both the CUDA path and the CPU oracle consume what it returns
(the same BF16 bytes).  Every tensor is drawn on the CPU from
``torch.Generator().manual_seed(seed)`` in FP32, in the order X, W, dY, then
rounded to BF16 (round to nearest even).

The shapes follow a ~2B dense transformer's linear layers (hidden 2048,
FFN 6144; the Puro-2B report's Qwen3-1.7B-class model, paper.rainbus.top
summary, 核心方法).  The pages publish no dataset for this path; these
distributions stand in for real activations, weights and gradients.

Workloads (name -> what it is):
  single_fprop      X[256,512] ~N(0,1), 0.1% entries x100; W[384,512] ~N(0,.02)
  attn_proj         M=8192 tokens, hidden 2048: QKV W[3072,2048] and output
                    projection W[2048,2048]; X ~N(0,1), W ~N(0,.02), dY ~N(0,1e-3)
  swiglu_gate_up    M=16384, K=2048, N=12288; 8 fixed channels of X x50
  mlp_down_heavy    M=16384, K=6144, N=2048; X Student-t(3) clipped to +-6e4,
                    dY Laplace(0,1e-3); 1% of (row,128-col) groups and 8
                    128-row bands of X and dY set to zero
  full_block        every linear of one hidden-2048/FFN-6144 block at M tokens
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass
class Linear:
    """One linear layer's tensors: X [M,K], W [N,K], dY [M,N] (BF16, CPU)."""
    name: str
    x: torch.Tensor
    w: torch.Tensor
    dy: torch.Tensor | None = None

    @property
    def m(self) -> int:
        return self.x.shape[0]

    @property
    def n(self) -> int:
        return self.w.shape[0]

    @property
    def k(self) -> int:
        return self.x.shape[1]


@dataclass
class Workload:
    name: str
    seed: int
    layers: list = field(default_factory=list)

    def gemm_flops(self) -> int:
        """2*M*N*K per GEMM: fprop always, dgrad and wgrad where dY exists."""
        total = 0
        for L in self.layers:
            per = 2 * L.m * L.n * L.k
            total += per * (3 if L.dy is not None else 1)
        return total


def _normal(g, shape, std=1.0):
    return torch.randn(*shape, generator=g, dtype=torch.float32) * std


def _bf16(t: torch.Tensor) -> torch.Tensor:
    return t.to(torch.bfloat16)


def _student_t3(g, shape):
    # t = Z / sqrt(V/3) with V ~ chi^2(3) = sum of three squared normals.
    z = torch.randn(*shape, generator=g, dtype=torch.float32)
    v = torch.zeros(shape, dtype=torch.float32)
    for _ in range(3):
        v += torch.randn(*shape, generator=g, dtype=torch.float32) ** 2
    return z / torch.sqrt(v / 3.0)


def _laplace(g, shape, b):
    u = torch.rand(*shape, generator=g, dtype=torch.float32) - 0.5
    u = u.clamp(-0.5 + 1e-7, 0.5 - 1e-7)
    return -b * torch.sign(u) * torch.log1p(-2.0 * u.abs())


def _zero_groups(g, t: torch.Tensor, frac: float = 0.01, bands: int = 8):
    """Zero `frac` of the (row, 128-column) groups and the columns of `bands`
    random 128-row bands (exercises both zero-amax paths)."""
    R, C = t.shape
    G = C // 128
    mask = torch.rand(R, G, generator=g) < frac
    t.view(R, G, 128)[mask] = 0
    nb = (R + 127) // 128
    chosen = torch.randperm(nb, generator=g)[:min(bands, nb)]
    for b in chosen.tolist():
        t[b * 128:(b + 1) * 128, :] = 0
    return t


def single_fprop(seed: int = 0) -> Workload:
    g = torch.Generator().manual_seed(seed)
    x = _normal(g, (256, 512))
    outl = torch.rand(256, 512, generator=g) < 1e-3
    x = torch.where(outl, x * 100.0, x)
    w = _normal(g, (384, 512), 0.02)
    return Workload("single_fprop", seed, [Linear("fprop", _bf16(x), _bf16(w))])


def attn_proj(seed: int = 1, m: int = 8192) -> Workload:
    g = torch.Generator().manual_seed(seed)
    x = _normal(g, (m, 2048))
    w_qkv = _normal(g, (3072, 2048), 0.02)
    w_o = _normal(g, (2048, 2048), 0.02)
    dy_qkv = _normal(g, (m, 3072), 1e-3)
    dy_o = _normal(g, (m, 2048), 1e-3)
    xb = _bf16(x)
    return Workload("attn_proj", seed, [
        Linear("qkv", xb, _bf16(w_qkv), _bf16(dy_qkv)),
        Linear("o_proj", xb, _bf16(w_o), _bf16(dy_o)),
    ])


def swiglu_gate_up(seed: int = 2, m: int = 16384) -> Workload:
    g = torch.Generator().manual_seed(seed)
    x = _normal(g, (m, 2048))
    ch = torch.randperm(2048, generator=g)[:8]
    x[:, ch] *= 50.0
    w = _normal(g, (12288, 2048), 0.02)
    dy = _normal(g, (m, 12288), 1e-3)
    return Workload("swiglu_gate_up", seed, [Linear("gate_up", _bf16(x), _bf16(w), _bf16(dy))])


def mlp_down_heavy(seed: int = 3, m: int = 16384) -> Workload:
    g = torch.Generator().manual_seed(seed)
    x = _student_t3(g, (m, 6144)).clamp(-6e4, 6e4)
    w = _normal(g, (2048, 6144), 0.02)
    dy = _laplace(g, (m, 2048), 1e-3)
    x = _zero_groups(g, x)
    dy = _zero_groups(g, dy)
    return Workload("mlp_down_heavy", seed, [Linear("down", _bf16(x), _bf16(w), _bf16(dy))])


def full_block(seed: int = 4, m: int = 4096) -> Workload:
    """QKV (2048->3072), O (2048->2048), gate+up (2048->12288), down (6144->2048)."""
    g = torch.Generator().manual_seed(seed)
    shapes = [("qkv", 3072, 2048), ("o_proj", 2048, 2048),
              ("gate_up", 12288, 2048), ("down", 2048, 6144)]
    xs = [_normal(g, (m, k)) for _, _, k in shapes]
    ws = [_normal(g, (n, k), 0.02) for _, n, k in shapes]
    dys = [_normal(g, (m, n), 1e-3) for _, n, _ in shapes]
    layers = [Linear(name, _bf16(x), _bf16(w), _bf16(dy))
              for (name, _, _), x, w, dy in zip(shapes, xs, ws, dys)]
    return Workload("full_block_m%d" % m, seed, layers)


WORKLOADS = {
    "single_fprop": single_fprop,
    "attn_proj": attn_proj,
    "swiglu_gate_up": swiglu_gate_up,
    "mlp_down_heavy": mlp_down_heavy,
    "full_block": full_block,
}
