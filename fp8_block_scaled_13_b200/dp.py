"""Data-parallel weight-gradient exchange for the FP8 linear layers.

The pages train with pure data parallelism plus pipeline stages and no tensor
parallelism: every data-parallel rank runs the linear layers on its own
micro-batches, keeps gradients in FP32, and the ranks then combine the weight
gradients with an all-reduce (paper.rainbus.top, "方法步骤详情" step (2):
MBS = 2, PP = 2, DP = 12, no TP; step (1): the AllReduce bandwidth work;
paperlayer.ai Appendix C: gradients kept in FP32).

Here the FP32 gradient buffers of a group of linear layers live in one flat
allocation (`MainGrads`): the weight-gradient GEMM accumulates straight into
each layer's view (gemm_wgrad(..., accumulate=True)), and the exchange is a
collective over the flat buffer or over one layer's slice of it, either an
all-reduce (every rank gets the summed or averaged gradient) or a
reduce-scatter (each rank gets the sum for its own contiguous shard, for an
optimizer that updates only the parameters it owns).  Per-layer exchanges can
be issued asynchronously right after that layer's weight gradient, so they
overlap the rest of the backward pass.  The collectives are torch.distributed
ones (NCCL over NVLink on B200, gloo on CPU for the tests); this module only
lays out the buffer and orders the calls identically on every rank.

A sharding fact the tests pin: the weight gradient is a sum over 128-token
quantization groups, so when every rank's token count is a multiple of 128 the
ranks' groups are exactly the full batch's groups, and the summed per-rank
gradients equal the full-batch gradient up to the FP32 rounding of the sum.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

# Each layer's view starts on a 64-byte boundary (16 FP32 values): the GEMM's
# TMA output descriptor needs a 16-byte-aligned base.
_ALIGN = 16


@dataclass
class _Slot:
    offset: int
    n: int
    k: int


class MainGrads:
    """FP32 gradient buffers [n_i, k_i] of several linear layers in one flat,
    zero-initialised allocation whose length is a multiple of the group size
    (so a reduce-scatter gives every rank an equal, contiguous shard)."""

    def __init__(self, shapes, device=None, group=None):
        self.group = group
        world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.world = world
        self.slots = []
        off = 0
        for (n, k) in shapes:
            if n <= 0 or k <= 0:
                raise ValueError("gradient shapes must be positive")
            off = (off + _ALIGN - 1) // _ALIGN * _ALIGN
            self.slots.append(_Slot(off, n, k))
            off += n * k
        unit = _ALIGN * world
        total = (off + unit - 1) // unit * unit
        self.flat = torch.zeros(total, dtype=torch.float32, device=device)
        self.views = [self.flat[s.offset:s.offset + s.n * s.k].view(s.n, s.k) for s in self.slots]
        self._pending = []

    def __len__(self):
        return len(self.views)

    def __getitem__(self, i) -> torch.Tensor:
        return self.views[i]

    def zero_(self):
        self.flat.zero_()

    @property
    def shard_numel(self) -> int:
        return self.flat.numel() // self.world

    def shard_range(self, rank: int):
        """[start, end) of `rank`'s reduce-scatter shard in the flat buffer."""
        s = self.shard_numel
        return rank * s, (rank + 1) * s

    def _op(self, average: bool):
        return dist.ReduceOp.AVG if average else dist.ReduceOp.SUM

    def all_reduce_(self, average: bool = True):
        """Sum (or average) the whole buffer over the group, in place."""
        if self.world > 1:
            dist.all_reduce(self.flat, op=self._op(average), group=self.group)
        return self.flat

    def reduce_scatter(self, average: bool = True, out: torch.Tensor | None = None) -> torch.Tensor:
        """This rank's shard of the summed (or averaged) buffer."""
        if out is None:
            out = torch.empty(self.shard_numel, dtype=torch.float32, device=self.flat.device)
        if self.world > 1:
            dist.reduce_scatter_tensor(out, self.flat, op=self._op(average), group=self.group)
        else:
            out.copy_(self.flat)
        return out

    def all_reduce_layer_async(self, i: int, average: bool = True):
        """Start the all-reduce of layer i's gradient (returns immediately);
        wait() completes every started exchange, in issue order."""
        if self.world > 1:
            s = self.slots[i]
            work = dist.all_reduce(self.flat[s.offset:s.offset + s.n * s.k], op=self._op(average),
                                   group=self.group, async_op=True)
            self._pending.append(work)

    def wait(self):
        for w in self._pending:
            w.wait()
        self._pending = []
