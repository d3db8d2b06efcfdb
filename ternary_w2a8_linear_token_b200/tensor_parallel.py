"""Tensor-parallel BitLinear across the ranks of a torch.distributed process group.

Page "BitNet：1-bit LLM推理框架技术实战指南" (the distributed engine: a model split by layer or by
tensor across devices) describes sharded inference without the arithmetic; these are the two
tensor splits of one BitLinear and what each rank computes:

- column split (over the N output rows): rank r owns rows [n0, n1) of the packed weights and
  of a per-row scale; every rank sees the whole x, runs bitnet_linear on its rows, and the
  outputs are all-gathered along N. Nothing crosses ranks before the gather.
- row split (over K): rank r owns x[:, k0:k1] and packed[:, k0/4 : k1/4] (k0, k1 multiples of
  64). The per-token scale needs the amax of the whole row and the accumulator the sum over
  all slices, so a rank takes its slice's amax (bitnet_act_amax), all-reduces it (max),
  quantises its slice with the global amax (bitnet_quant_act_amax), contracts it with its
  weight slice (bitnet_linear_i32), all-reduces the int32 partial accumulators (sum; integer
  addition is exact in any order), and runs the epilogue once (bitnet_dequant). The weight
  scale must be the one of the whole row (absmean over all of K), computed before sharding.

Both splits give bitnet_linear's output bit for bit. The collectives are torch.distributed's
(NCCL on GPUs); every compute step runs in the library's kernels through `ops` (CudaOps, the
default, calls the C ABI binding).
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist


def split_range(n: int, world: int, rank: int, align: int = 1) -> Tuple[int, int]:
    """[start, stop) of rank's share of n items taken in units of `align` (n % align == 0):
    contiguous, in rank order, shares differing by at most one unit."""
    if n % align != 0:
        raise ValueError(f"{n} is not a multiple of {align}")
    units = n // align
    base, extra = divmod(units, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start * align, stop * align


class CudaOps:
    """The per-rank steps, through the C ABI binding (the library's CUDA kernels)."""

    def __init__(self):
        import ternary_w2a8_linear_token_b200 as bn
        self.bn = bn

    def linear(self, x, packed, s_w, per_row, out_dtype):
        return self.bn.bitnet_linear(x, packed, s_w, per_row, out_dtype=out_dtype)

    def act_amax(self, x):
        return self.bn.bitnet_act_amax(x)

    def quant_act_amax(self, x, amax):
        return self.bn.bitnet_quant_act_amax(x, amax)

    def linear_i32(self, q, packed):
        return self.bn.bitnet_linear_i32(q, packed)

    def dequant(self, acc, s_x, s_w, per_row, out_dtype):
        return self.bn.bitnet_dequant(acc, s_x, s_w, per_row, out_dtype=out_dtype)


def _world(group):
    return dist.get_world_size(group), dist.get_rank(group)


class ColumnParallelLinear:
    """A BitLinear whose N output rows are split over the group's ranks."""

    def __init__(self, packed: torch.Tensor, s_w: torch.Tensor, per_row: bool,
                 group: Optional[dist.ProcessGroup] = None, ops=None):
        world, rank = _world(group)
        N = packed.shape[0]
        if N < world:
            raise ValueError("fewer output rows than ranks")
        self.ranges = [split_range(N, world, r) for r in range(world)]
        n0, n1 = self.ranges[rank]
        self.packed = packed[n0:n1].contiguous()
        self.s_w = s_w[n0:n1].contiguous() if per_row else s_w
        self.per_row, self.group, self.N = per_row, group, N
        self.ops = ops or CudaOps()

    def forward(self, x: torch.Tensor, out_dtype=torch.bfloat16) -> torch.Tensor:
        y = self.ops.linear(x, self.packed, self.s_w, self.per_row, out_dtype)
        width = max(b - a for a, b in self.ranges)
        if y.shape[1] < width:  # all_gather wants equal shapes: pad, gather, cut
            y = torch.cat([y, y.new_zeros((y.shape[0], width - y.shape[1]))], dim=1)
        parts = [torch.empty_like(y) for _ in self.ranges]
        dist.all_gather(parts, y.contiguous(), group=self.group)
        return torch.cat([p[:, : b - a] for p, (a, b) in zip(parts, self.ranges)], dim=1)


class RowParallelLinear:
    """A BitLinear whose K range is split over the group's ranks (K = 64 * units)."""

    def __init__(self, packed: torch.Tensor, s_w: torch.Tensor, per_row: bool,
                 group: Optional[dist.ProcessGroup] = None, ops=None):
        world, rank = _world(group)
        K = packed.shape[1] * 4
        if K % 64 != 0 or K < 64 * world:
            raise ValueError("K must be a multiple of 64 with at least 64 per rank")
        self.k0, self.k1 = split_range(K, world, rank, align=64)
        self.packed = packed[:, self.k0 // 4: self.k1 // 4].contiguous()
        self.s_w, self.per_row, self.group, self.K = s_w, per_row, group, K
        self.ops = ops or CudaOps()

    def slice_input(self, x: torch.Tensor) -> torch.Tensor:
        """This rank's columns of a whole (M, K) input."""
        return x[:, self.k0:self.k1].contiguous()

    def forward(self, x_local: torch.Tensor, out_dtype=torch.bfloat16) -> torch.Tensor:
        """x_local: this rank's (M, k1 - k0) slice of the input."""
        amax = self.ops.act_amax(x_local)
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=self.group)
        q, s_x = self.ops.quant_act_amax(x_local, amax)
        acc = self.ops.linear_i32(q, self.packed)
        dist.all_reduce(acc, op=dist.ReduceOp.SUM, group=self.group)
        return self.ops.dequant(acc, s_x, self.s_w, self.per_row, out_dtype)
