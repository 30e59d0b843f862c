"""Tensor parallelism over the intermediate size: every rank holds the same I/R slice of
every expert (the matching rows of the gate and up halves of W1, the matching columns of
W2) and runs the whole layer on all tokens with I/R; the layer's output is the sum of the
ranks' outputs, one all-reduce after GEMM2.

Why the sum is the layer: SwiGLU acts on each intermediate index on its own (gate and up
of index i only), GEMM2 sums over the intermediate index, and the routing-weighted
combine is linear, so splitting I splits the output into a sum of per-slice outputs.
Slices are whole multiples of 128 intermediate indices, so every weight block scale
(FP8 128x128), group scale (INT4, 32 along K) and block scale (NVFP4, 16 along K) and
every 1x128 block of h stays inside one rank: each rank computes exactly the slice of the
one-rank layer's arithmetic, up to the rounding of its partial output to bf16 and of the
all-reduce.

The routing (router, permutation) is replicated on every rank; the all-reduce is the
caller-supplied exchange (`TorchExchange.all_reduce`: torch.distributed, NCCL between
GPUs; `LocalExchange`: ranks as threads of one process).
"""
from __future__ import annotations

import torch

from . import _lib as _default_ops
from ._lib import MOE_WS_FORWARD, MoeDims


def shard_w1(t: torch.Tensor | None, rank: int, world: int) -> torch.Tensor | None:
    """This rank's slice of a W1-shaped tensor [G, 2*R*n, ...] (gate rows, then up rows,
    or their block-scale rows): rows [rank*n, (rank+1)*n) of each half."""
    if t is None:
        return None
    half = t.shape[1] // 2
    n = half // world
    if half % world or 2 * half != t.shape[1]:
        raise ValueError(f"W1 dimension {t.shape[1]} does not split over {world} ranks")
    return torch.cat([t[:, rank * n:(rank + 1) * n], t[:, half + rank * n:half + (rank + 1) * n]], dim=1).contiguous()


def shard_w2(t: torch.Tensor | None, rank: int, world: int) -> torch.Tensor | None:
    """This rank's slice of a W2-shaped tensor [G, H(/128), R*n] along its last (intermediate,
    packed-byte or scale) dimension."""
    if t is None:
        return None
    n = t.shape[-1] // world
    if t.shape[-1] % world:
        raise ValueError(f"W2 dimension {t.shape[-1]} does not split over {world} ranks")
    return t[..., rank * n:(rank + 1) * n].contiguous()


class TensorParallelMoE:
    """One rank of the tensor-parallel layer. `dims` describes the whole layer; weights are
    this rank's slices (`shard_w1` for w1 and w1_scale, `shard_w2` for w2 and w2_scale);
    gate/up scales and clamps are per expert and stay whole."""

    def __init__(self, dims: MoeDims, rank: int, world: int, w1, w2, w1_scale=None, w2_scale=None,
                 gate_scale=None, up_scale=None, limits=None, router_bias=None, exchange=None, ops=None):
        if world < 1 or not 0 <= rank < world or dims.I % (128 * world):
            raise ValueError(f"I = {dims.I} does not split into multiples of 128 over {world} ranks")
        self.dims = MoeDims.from_buffer_copy(dims)
        self.local = MoeDims.from_buffer_copy(dims)
        self.local.I = dims.I // world
        self.rank, self.world = rank, world
        self.w1, self.w2, self.w1_scale, self.w2_scale = w1, w2, w1_scale, w2_scale
        self.gate_scale, self.up_scale, self.limits, self.router_bias = gate_scale, up_scale, limits, router_bias
        if exchange is None:
            from .ep import TorchExchange
            exchange = TorchExchange()
        self.exchange = exchange
        self.ops = ops if ops is not None else _default_ops
        self.ws = None

    def forward(self, logits: torch.Tensor, x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        """logits [T, E + n_sink] fp32 and x [T, H] bf16 (the same on every rank) -> out [T, H]."""
        ops, d = self.ops, MoeDims.from_buffer_copy(self.local)
        d.T = x.shape[0]
        if self.ws is None or ops.moe_workspace_size(d, MOE_WS_FORWARD) > self.ws.numel():
            self.ws = ops.alloc_workspace(d, MOE_WS_FORWARD, device=x.device)
        if out is None:
            out = torch.empty((d.T, d.H), dtype=torch.bfloat16, device=x.device)
        ops.moe_forward(logits, self.router_bias, x, self.w1, self.w1_scale, self.gate_scale, self.up_scale,
                        self.limits, self.w2, self.w2_scale, d, out, ws=self.ws)
        self.exchange.all_reduce(out)
        return out

    def status(self) -> int:
        return self.ops.moe_read_status(self.ws) if self.ws is not None else 0
