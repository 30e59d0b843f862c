"""Expert parallelism: the routed experts partitioned over R ranks, one GPU each.

Rank r holds routed experts [r*E/R, (r+1)*E/R) and every shared expert, and serves its
own tokens. One layer pass on every rank:

  1. route and permute its tokens (moe_route_topk, moe_permute in bf16). Experts are
     partitioned in contiguous blocks, so the routed rows of the permuted activations are
     already grouped by the rank that owns their expert; moe_ep_row_ids tags each row
     with its global group id.
  2. exchange: every rank sends each routed row and its id to the owning rank
     (all_to_all of the per-rank row counts, then of the rows and ids).
  3. the owning rank rebases the ids it received (moe_ep_rebase: global ids are rebased
     by the local expert offset and checked against the local expert count, an id of
     another rank is an error; xorl-wheels "FlashInfer 0.6.18 SM100a+SM103a MoE-LoRA
     AOT", "Changes"), appends its own tokens' shared-expert rows, and runs the
     one-rank path over its local groups: moe_permute (k = 1; the FP8 activation
     quantisation happens here), moe_experts, and moe_combine with unit weights, which
     puts the expert outputs back in arrival order (an exact copy: 1.0 * bf16).
  4. exchange back: the rows return to their source rank in the order they left, so
     the source's own offsets, inverse permutation and routing weights finish the layer
     with moe_combine exactly as on one rank.

The exchange is a caller-supplied object (`TorchExchange` wraps torch.distributed's
all_to_all_single; NCCL between GPUs); the compute steps are this library's kernels.
The per-rank row counts are read on the host to size the exchange.
"""
from __future__ import annotations

import threading
from dataclasses import dataclass

import torch

from . import _lib as _default_ops
from ._lib import (MOE_SCORE_SOFTMAX, MOE_WDTYPE_BF16, MOE_WDTYPE_FP8_E4M3_BLOCK128, MOE_WS_COMBINE,
                   MOE_WS_EXPERTS, MOE_WS_PERMUTE, MoeDims)


class TorchExchange:
    """all_to_all_single over a torch.distributed process group (NCCL on GPUs, gloo on CPU)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_to_all(self, out: torch.Tensor, inp: torch.Tensor, out_splits: list[int], in_splits: list[int]) -> None:
        self.dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)

    def all_reduce(self, t: torch.Tensor) -> None:
        """In-place sum over the ranks."""
        self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM, group=self.group)


class LocalExchange:
    """R ranks as threads of one process on one device: all_to_all (and all_reduce) by
    device copies between the ranks' buffers, after every rank's work so far has finished
    (the ranks' kernels never wait on one another; the threads meet on the host)."""

    def __init__(self, world: int):
        self.world = world
        self._barrier = threading.Barrier(world, timeout=120)  # a failed rank breaks it for all
        self._posted: dict[int, tuple[torch.Tensor, list[int]]] = {}

    def for_rank(self, rank: int) -> "_LocalRankExchange":
        return _LocalRankExchange(self, rank)


class _LocalRankExchange:
    def __init__(self, hub: LocalExchange, rank: int):
        self.hub, self.rank, self.world = hub, rank, hub.world

    def all_to_all(self, out, inp, out_splits, in_splits) -> None:
        hub = self.hub
        if inp.is_cuda:
            torch.cuda.synchronize(inp.device)
        hub._posted[self.rank] = (inp, list(in_splits))
        hub._barrier.wait()
        pos = 0
        for src in range(self.world):
            src_inp, src_splits = hub._posted[src]
            start = sum(src_splits[:self.rank])
            n = src_splits[self.rank]
            assert n == out_splits[src], "row counts disagree between ranks"
            if n:
                out[pos:pos + n].copy_(src_inp[start:start + n])
            pos += n
        if out.is_cuda:
            torch.cuda.synchronize(out.device)
        hub._barrier.wait()  # every rank has read the posted buffers

    def all_reduce(self, t: torch.Tensor) -> None:
        """In-place sum over the ranks, in fp32 and rank order (the same bits on every rank)."""
        hub = self.hub
        if t.is_cuda:
            torch.cuda.synchronize(t.device)
        hub._posted[self.rank] = (t, [])
        hub._barrier.wait()
        acc = torch.zeros(t.shape, dtype=torch.float32, device=t.device)
        for src in range(self.world):
            acc += hub._posted[src][0].float()
        hub._barrier.wait()  # every rank has read every tensor before any is overwritten
        t.copy_(acc.to(t.dtype))
        if t.is_cuda:
            torch.cuda.synchronize(t.device)


def shard(t: torch.Tensor | None, rank: int, world: int, E: int, n_shared: int):
    """This rank's slice of a per-group tensor [E + n_shared, ...]: its routed experts, then
    every shared expert (replicated on all ranks)."""
    if t is None:
        return None
    n_local = E // world
    return torch.cat([t[rank * n_local:(rank + 1) * n_local], t[E:E + n_shared]]).contiguous()


@dataclass
class _Sent:
    """What a rank keeps from its dispatch to finish the layer for its own tokens."""
    T: int
    dims: MoeDims
    tw: torch.Tensor
    sw: torch.Tensor | None
    offsets: torch.Tensor
    inv: torch.Tensor
    x_perm: torch.Tensor
    row_ids: torch.Tensor
    a_routed: int
    send_splits: list[int]


class ExpertParallelMoE:
    """One rank of the expert-parallel layer. Weights are this rank's groups only:
    w1 [E/R + n_shared, 2I, H], w2 [E/R + n_shared, H, I] and the matching scales,
    gate/up scales and clamps (see `shard`). `dims` describes the whole layer (global E);
    dims.T is ignored (each call takes its own token count)."""

    def __init__(self, dims: MoeDims, rank: int, world: int, w1, w2, w1_scale=None, w2_scale=None,
                 gate_scale=None, up_scale=None, limits=None, router_bias=None, exchange=None, ops=None):
        if world < 1 or not 0 <= rank < world or dims.E % world:
            raise ValueError(f"E = {dims.E} routed experts do not split evenly over {world} ranks")
        self.dims = MoeDims.from_buffer_copy(dims)
        self.rank, self.world = rank, world
        self.n_local = dims.E // world
        self.local_offset = rank * self.n_local
        self.w1, self.w2, self.w1_scale, self.w2_scale = w1, w2, w1_scale, w2_scale
        self.gate_scale, self.up_scale, self.limits, self.router_bias = gate_scale, up_scale, limits, router_bias
        self.exchange = exchange if exchange is not None else TorchExchange()
        self.ops = ops if ops is not None else _default_ops
        self.status_words: list[torch.Tensor] = []

    # ---------------------------------------------------------------- phase 1 (local)
    def _dispatch(self, logits: torch.Tensor, x: torch.Tensor) -> _Sent:
        ops, dev = self.ops, x.device
        T = x.shape[0]
        d = MoeDims.from_buffer_copy(self.dims)
        d.T = T
        ids = torch.empty((T, d.k), dtype=torch.int32, device=dev)
        tw = torch.empty((T, d.k), dtype=torch.float32, device=dev)
        sw = torch.empty((T, d.n_sink), dtype=torch.float32, device=dev) if d.n_sink else None
        ops.moe_route_topk(logits, d, self.router_bias, ids, tw, sw)
        # the rows travel in bf16; an FP8 layer quantises them on the owning rank
        sd = MoeDims.from_buffer_copy(d)
        sd.wdtype = MOE_WDTYPE_BF16
        A, G = d.A, d.G
        offsets = torch.empty((G + 1,), dtype=torch.int32, device=dev)
        perm = torch.empty((A,), dtype=torch.int32, device=dev)
        inv = torch.empty((T, d.k), dtype=torch.int32, device=dev)
        x_perm = torch.empty((A, d.H), dtype=torch.bfloat16, device=dev)
        ws_p = ops.alloc_workspace(sd, MOE_WS_PERMUTE, device=dev)
        ops.moe_permute(ids, x, sd, offsets, perm, inv, x_perm, None, ws_p)
        row_ids = torch.empty((A,), dtype=torch.int32, device=dev)
        ops.moe_ep_row_ids(offsets, sd, row_ids)
        self.status_words.append(ws_p)
        offs = offsets.cpu().tolist()  # host copy of the group bounds sizes the exchange
        nl = self.n_local
        send = [offs[(r + 1) * nl] - offs[r * nl] for r in range(self.world)]
        return _Sent(T, d, tw, sw, offsets, inv, x_perm, row_ids, offs[d.E], send)

    # ---------------------------------------------------------------- phase 3 (local)
    def _local_experts(self, rows: torch.Tensor, row_ids: torch.Tensor) -> torch.Tensor:
        """The one-rank path over this rank's groups, for rows in arrival order; returns
        their expert outputs (bf16, unweighted) in the same order."""
        ops, dev, d = self.ops, rows.device, self.dims
        n = rows.shape[0]
        G = self.n_local + d.n_shared
        ld = MoeDims.from_buffer_copy(d)
        ld.T, ld.k, ld.E, ld.n_sink, ld.n_shared = n, 1, G, 0, 0
        ld.score, ld.route_scale = MOE_SCORE_SOFTMAX, 1.0
        y_back = torch.empty((n, d.H), dtype=torch.bfloat16, device=dev)
        if n == 0:
            return y_back
        fp8 = d.wdtype == MOE_WDTYPE_FP8_E4M3_BLOCK128
        local_ids = torch.empty((n, 1), dtype=torch.int32, device=dev)
        ops.moe_ep_rebase(row_ids, n, d.E, d.n_shared, self.local_offset, self.n_local, local_ids)
        offsets = torch.empty((G + 1,), dtype=torch.int32, device=dev)
        perm = torch.empty((n,), dtype=torch.int32, device=dev)
        inv = torch.empty((n, 1), dtype=torch.int32, device=dev)
        x_loc = torch.empty((n, d.H), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
        xs = torch.empty((d.H // 128, n), dtype=torch.float32, device=dev) if fp8 else None
        h = torch.empty((n, d.I), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
        hs = torch.empty((d.I // 128, n), dtype=torch.float32, device=dev) if fp8 else None
        y = torch.empty((n, d.H), dtype=torch.bfloat16, device=dev)
        ws_p = ops.alloc_workspace(ld, MOE_WS_PERMUTE, device=dev)
        ws_e = ops.alloc_workspace(ld, MOE_WS_EXPERTS, device=dev)
        ws_c = ops.alloc_workspace(ld, MOE_WS_COMBINE, device=dev)
        ops.moe_permute(local_ids, rows, ld, offsets, perm, inv, x_loc, xs, ws_p)
        ops.moe_experts(x_loc, xs, offsets, self.w1, self.w1_scale, self.gate_scale, self.up_scale, self.limits,
                        self.w2, self.w2_scale, ld, h, hs, y, ws_e)
        ones = torch.ones((n, 1), dtype=torch.float32, device=dev)
        ops.moe_combine(y, offsets, inv, ones, None, ld, y_back, ws_c)
        self.status_words += [ws_p, ws_e, ws_c]
        return y_back

    # ---------------------------------------------------------------- the whole pass
    def forward(self, logits: torch.Tensor, x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        """logits [T, E + n_sink] fp32 and x [T, H] bf16 of this rank's tokens -> out [T, H]."""
        ops, ex, d = self.ops, self.exchange, self.dims
        dev = x.device
        self.status_words = []
        s = self._dispatch(logits, x)
        R = self.world
        # per-rank row counts
        cnt_out = torch.empty((R,), dtype=torch.int64, device=dev)
        ex.all_to_all(cnt_out, torch.tensor(s.send_splits, dtype=torch.int64, device=dev), [1] * R, [1] * R)
        recv_splits = [int(v) for v in cnt_out.cpu().tolist()]
        n_recv = sum(recv_splits)
        n_sh = s.x_perm.shape[0] - s.a_routed  # this rank's own shared-expert rows
        rows = torch.empty((n_recv + n_sh, d.H), dtype=torch.bfloat16, device=dev)
        row_ids = torch.empty((n_recv + n_sh,), dtype=torch.int32, device=dev)
        ex.all_to_all(rows[:n_recv], s.x_perm[:s.a_routed], recv_splits, s.send_splits)
        ex.all_to_all(row_ids[:n_recv], s.row_ids[:s.a_routed], recv_splits, s.send_splits)
        rows[n_recv:].copy_(s.x_perm[s.a_routed:])
        row_ids[n_recv:].copy_(s.row_ids[s.a_routed:])
        y_back = self._local_experts(rows, row_ids)
        # the routed rows go home in the order they came; the shared rows never left
        y = torch.empty((s.x_perm.shape[0], d.H), dtype=torch.bfloat16, device=dev)
        ex.all_to_all(y[:s.a_routed], y_back[:n_recv], s.send_splits, recv_splits)
        y[s.a_routed:].copy_(y_back[n_recv:])
        if out is None:
            out = torch.empty((s.T, d.H), dtype=torch.bfloat16, device=dev)
        ws_c = ops.alloc_workspace(s.dims, MOE_WS_COMBINE, device=dev)
        ops.moe_combine(y, s.offsets, s.inv, s.tw, s.sw, s.dims, out, ws_c)
        self.status_words.append(ws_c)
        return out

    def status(self) -> int:
        """The first nonzero device status of the last forward's calls (0 = all fine)."""
        for ws in self.status_words:
            st = self.ops.moe_read_status(ws)
            if st:
                return st
        return 0
