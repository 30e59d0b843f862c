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
Every buffer and workspace is allocated once, for a token capacity (`max_tokens`, grown
if a call brings more), and reused by every pass. The per-rank row counts are computed
on the device from the offsets, exchanged on the device, and read on the host once per
pass (send and receive counts together) to size the exchange.
"""
from __future__ import annotations

import threading

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
        """In-place sum over the ranks, accumulated in fp32 (a bf16 tensor is widened, summed
        and rounded once, as LocalExchange does; NCCL gives every rank the same bits, and
        the fp32 sum equals the rank-order sum up to fp32 reassociation)."""
        if t.dtype == torch.float32:
            self.dist.all_reduce(t, op=self.dist.ReduceOp.SUM, group=self.group)
            return
        acc = t.float()
        self.dist.all_reduce(acc, op=self.dist.ReduceOp.SUM, group=self.group)
        t.copy_(acc)


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


class _Buffers:
    """The source side of a pass (this rank's tokens), sized for a token capacity."""

    def __init__(self, layer: "ExpertParallelMoE", T_cap: int, dev):
        ops, d, R = layer.ops, layer.dims, layer.world
        self.T_cap = T_cap
        k, S, E, H, I = d.k, d.n_shared, d.E, d.H, d.I
        A = T_cap * (k + S)
        fp8 = d.wdtype == MOE_WDTYPE_FP8_E4M3_BLOCK128
        cap = MoeDims.from_buffer_copy(d)
        cap.T = T_cap
        sd = MoeDims.from_buffer_copy(cap)  # the rows travel in bf16
        sd.wdtype = MOE_WDTYPE_BF16
        # source side: routing and the permutation of this rank's tokens
        self.ids = torch.empty((T_cap, k), dtype=torch.int32, device=dev)
        self.tw = torch.empty((T_cap, k), dtype=torch.float32, device=dev)
        self.sw = torch.empty((T_cap, d.n_sink), dtype=torch.float32, device=dev) if d.n_sink else None
        self.offsets = torch.empty((d.G + 1,), dtype=torch.int32, device=dev)
        self.perm = torch.empty((A,), dtype=torch.int32, device=dev)
        self.inv = torch.empty((T_cap, k), dtype=torch.int32, device=dev)
        self.x_perm = torch.empty((A, H), dtype=torch.bfloat16, device=dev)
        self.row_ids = torch.empty((A,), dtype=torch.int32, device=dev)
        self.ws_p = ops.alloc_workspace(sd, MOE_WS_PERMUTE, device=dev)
        self.ws_c = ops.alloc_workspace(cap, MOE_WS_COMBINE, device=dev)
        self.y_home = torch.empty((A, H), dtype=torch.bfloat16, device=dev)
        # counts: [send R | recv R | routed rows 1], device and host
        self.counts = torch.empty((2 * R + 1,), dtype=torch.int64, device=dev)
        self.bounds = torch.arange(0, E + 1, layer.n_local, dtype=torch.long, device=dev)  # group bounds per rank
        self.status_words = [self.ws_p, self.ws_c]


class _OwnerBuffers:
    """The owner side of a pass: the rows this rank's experts serve (every rank's routed
    rows for them, and its own tokens' shared-expert rows), sized for n_cap rows."""

    def __init__(self, layer: "ExpertParallelMoE", n_cap: int, dev):
        ops, d = layer.ops, layer.dims
        S, H, I = d.n_shared, d.H, d.I
        fp8 = d.wdtype == MOE_WDTYPE_FP8_E4M3_BLOCK128
        self.n_cap = n_cap
        G = layer.n_local + S
        ld = MoeDims.from_buffer_copy(d)
        ld.T, ld.k, ld.E, ld.n_sink, ld.n_shared = n_cap, 1, G, 0, 0
        ld.score, ld.route_scale = MOE_SCORE_SOFTMAX, 1.0
        self.rows = torch.empty((n_cap, H), dtype=torch.bfloat16, device=dev)
        self.recv_ids = torch.empty((n_cap,), dtype=torch.int32, device=dev)
        self.local_ids = torch.empty((n_cap, 1), dtype=torch.int32, device=dev)
        self.l_offsets = torch.empty((G + 1,), dtype=torch.int32, device=dev)
        self.l_perm = torch.empty((n_cap,), dtype=torch.int32, device=dev)
        self.l_inv = torch.empty((n_cap, 1), dtype=torch.int32, device=dev)
        self.x_loc = torch.empty((n_cap, H), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
        self.xs = torch.empty((H // 128, n_cap), dtype=torch.float32, device=dev) if fp8 else None
        self.h = torch.empty((n_cap, I), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
        self.hs = torch.empty((I // 128, n_cap), dtype=torch.float32, device=dev) if fp8 else None
        self.y = torch.empty((n_cap, H), dtype=torch.bfloat16, device=dev)
        self.y_back = torch.empty((n_cap, H), dtype=torch.bfloat16, device=dev)
        self.ones = torch.ones((n_cap, 1), dtype=torch.float32, device=dev)
        self.ws_lp = ops.alloc_workspace(ld, MOE_WS_PERMUTE, device=dev)
        self.ws_le = ops.alloc_workspace(ld, MOE_WS_EXPERTS, device=dev)
        self.ws_lc = ops.alloc_workspace(ld, MOE_WS_COMBINE, device=dev)
        self.status_words = [self.ws_lp, self.ws_le, self.ws_lc]


class ExpertParallelMoE:
    """One rank of the expert-parallel layer. Weights are this rank's groups only:
    w1 [E/R + n_shared, 2I, H], w2 [E/R + n_shared, H, I] and the matching scales,
    gate/up scales and clamps (see `shard`). `dims` describes the whole layer (global E);
    dims.T is ignored (each call takes its own token count). Buffers are allocated for
    `max_tokens` tokens per rank on the first call (more if a call brings more) and
    reused; the receive side holds every other rank's routed rows in the worst case."""

    def __init__(self, dims: MoeDims, rank: int, world: int, w1, w2, w1_scale=None, w2_scale=None,
                 gate_scale=None, up_scale=None, limits=None, router_bias=None, exchange=None, ops=None,
                 max_tokens: int = 0):
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
        self.max_tokens = max_tokens
        self.buf: _Buffers | None = None
        self.own: _OwnerBuffers | None = None
        self.status_words: list[torch.Tensor] = []

    def _buffers(self, T: int, dev) -> _Buffers:
        if self.buf is None or T > self.buf.T_cap:
            self.buf = _Buffers(self, max(T, self.max_tokens, 1), dev)
        return self.buf

    def _owner(self, n: int, dev) -> _OwnerBuffers:
        """Owner-side buffers for n rows: sized for every rank bringing max_tokens tokens of
        routed rows, and grown (to the rows that arrived) when a pass brings more."""
        d = self.dims
        if self.own is None or n > self.own.n_cap:
            T = max(self.max_tokens, 1)
            self.own = _OwnerBuffers(self, max(n, self.world * T * d.k + T * d.n_shared), dev)
        return self.own

    # ---------------------------------------------------------------- the whole pass
    def forward(self, logits: torch.Tensor, x: torch.Tensor, out: torch.Tensor | None = None) -> torch.Tensor:
        """logits [T, E + n_sink] fp32 and x [T, H] bf16 of this rank's tokens -> out [T, H]."""
        ops, ex, R = self.ops, self.exchange, self.world
        dev = x.device
        T = x.shape[0]
        b = self._buffers(T, dev)
        d = MoeDims.from_buffer_copy(self.dims)
        d.T = T
        k, S, H = d.k, d.n_shared, d.H
        A = d.A
        # 1. route and permute this rank's tokens (bf16 rows), tag rows with global group ids
        ids, tw, inv = b.ids[:T], b.tw[:T], b.inv[:T]
        sw = b.sw[:T] if b.sw is not None else None
        ops.moe_route_topk(logits, d, self.router_bias, ids, tw, sw)
        sd = MoeDims.from_buffer_copy(d)
        sd.wdtype = MOE_WDTYPE_BF16
        x_perm, row_ids = b.x_perm[:A], b.row_ids[:A]
        ops.moe_permute(ids, x, sd, b.offsets, b.perm[:A], inv, x_perm, None, b.ws_p)
        ops.moe_ep_row_ids(b.offsets, sd, row_ids)
        # 2. row counts per destination rank on the device, exchanged there, read once
        off64 = b.offsets.to(torch.int64)
        b.counts[:R].copy_(off64[b.bounds[1:]] - off64[b.bounds[:-1]])
        b.counts[2 * R].copy_(off64[d.E])
        ex.all_to_all(b.counts[R:2 * R], b.counts[:R], [1] * R, [1] * R)
        host = b.counts.cpu().tolist()  # the pass's one host read of counts
        send, recv, a_routed = host[:R], host[R:2 * R], host[2 * R]
        n_recv = sum(recv)
        n = n_recv + (A - a_routed)  # received rows + this rank's own shared-expert rows
        o = self._owner(n, dev)
        self.status_words = b.status_words + o.status_words
        rows, recv_ids = o.rows[:n], o.recv_ids[:n]
        ex.all_to_all(rows[:n_recv], x_perm[:a_routed], recv, send)
        ex.all_to_all(recv_ids[:n_recv], row_ids[:a_routed], recv, send)
        rows[n_recv:].copy_(x_perm[a_routed:])
        recv_ids[n_recv:].copy_(row_ids[a_routed:])
        # 3. this rank's experts over the rows in arrival order
        y_back = o.y_back[:n]
        if n:
            G = self.n_local + S
            ld = MoeDims.from_buffer_copy(self.dims)
            ld.T, ld.k, ld.E, ld.n_sink, ld.n_shared = n, 1, G, 0, 0
            ld.score, ld.route_scale = MOE_SCORE_SOFTMAX, 1.0
            local_ids = o.local_ids[:n]
            ops.moe_ep_rebase(recv_ids, n, d.E, S, self.local_offset, self.n_local, local_ids)
            xs = hs = None
            if o.xs is not None:  # block-major scales of n rows: contiguous [K/128][n] views
                xs = o.xs.view(-1)[:(H // 128) * n].view(H // 128, n)
                hs = o.hs.view(-1)[:(d.I // 128) * n].view(d.I // 128, n)
            ops.moe_permute(local_ids, rows, ld, o.l_offsets, o.l_perm[:n], o.l_inv[:n], o.x_loc[:n], xs, o.ws_lp)
            ops.moe_experts(o.x_loc[:n], xs, o.l_offsets, self.w1, self.w1_scale, self.gate_scale, self.up_scale,
                            self.limits, self.w2, self.w2_scale, ld, o.h[:n], hs, o.y[:n], o.ws_le)
            # back to arrival order: a unit-weight combine (an exact copy of each row)
            ops.moe_combine(o.y[:n], o.l_offsets, o.l_inv[:n], o.ones[:n], None, ld, y_back, o.ws_lc)
        # 4. the routed rows go home in the order they came; the shared rows never left
        y = b.y_home[:A]
        ex.all_to_all(y[:a_routed], y_back[:n_recv], send, recv)
        y[a_routed:].copy_(y_back[n_recv:])
        if out is None:
            out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
        ops.moe_combine(y, b.offsets, inv, tw, sw, d, out, b.ws_c)
        return out

    def status(self) -> int:
        """The first nonzero device status recorded by this layer's calls since its buffers
        were allocated (0 = all fine)."""
        for ws in self.status_words:
            st = self.ops.moe_read_status(ws)
            if st:
                return st
        return 0
