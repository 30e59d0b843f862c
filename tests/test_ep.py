"""The expert-parallel layer's exchange logic on CPU: ranks as gloo processes (the way
torchrun starts them, on 127.0.0.1) and as threads of one process (LocalExchange). The
compute calls are plain-torch stand-ins with the library's names and arguments and a
toy per-group transform, so the expert-parallel result must equal the one-rank pipeline
of the same stand-ins bit for bit: what this checks is who sends which row where, the
rebase of global ids, the shared rows that stay home and the return order. The real
kernels run the same path on a GPU in test_gpu_ep.py."""
import os
import socket
import threading

import pytest
import torch
import torch.multiprocessing as mp

from grouped_gemm_swiglu_b200 import ep
from grouped_gemm_swiglu_b200._lib import MoeDims

MOE_ERR_EXPERT_ID = -5


class CpuOps:
    """Stand-ins for the library calls the expert-parallel layer makes (CPU tensors)."""

    @staticmethod
    def alloc_workspace(dims, kind, device="cpu"):
        return torch.zeros(1, dtype=torch.int32)

    @staticmethod
    def moe_read_status(ws):
        return int(ws[0])

    @staticmethod
    def moe_route_topk(logits, d, bias, ids, tw, sw=None, packed=None):
        key = logits[:, :d.E].double()
        order = torch.argsort(-key, dim=1, stable=True)[:, :d.k]  # ties to the lower id
        ids.copy_(order.int())
        tw.copy_(torch.softmax(torch.gather(key, 1, order), 1).float())
        if sw is not None:
            sw.copy_(torch.sigmoid(logits[:, d.E:d.E + d.n_sink]).float())

    @staticmethod
    def moe_permute(ids, x, d, offsets, perm, inv, x_perm, x_scale, ws):
        T, k, E, S = d.T, d.k, d.E, d.n_shared
        rows = []
        for e in range(E):
            for t in range(T):
                for j in range(k):
                    if int(ids[t, j]) == e:
                        inv[t, j] = len(rows)
                        rows.append(t)
        for t in range(T):
            for j in range(k):
                if not 0 <= int(ids[t, j]) < E:
                    ws[0] = MOE_ERR_EXPERT_ID
                    inv[t, j] = 0
        bounds = [0]
        for e in range(E):
            bounds.append(bounds[-1] + sum(1 for t in range(T) for j in range(k) if int(ids[t, j]) == e))
        for s in range(S):
            rows.extend(range(T))
            bounds.append(bounds[-1] + T)
        offsets.copy_(torch.tensor(bounds, dtype=torch.int32))
        perm[:len(rows)] = torch.tensor(rows, dtype=torch.int32)
        x_perm[:len(rows)] = x[torch.tensor(rows, dtype=torch.long)] if rows else x_perm[:0]

    @staticmethod
    def moe_ep_row_ids(offsets, d, row_ids):
        o = offsets.tolist()
        for g in range(d.E + d.n_shared):
            row_ids[o[g]:o[g + 1]] = g

    @staticmethod
    def moe_ep_rebase(ids, n, E, n_shared, off, n_local, out):
        for i in range(n):
            g = int(ids[i])
            out.view(-1)[i] = g - off if off <= g < off + n_local else (n_local + g - E if E <= g < E + n_shared
                                                                         else -1)

    @staticmethod
    def moe_experts(x_perm, xs, offsets, w1, w1s, gs, us, lim, w2, w2s, d, h, hs, y, ws):
        # toy expert g: y = bf16(x * w1[g] + w2[g]), row by row
        o = offsets.tolist()
        for g in range(d.E + d.n_shared):
            y[o[g]:o[g + 1]] = (x_perm[o[g]:o[g + 1]].double() * float(w1[g]) + float(w2[g])).to(torch.bfloat16)

    @staticmethod
    def moe_combine(y, offsets, inv, tw, sw, d, out, ws):
        o = offsets.tolist()
        for t in range(d.T):
            acc = torch.zeros(d.H, dtype=torch.float64)
            for j in range(d.k):
                acc += float(tw[t, j]) * y[int(inv[t, j])].double()
            for s in range(d.n_shared):
                acc += (float(sw[t, s]) if d.n_sink else 1.0) * y[o[d.E + s] + t].double()
            out[t] = acc.to(torch.bfloat16)


def _dims(T, E, k, n_sink, n_shared, H=128):
    d = MoeDims()
    d.T, d.H, d.I, d.E, d.k, d.n_sink, d.n_shared = T, H, 128, E, k, n_sink, n_shared
    d.wdtype, d.score, d.alpha, d.beta, d.limit, d.route_scale = 0, 1, 1.0, 0.0, float("inf"), 1.0
    return d


def _inputs(rank, T, E, n_sink, H, seed=0):
    g = torch.Generator().manual_seed(1000 * seed + rank)
    logits = torch.randn((T, E + n_sink), generator=g)
    if T:
        logits[0, :E] = 0.25  # a row of exact ties
    x = torch.randn((T, H), generator=g).to(torch.bfloat16)
    return logits, x


def _weights(E, S, seed=0):
    g = torch.Generator().manual_seed(77 + seed)
    return torch.rand((E + S,), generator=g) + 0.5, torch.randn((E + S,), generator=g)


def _one_rank(d, logits, x, w1, w2, ops=None):
    """The plain pipeline of the stand-ins with every expert on one rank."""
    ops = ops if ops is not None else CpuOps
    T = x.shape[0]
    dd = MoeDims.from_buffer_copy(d)
    dd.T = T
    ids = torch.empty((T, d.k), dtype=torch.int32)
    tw = torch.empty((T, d.k))
    sw = torch.empty((T, d.n_sink)) if d.n_sink else None
    ops.moe_route_topk(logits, dd, None, ids, tw, sw)
    A = T * (d.k + d.n_shared)
    offsets = torch.empty((d.E + d.n_shared + 1,), dtype=torch.int32)
    perm = torch.empty((A,), dtype=torch.int32)
    inv = torch.empty((T, d.k), dtype=torch.int32)
    xp = torch.empty((A, d.H), dtype=torch.bfloat16)
    ws = torch.zeros(1, dtype=torch.int32)
    ops.moe_permute(ids, x, dd, offsets, perm, inv, xp, None, ws)
    y = torch.empty((A, d.H), dtype=torch.bfloat16)
    ops.moe_experts(xp, None, offsets, w1, None, None, None, None, w2, None, dd, None, None, y, ws)
    out = torch.empty((T, d.H), dtype=torch.bfloat16)
    ops.moe_combine(y, offsets, inv, tw, sw, dd, out, ws)
    return out


CASES = [  # (tokens per rank, E, k, n_sink, n_shared)
    ((5, 7), 8, 2, 2, 2),
    ((6, 0), 8, 3, 0, 1),     # a rank without tokens still serves its experts
    ((9, 4), 8, 2, 0, 0),
]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank, world, port, case, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        Ts, E, k, n_sink, n_shared = case
        d = _dims(0, E, k, n_sink, n_shared)
        w1, w2 = _weights(E, n_shared)
        logits, x = _inputs(rank, Ts[rank], E, n_sink, d.H)
        layer = ep.ExpertParallelMoE(d, rank, world, ep.shard(w1, rank, world, E, n_shared),
                                     ep.shard(w2, rank, world, E, n_shared), exchange=ep.TorchExchange(),
                                     ops=CpuOps)
        out = layer.forward(logits, x)
        ref = _one_rank(d, logits, x, w1, w2)
        q.put((rank, bool(torch.equal(out, ref)), layer.status()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("case", CASES)
def test_two_gloo_ranks_match_the_one_rank_pipeline_bit_for_bit(case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_rank, args=(r, 2, port, case, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [True, True]
    assert [r[2] for r in res] == [0, 0]


def _run_threads(world, Ts, E, k, n_sink, n_shared, ops=CpuOps, layer_kw=None):
    d = _dims(0, E, k, n_sink, n_shared)
    w1, w2 = _weights(E, n_shared)
    hub = ep.LocalExchange(world)
    outs, errs, layers = [None] * world, [], [None] * world

    def run(r):
        try:
            logits, x = _inputs(r, Ts[r], E, n_sink, d.H)
            layers[r] = ep.ExpertParallelMoE(d, r, world, ep.shard(w1, r, world, E, n_shared),
                                             ep.shard(w2, r, world, E, n_shared), exchange=hub.for_rank(r), ops=ops,
                                             **(layer_kw or {}))
            outs[r] = (layers[r].forward(logits, x), _one_rank(d, logits, x, w1, w2))
        except Exception as e:  # noqa: BLE001 (reported below)
            errs.append(e)
            hub._barrier.abort()

    ts = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in ts:
        t.start()
    for t in ts:
        t.join(timeout=120)
    return outs, errs, layers


@pytest.mark.parametrize("world", [1, 2, 4])
def test_thread_ranks_match_the_one_rank_pipeline_bit_for_bit(world):
    Ts = [7, 3, 0, 5][:world]
    outs, errs, layers = _run_threads(world, Ts, 8, 2, 2, 2)
    assert not errs, errs
    for r in range(world):
        got, ref = outs[r]
        assert torch.equal(got, ref), f"rank {r}"
        assert layers[r].status() == 0


def test_buffers_are_kept_and_reused_across_passes_of_varying_size():
    """Several passes per rank with token counts that grow and shrink (including a pass
    with more tokens than max_tokens, and one where the other rank sends more rows than
    any earlier pass): every pass matches the one-rank pipeline, and a pass that fits the
    buffers allocates none."""
    world, E, k, n_sink, n_shared = 2, 8, 2, 2, 2
    d = _dims(0, E, k, n_sink, n_shared)
    w1, w2 = _weights(E, n_shared)
    hub = ep.LocalExchange(world)
    sizes = [[4, 6], [2, 1], [9, 3], [3, 12], [1, 1]]  # per pass: tokens of rank 0, rank 1
    res, errs = {}, []

    def run(r):
        try:
            layer = ep.ExpertParallelMoE(d, r, world, ep.shard(w1, r, world, E, n_shared),
                                         ep.shard(w2, r, world, E, n_shared), exchange=hub.for_rank(r), ops=CpuOps,
                                         max_tokens=8)
            got = []
            for i, Ts in enumerate(sizes):
                logits, x = _inputs(r, Ts[r], E, n_sink, d.H, seed=i)
                before = (layer.buf, layer.own)
                out = layer.forward(logits, x)
                got.append((torch.equal(out, _one_rank(d, logits, x, w1, w2)), before[0] is layer.buf,
                            before[1] is layer.own, layer.buf.T_cap, layer.own.n_cap))
            res[r] = (got, layer.status())
        except Exception as e:  # noqa: BLE001 (reported below)
            errs.append(e)
            hub._barrier.abort()

    ts = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in ts:
        t.start()
    for t in ts:
        t.join(timeout=120)
    assert not errs, errs
    for r in range(world):
        got, st = res[r]
        assert st == 0
        assert all(g[0] for g in got), [g[0] for g in got]
        # the first pass allocates (capacity 8 tokens, every rank's routed rows: 2*8*2 + 8*2);
        # the second reuses; a pass of 9 or 12 own tokens grows the source side
        assert got[0][3] == 8 and got[0][4] == world * 8 * k + 8 * n_shared
        assert got[1][1] and got[1][2]
        assert got[4][1] and got[4][2]


def test_uneven_expert_split_is_rejected():
    d = _dims(0, 6, 2, 0, 0)
    with pytest.raises(ValueError):
        ep.ExpertParallelMoE(d, 0, 4, torch.zeros(2), torch.zeros(2), exchange=object(), ops=CpuOps)


class MisroutingOps(CpuOps):
    """Sends every routed row of rank 0 with the id of an expert rank 1 does not hold."""

    @staticmethod
    def moe_ep_row_ids(offsets, d, row_ids):
        CpuOps.moe_ep_row_ids(offsets, d, row_ids)
        routed = int(offsets[d.E])
        row_ids[:routed] = torch.where(row_ids[:routed] >= d.E // 2, torch.zeros_like(row_ids[:routed]),
                                       row_ids[:routed])


def test_an_id_outside_the_local_range_is_reported():
    outs, errs, layers = _run_threads(2, [6, 6], 8, 2, 0, 0, ops=MisroutingOps)
    assert not errs, errs
    # rows meant for rank 1 arrive with id 0 (rank 0's expert): rank 1's rebase turns them
    # into -1 and its local permutation records the error
    assert layers[1].status() == MOE_ERR_EXPERT_ID


def _dying_rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:  # leaves between steps, before its first exchange
        _put_and_exit(q, (rank, "left"))
    d = _dims(0, 8, 2, 0, 0)
    w1, w2 = _weights(8, 0)
    logits, x = _inputs(rank, 6, 8, 0, d.H)
    layer = ep.ExpertParallelMoE(d, rank, world, ep.shard(w1, rank, world, 8, 0), ep.shard(w2, rank, world, 8, 0),
                                 exchange=ep.TorchExchange(), ops=CpuOps)
    try:
        layer.forward(logits, x)
        msg = "finished"
    except Exception as e:  # noqa: BLE001 (the expected outcome)
        msg = "error: " + type(e).__name__
    _put_and_exit(q, (rank, msg))


def _put_and_exit(q, item):
    """Report, then leave without the process group's orderly shutdown (which would wait
    for the other rank)."""
    q.put(item)
    q.close()
    q.join_thread()
    os._exit(0)


def test_a_rank_that_leaves_ends_the_others_exchange_with_an_error():
    """Failure detection on the host: one rank exits before the exchange; the other's
    all_to_all ends with an error within the process group's short timeout, not a hang."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dying_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = dict(q.get(timeout=10) for _ in range(2))
    assert res[1] == "left"
    assert res[0].startswith("error"), res[0]


def _random_configs(n, seed=5):
    import random
    rnd = random.Random(seed)
    out = []
    while len(out) < n:
        world = rnd.choice([1, 2, 3, 4])
        E = world * rnd.randint(1, 4)
        k = rnd.randint(1, min(E, 4))
        n_sink = rnd.choice([0, 0, 2])
        n_shared = n_sink if n_sink and rnd.random() < 0.5 else (0 if n_sink else rnd.choice([0, 1, 2]))
        Ts = [rnd.choice([0, 1, 3, 8]) for _ in range(world)]
        out.append((world, tuple(Ts), E, k, n_sink, n_shared))
    return out


@pytest.mark.parametrize("cfg", _random_configs(16), ids=lambda c: "w{}-T{}-E{}-k{}-s{}-sh{}".format(
    c[0], "_".join(map(str, c[1])), *c[2:]))
def test_random_layouts_match_the_one_rank_pipeline(cfg):
    world, Ts, E, k, n_sink, n_shared = cfg
    outs, errs, layers = _run_threads(world, list(Ts), E, k, n_sink, n_shared)
    assert not errs, errs
    for r in range(world):
        got, ref = outs[r]
        assert torch.equal(got, ref), f"rank {r}"
        assert layers[r].status() == 0
