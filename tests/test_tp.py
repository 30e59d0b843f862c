"""Tensor parallelism over the intermediate size, on CPU: the weight slicing helpers, the
identity the split rests on (the oracle's layer equals the sum of its layers over the
ranks' slices of I, in bf16, FP8, INT4 and NVFP4, to fp64 rounding), and the all-reduce
of the exchange objects on two gloo processes and on thread-ranks."""
import os
import socket
import threading

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from grouped_gemm_swiglu_b200 import ep, tp
from grouped_gemm_swiglu_b200 import workloads as W
from helpers import oracle_layer


def test_shard_w1_takes_the_same_rows_of_gate_and_up():
    G, I, K = 3, 512, 8
    w1 = torch.arange(G * 2 * I * K, dtype=torch.int64).view(G, 2 * I, K)
    for world in (1, 2, 4):
        n = I // world
        parts = [tp.shard_w1(w1, r, world) for r in range(world)]
        for r, p in enumerate(parts):
            assert p.shape == (G, 2 * n, K)
            assert torch.equal(p[:, :n], w1[:, r * n:(r + 1) * n])
            assert torch.equal(p[:, n:], w1[:, I + r * n:I + (r + 1) * n])
        assert torch.equal(torch.cat([p[:, :n] for p in parts], 1), w1[:, :I])
        assert torch.equal(torch.cat([p[:, n:] for p in parts], 1), w1[:, I:])
    with pytest.raises(ValueError):
        tp.shard_w1(torch.zeros(2, 6, 4), 0, 4)


def test_shard_w2_takes_a_slice_of_the_last_dimension():
    w2 = torch.arange(2 * 16 * 64, dtype=torch.int64).view(2, 16, 64)
    parts = [tp.shard_w2(w2, r, 4) for r in range(4)]
    assert torch.equal(torch.cat(parts, -1), w2)
    assert tp.shard_w2(None, 0, 2) is None and tp.shard_w1(None, 0, 2) is None
    with pytest.raises(ValueError):
        tp.shard_w2(torch.zeros(2, 4, 6), 0, 4)


CASES = [
    (W.Workload("tp_bf16", T=9, H=256, I=512, E=8, k=2, n_sink=2, n_shared=2, score=W.SCORE_SIGMOID), 4),
    (W.Workload("tp_oai", T=9, H=256, I=256, E=8, k=2, score=W.SCORE_SOFTMAX, alpha=1.702, beta=1.0, limit=7.0,
                gate_up_mult=4.0, expert_scales=(0.52, 1.22)), 2),
    (W.Workload("tp_fp8", T=9, H=256, I=256, E=4, k=2, n_shared=1, wdtype=W.WDTYPE_FP8, score=W.SCORE_SIGMOID,
                limit=10.0), 2),
    (W.Workload("tp_int4", T=9, H=256, I=512, E=4, k=2, wdtype=W.WDTYPE_INT4, score=W.SCORE_SIGMOID), 4),
    (W.Workload("tp_nvfp4", T=9, H=256, I=256, E=4, k=2, n_shared=1, wdtype=W.WDTYPE_NVFP4,
                score=W.SCORE_SIGMOID, expert_scales=(0.52, 1.22)), 2),
]


@pytest.mark.parametrize("wl,world", CASES, ids=[f"{w.name}-r{r}" for w, r in CASES])
def test_the_layer_is_the_sum_of_its_intermediate_slices(wl, world):
    inp = W.make_inputs(wl, "cpu")
    full = oracle_layer(wl, inp).moe_rows(np.arange(wl.T, dtype=np.int32))
    total = np.zeros_like(full)
    for r in range(world):
        part = dict(inp)
        part["w1"] = tp.shard_w1(inp["w1"], r, world)
        part["w1_scale"] = tp.shard_w1(inp["w1_scale"], r, world)
        part["w2"] = tp.shard_w2(inp["w2"], r, world)
        part["w2_scale"] = tp.shard_w2(inp["w2_scale"], r, world)
        total += oracle_layer(wl.with_(I=wl.I // world), part).moe_rows(np.arange(wl.T, dtype=np.int32))
    assert np.allclose(total, full, rtol=1e-9, atol=1e-12 * float(np.abs(full).max()))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        t = torch.full((3, 5), float(rank + 1), dtype=torch.bfloat16)
        ep.TorchExchange().all_reduce(t)
        q.put((rank, t.float().tolist()))
    finally:
        dist.destroy_process_group()


def test_all_reduce_sums_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gloo_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    for _ in range(2):
        _, v = q.get(timeout=10)
        assert v == [[3.0] * 5] * 3


def test_thread_ranks_all_reduce_to_the_same_bits():
    world = 4
    hub = ep.LocalExchange(world)
    ts_ = [torch.randn(4, 8, generator=torch.Generator().manual_seed(r)).to(torch.bfloat16) for r in range(world)]
    want = sum(t.float() for t in ts_).to(torch.bfloat16)
    outs = [t.clone() for t in ts_]

    def run(r):
        hub.for_rank(r).all_reduce(outs[r])

    th = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in th:
        t.start()
    for t in th:
        t.join(timeout=60)
    for o in outs:
        assert torch.equal(o, want)


def test_uneven_intermediate_split_is_rejected():
    from grouped_gemm_swiglu_b200 import MoeDims
    d = MoeDims.of(W.Workload("x", T=1, H=256, I=384, E=4, k=2))
    with pytest.raises(ValueError):
        tp.TensorParallelMoE(d, 0, 2, None, None, exchange=object())
