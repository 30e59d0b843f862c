"""bench.py --mode ep|tp on CPU: two gloo ranks (as torchrun starts them, on 127.0.0.1)
drive the expert-parallel and tensor-parallel timing loop with plain-torch stand-ins for
the library calls and print one JSON line from rank 0. What is checked is the plumbing:
the layer runs on every rank, the slowest rank's time is reported, the whole-job rate
counts every rank's tokens for expert parallelism and the shared tokens once for tensor
parallelism, and the line names the mode. The kernels run the same layers on a GPU in
test_gpu_ep.py and test_gpu_tp.py."""
import importlib.util
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from test_ep import CpuOps, _one_rank

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_par", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class ToyOps(CpuOps):
    """CpuOps with tensor-shaped toy weights (an expert scales by the mean of its W1 slice
    and shifts by the mean of its W2 slice) and the one-call layer the tensor-parallel
    path uses."""

    @staticmethod
    def moe_workspace_size(d, kind):
        return 4

    @staticmethod
    def moe_experts(x_perm, xs, offsets, w1, w1s, gs, us, lim, w2, w2s, d, h, hs, y, ws):
        o = offsets.tolist()
        for g in range(d.E + d.n_shared):
            a, b = float(w1[g].double().mean()), float(w2[g].double().mean())
            y[o[g]:o[g + 1]] = (x_perm[o[g]:o[g + 1]].double() * a + b).to(torch.bfloat16)

    @staticmethod
    def moe_forward(logits, bias, x, w1, w1s, gs, us, lim, w2, w2s, d, out, ws=None):
        out.copy_(_one_rank(d, logits, x, w1, w2, ops=ToyOps))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, mode, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    bench = _load_bench()
    from grouped_gemm_swiglu_b200 import workloads as W
    from grouped_gemm_swiglu_b200._lib import MoeDims
    ranks = bench.Ranks("gloo", torch.device("cpu"), timeout_s=60)
    try:
        wl = W.Workload("toy", T=6, H=128, I=256, E=4, k=2, n_shared=1, score=W.SCORE_SOFTMAX)
        g = torch.Generator().manual_seed(3)
        inp = {"dims": MoeDims.of(wl),
               "x": torch.randn((wl.T, wl.H), generator=g).to(torch.bfloat16),
               "logits": torch.randn((wl.T, wl.E), generator=g),
               "w1": torch.rand((wl.G, 2 * wl.I), generator=g) + 0.5,
               "w2": torch.randn((wl.G, wl.I), generator=g)}
        line = bench.parallel_bench(mode, wl, ranks, "cpu", K=3, Wm=1, ops=ToyOps, inputs=inp)
        q.put((rank, line))
    finally:
        ranks.close()


@pytest.mark.parametrize("mode", ["ep", "tp"])
def test_parallel_modes_on_two_gloo_ranks(mode):
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    lines = dict(q.get(timeout=10) for _ in range(world))
    line = lines[0]
    assert line["n_gpus"] == 2 and line["status"] == 0 and line["config"]["parallelism"] == f"{mode}2"
    assert line["scaling"] == ("weak" if mode == "ep" else "strong")
    # the reported step is the slowest rank's, identical on both ranks
    assert lines[1]["ms_per_step"] == line["ms_per_step"] > 0
    tokens = 2 * 6 if mode == "ep" else 6
    assert line["value"] == pytest.approx(tokens / (line["ms_per_step"] / 1e3))
