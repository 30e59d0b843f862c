"""The bench's multi-rank plumbing on CPU: two `gloo` ranks started the way torchrun starts
them (RANK, LOCAL_RANK, WORLD_SIZE, MASTER_ADDR/PORT on 127.0.0.1). The layer is
token-parallel (each rank its own batch, replicated weights, no data-path collective), so
what N > 1 adds is the barrier around the timed region, the MAX over ranks of every timing
and the whole-job rate; the reference arm runs on rank 0 alone."""
import argparse
import importlib.util
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, step_ms: list, q):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    bench = _load_bench()
    r = bench.Ranks("gloo", timeout_s=60)
    r.barrier()
    ms = r.max_over_ranks(step_ms[rank])
    stages = {k: r.max_over_ranks(v * (rank + 1)) for k, v in (("route", 0.01), ("experts", 0.05))}
    rate = r.rate(256, ms)
    r.barrier()
    q.put((rank, r.world, ms, stages, rate))
    r.close()


@pytest.mark.parametrize("step_ms", [[0.090, 0.087], [0.080, 0.095]])
def test_two_gloo_ranks_report_the_slowest_rank_and_every_ranks_tokens(step_ms):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, step_ms, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=10) for _ in range(2))
    slowest = max(step_ms)
    for rank, world, ms, stages, rate in res:
        assert world == 2
        assert ms == pytest.approx(slowest)  # every rank sees the same, slowest time
        assert stages["route"] == pytest.approx(0.02) and stages["experts"] == pytest.approx(0.10)
        assert rate == pytest.approx(2 * 256 / (slowest / 1e3))  # both ranks' tokens, slowest clock


def test_single_process_needs_no_process_group(monkeypatch):
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE"):
        monkeypatch.delenv(k, raising=False)
    bench = _load_bench()
    r = bench.Ranks("gloo")
    assert r.world == 1 and r.rank == 0
    r.barrier()
    assert r.max_over_ranks(1.25) == 1.25 and r.rate(16, 2.0) == pytest.approx(8000.0)
    r.close()


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    bench = _load_bench()
    args = argparse.Namespace(impl="reference", gpus=2, steps=3, warmup=3, workload=None, tokens=None,
                              experts=None, no_cpu_baseline=True, cpu_seconds=1.0)
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""  # the other ranks exit 0 without work or output
