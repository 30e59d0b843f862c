"""Router / gate epilogue on the GPU against the oracle: ids bit-exact, weights within
1e-6 absolute (fp32), on every workload and on the pages' edge cases (sglang PR #36385:
ties, a dominating shared sink, a tail at T=37, all-negative rows at -40/-90/-200, the
route_scale*global_scale = 10.4 invariant)."""
import json
import os

import numpy as np
import pytest
import torch

import oracle
import grouped_gemm_swiglu_b200 as moe
from grouped_gemm_swiglu_b200 import workloads as W
from helpers import TOL_WEIGHTS, f32

pytestmark = pytest.mark.gpu
GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_constants.json")))


def gpu_route(logits: torch.Tensor, E: int, k: int, score: int, route_scale=1.0):
    T, cols = logits.shape
    S = cols - E
    d = moe.MoeDims(T=T, H=128, I=128, E=E, k=k, n_sink=S, n_shared=0, wdtype=0, score=score, alpha=1.0,
                    beta=0.0, limit=float("inf"), route_scale=route_scale)
    dev = logits.device
    ids = torch.full((T, k), -7, dtype=torch.int32, device=dev)
    w = torch.full((T, k), float("nan"), dtype=torch.float32, device=dev)
    sw = torch.full((T, S), float("nan"), dtype=torch.float32, device=dev) if S else None
    moe.moe_route_topk(logits, d, ids, w, sw)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy(), (sw.cpu().numpy() if S else np.zeros((T, 0)))


def check(logits: torch.Tensor, E, k, score, route_scale=1.0):
    ids, w, sw = gpu_route(logits, E, k, score, route_scale)
    oids, ow, osw = oracle.route(f32(logits), E, k, score, route_scale)
    assert np.array_equal(ids, oids), f"id mismatch in rows {np.where((ids != oids).any(1))[0][:10]}"
    assert np.all(np.isfinite(w)) and np.all(np.isfinite(sw))
    err = max(np.abs(w - ow).max(initial=0), np.abs(sw - osw).max(initial=0))
    assert err <= TOL_WEIGHTS * max(1.0, abs(route_scale)), f"max weight error {err:.3e}"
    return ids, w, sw


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_router_on_workloads(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, "cuda")
    check(inp["logits"], wl.E, wl.k, wl.score, wl.route_scale)


@pytest.mark.parametrize("T,N,S,k,score", [
    (37, 256, 2, 6, 1),     # Inkling gate shape with a BLOCK tail
    (37, 256, 0, 6, 0),
    (5, 9, 0, 9, 0),        # k = E, width not a multiple of 32
    (64, 288, 0, 8, 1),     # GLM width
    (16, 1000, 2, 30, 1),   # widest supported row, k + sinks = 32
    (16, 33, 0, 1, 0),      # k = 1: weight 1
    (200, 64, 0, 32, 0),
])
def test_router_ties_and_shapes(T, N, S, k, score):
    g = torch.Generator().manual_seed(T * 7 + N)
    logits = torch.randint(-3, 3, (T, N + S), generator=g).float()  # exact ties everywhere
    logits[::2] += torch.randn((len(logits[::2]), N + S), generator=g)
    check(logits.cuda(), N, k, score)


@pytest.mark.parametrize("base", GOLD["all_negative_bases"]["bases"])
def test_router_all_negative_rows(base):
    g = torch.Generator().manual_seed(int(-base))
    N, S, k = GOLD["inkling_gate"]["routed"], GOLD["inkling_gate"]["sinks"], GOLD["inkling_gate"]["top_k"]
    logits = base + 5 * (torch.rand((64, N + S), generator=g) - 0.5)
    logits[:4] = torch.tensor(base).expand(4, N + S)  # whole rows of exact ties
    _, w, sw = check(logits.cuda(), N, k, 1)
    total = w.sum(1) + sw.sum(1)
    assert np.all(np.abs(total - 1.0) < 1e-6)


def test_router_dominating_sink_and_invariant():
    inv = GOLD["free_invariant"]
    g = torch.Generator().manual_seed(3)
    N, S, k = 256, 2, 6
    logits = torch.randn((128, N + S), generator=g) * 2
    _, w, sw = check(logits.cuda(), N, k, 1, inv["route_scale_times_global_scale"])
    total = w.sum(1) + sw.sum(1)
    assert np.all(total >= inv["observed_min"] - 1e-6) and np.all(total <= inv["observed_max"] + 1e-6)
    logits[:, :N] -= 40.0
    logits[:, N] = 50.0
    logits[:, N + 1] = -40.0
    _, w, sw = check(logits.cuda(), N, k, 1)
    assert np.all(sw[:, 0] > 1 - 1e-6) and np.all(w.sum(1) < 1e-6)


def test_router_empty_batch():
    ids, w, sw = gpu_route(torch.zeros((0, 258), device="cuda"), 256, 6, 1)
    assert ids.shape == (0, 6)
