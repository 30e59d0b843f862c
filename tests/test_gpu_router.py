"""Router / gate epilogue on the GPU against the oracle: ids bit-exact, weights within
1e-6 absolute (fp32), on every workload and on the pages' edge cases (sglang PR #36385:
ties, a dominating shared sink, a tail at T=37, all-negative rows at -40/-90/-200, the
route_scale*global_scale = 10.4 invariant)."""
import json
import os

import numpy as np
import pytest
import scipy.special
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
    moe.moe_route_topk(logits, d, None, ids, w, sw)
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


# ------------------------------------------------------------- correction bias, packed output
# With a bias the device ranks on fp32 sigmoid(logit) + bias and the oracle on the same key
# in fp64; where two keys lie within KEY_TIE of each other both orders are correct, so the
# test checks what is unique (a valid top-k of the fp64 keys) and the rest for validity.
KEY_TIE = 1e-6


def gpu_route_ex(logits, E, k, score, bias, route_scale=1.0):
    T, cols = logits.shape
    S = cols - E
    d = moe.MoeDims(T=T, H=128, I=128, E=E, k=k, n_sink=S, n_shared=0, wdtype=0, score=score, alpha=1.0,
                    beta=0.0, limit=float("inf"), route_scale=route_scale)
    dev = logits.device
    ids = torch.full((T, k), -7, dtype=torch.int32, device=dev)
    w = torch.full((T, k), float("nan"), dtype=torch.float32, device=dev)
    sw = torch.full((T, S), float("nan"), dtype=torch.float32, device=dev) if S else None
    packed = torch.zeros((T, k), dtype=torch.int32, device=dev)
    moe.moe_route_topk(logits, d, bias, ids, w, sw, packed)
    torch.cuda.synchronize()
    return (ids.cpu().numpy(), w.cpu().numpy(), (sw.cpu().numpy() if S else np.zeros((T, 0))),
            packed.cpu().numpy().view(np.uint32))


def check_packed(ids, w, packed):
    """(id << 16) | bf16 bits of the weight, rounded to nearest even (torch's conversion)."""
    wb = torch.from_numpy(w).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).astype(np.uint32)
    assert np.array_equal(packed >> 16, ids.astype(np.uint32))
    assert np.array_equal(packed & 0xFFFF, wb)


def check_biased(logits, E, k, bias, route_scale=1.0):
    ids, w, sw, packed = gpu_route_ex(logits, E, k, 1, bias, route_scale)
    lg, b = f32(logits).astype(np.float64), f32(bias).astype(np.float64)
    oids, ow, osw = oracle.route(f32(logits), E, k, 1, route_scale, bias=f32(bias))
    key = scipy.special.expit(lg[:, :E]) + b
    sig = scipy.special.expit(lg)
    ties = 0
    for t in range(len(lg)):
        sel, rest = key[t, ids[t]], np.delete(key[t], ids[t])
        assert len(set(ids[t].tolist())) == k and ids[t].min() >= 0 and ids[t].max() < E
        assert sel.min() >= rest.max() - KEY_TIE and np.all(np.diff(sel) <= KEY_TIE), f"token {t}"
        if np.array_equal(ids[t], oids[t]):
            assert np.abs(w[t] - ow[t]).max() <= TOL_WEIGHTS * max(1.0, route_scale)
            assert np.abs(sw[t] - osw[t]).max(initial=0) <= TOL_WEIGHTS * max(1.0, route_scale)
        else:
            ties += 1  # a near-tie decided the other way: weights of the device's own selection
            den = sig[t, ids[t]].sum() + sig[t, E:].sum()
            assert np.abs(w[t] - route_scale * sig[t, ids[t]] / den).max() <= TOL_WEIGHTS * max(1.0, route_scale)
    check_packed(ids, w, packed)
    return ids, w, sw, ties


@pytest.mark.parametrize("T,N,S,k,bias_std", [
    (64, 256, 2, 8, 0.05),    # decode shape with sinks, DeepSeek-style small correction bias
    (37, 288, 0, 8, 0.5),     # GLM width, bias comparable to the sigmoid range
    (200, 128, 0, 6, 0.02),
])
def test_router_correction_bias(T, N, S, k, bias_std):
    g = torch.Generator().manual_seed(T + N)
    logits = torch.randn((T, N + S), generator=g) * 1.5
    bias = torch.randn((N,), generator=g) * bias_std
    _, _, _, ties = check_biased(logits.cuda(), N, k, bias.cuda())
    assert ties <= 2


def test_router_bias_under_fp32_saturation():
    """sigmoid is exactly 1 above ~17 and exactly 0 below ~-104 in fp32: the bias alone then
    ranks, and equal biases fall back to the lower id (any order of near-equal fp64 keys is
    accepted); the weights still come from the raw logits and stay finite."""
    g = torch.Generator().manual_seed(5)
    N, S, k = 256, 2, 8
    logits = torch.randn((48, N + S), generator=g)
    logits[:16, :N] = 20 + 10 * torch.rand((16, N), generator=g)   # saturated at 1
    logits[16:32] = -150 + 5 * torch.rand((16, N + S), generator=g)  # saturated at 0
    bias = torch.round(torch.randn((N,), generator=g) * 4) / 8       # many equal biases
    ids, w, sw, _ = check_biased(logits.cuda(), N, k, bias.cuda())
    assert np.all(np.isfinite(w)) and np.all(np.isfinite(sw))
    b = bias.numpy()
    for t in range(32):  # saturated rows: the selection is a top-k of the bias, lower id on ties
        want = sorted(range(N), key=lambda e: (-b[e], e))[:k]
        assert list(ids[t]) == want


def test_router_dominant_bias_forces_ids():
    g = torch.Generator().manual_seed(6)
    N, S, k = 256, 2, 8
    logits = torch.randn((32, N + S), generator=g) * 3
    bias = 10.0 * torch.randperm(N, generator=g).float()
    ids, _, _, ties = check_biased(logits.cuda(), N, k, bias.cuda(), route_scale=2.5)
    want = torch.argsort(-bias)[:k].numpy()
    assert ties == 0 and np.all(ids == want[None, :])


@pytest.mark.parametrize("score", [0, 1])
def test_router_packed_output_without_bias(score):
    g = torch.Generator().manual_seed(7 + score)
    N, k = 128, 6
    logits = (torch.randn((50, N), generator=g) * 2).cuda()
    ids, w, _, packed = gpu_route_ex(logits, N, k, score, None)
    oids, ow, _ = oracle.route(f32(logits), N, k, score)
    assert np.array_equal(ids, oids) and np.abs(w - ow).max() <= TOL_WEIGHTS
    check_packed(ids, w, packed)
