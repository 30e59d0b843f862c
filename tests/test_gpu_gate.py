"""Fused gate GEMV + router (moe_gate_route) on the GPU: the logits against the fp64
oracle GEMV within the fp32 summation bound, the routing against the oracle on the
device's own fp32 logits (ids bit-exact, weights 1e-6) and against the oracle's routing of
its own fp64 logits wherever the top-k gaps exceed that bound, the packed form, and reuse."""
import numpy as np
import pytest
import scipy.special
import torch

import oracle
import grouped_gemm_swiglu_b200 as moe
from helpers import TOL_WEIGHTS, f32

pytestmark = pytest.mark.gpu


def bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def run_gate(T, H, N, S, k, score, seed, bias_std=0.0, route_scale=1.0):
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn((T, H), generator=g, device="cuda").to(torch.bfloat16)
    wg = (torch.randn((N + S, H), generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    bias = (torch.randn((N,), generator=g, device="cuda") * bias_std) if bias_std else None
    d = moe.MoeDims(T=T, H=H, I=128, E=N, k=k, n_sink=S, n_shared=0, wdtype=0, score=score, alpha=1.0, beta=0.0,
                    limit=float("inf"), route_scale=route_scale)
    ws = moe.alloc_workspace(d, moe.MOE_WS_GATE_ROUTE)
    logits = torch.full((T, N + S), float("nan"), device="cuda")
    ids = torch.full((T, k), -1, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), float("nan"), device="cuda")
    sw = torch.full((T, S), float("nan"), device="cuda") if S else None
    packed = torch.zeros((T, k), dtype=torch.int32, device="cuda")
    outs = []
    for _ in range(2):  # the completion counter is left at zero: a second call repeats the first
        moe.moe_gate_route(x, wg, d, bias, logits, ids, w, sw, packed, ws)
        torch.cuda.synchronize()
        outs.append([t.clone() for t in (logits, ids, w, packed)])
    for a, b in zip(*outs):
        assert torch.equal(a, b)
    assert moe.moe_read_status(ws) == 0
    return x, wg, bias, logits, ids, w, sw, packed


@pytest.mark.parametrize("T,H,N,S,k,score,bias_std", [
    (1, 4096, 256, 2, 8, 1, 0.0),     # decode, Inkling-like gate (256 routed + 2 sinks)
    (4, 4096, 256, 2, 6, 1, 0.05),    # the pages' fused path bound (<= 4 tokens), with a bias
    (3, 4096, 288, 0, 8, 1, 0.0),     # GLM width
    (8, 2048, 128, 0, 8, 0, 0.0),     # softmax scoring
    (16, 1024, 32, 0, 4, 0, 0.0),     # the largest supported batch
    (5, 128, 9, 0, 9, 0, 0.0),        # tiny row: k = E, H = 128
])
def test_gate_route_matches_oracle(T, H, N, S, k, score, bias_std):
    x, wg, bias, logits, ids, w, sw, packed = run_gate(T, H, N, S, k, score, seed=T * 31 + N, bias_std=bias_std)
    # GEMV: each lane sums H/128 exact bf16 products in fp32, then 5 shuffle levels and 3
    # partial adds: |error| <= (H/128 + 8) * 2^-24 * sum_h |x_h w_h|
    ref = oracle.gate_logits(bits(x), bits(wg))
    mag = np.abs(f32(x).astype(np.float64)) @ np.abs(f32(wg).astype(np.float64)).T
    bound = (H / 128 + 8) * 2.0 ** -24 * mag
    err = np.abs(f32(logits) - ref)
    assert np.all(err <= bound), f"max err/bound {np.max(err / np.maximum(bound, 1e-300)):.3f}"
    # Routing of the device's own fp32 logits: decided in the same precision on both sides
    got_ids, got_w = ids.cpu().numpy(), w.cpu().numpy()
    lg = f32(logits)
    if bias is None:
        o_ids, o_w, o_sw = oracle.route(lg, N, k, score)
        assert np.array_equal(got_ids, o_ids)
        assert np.abs(got_w - o_w).max() <= TOL_WEIGHTS
        if S:
            assert np.abs(sw.cpu().numpy() - o_sw).max() <= TOL_WEIGHTS
    else:  # fp32 key on the device, fp64 in the oracle: a valid top-k up to 1e-6 near-ties
        key = scipy.special.expit(lg[:, :N].astype(np.float64)) + f32(bias)
        for t in range(T):
            sel, rest = key[t, got_ids[t]], np.delete(key[t], got_ids[t])
            assert sel.min() >= rest.max() - 1e-6 and len(set(got_ids[t].tolist())) == k
        sig = scipy.special.expit(lg.astype(np.float64))
        den = np.take_along_axis(sig, got_ids.astype(np.int64), 1).sum(1) + sig[:, N:].sum(1)
        want = np.take_along_axis(sig, got_ids.astype(np.int64), 1) / den[:, None]
        assert np.abs(got_w - want).max() <= TOL_WEIGHTS
    # Routing of the oracle's own fp64 logits: wherever the fp64 gaps around the selection
    # exceed twice the fp32 summation bound (plus the fp32 rounding of each side), the
    # device's fp32 logits cannot reorder them, so its selection (and, where every gap in
    # the top k + 1 is that wide, its slot order) must be the oracle's.
    if bias is None:
        r_ids, _, _ = oracle.route(ref.astype(np.float32), N, k, score)
        n_set = n_order = 0
        for t in range(T):
            r = ref[t, :N]
            tol = 2 * bound[t, :N].max() + 2 * float(np.spacing(np.float32(np.abs(r).max())))
            order = np.lexsort((np.arange(N), -r))[:k + 1]
            gaps = r[order[:-1]] - r[order[1:]]
            if k == N or gaps[k - 1] > tol:
                assert set(got_ids[t].tolist()) == set(r_ids[t].tolist()), t
                n_set += 1
            if k == N or gaps[:k].min() > tol:
                assert np.array_equal(got_ids[t], r_ids[t]), t
                n_order += 1
        assert n_set >= 1, "no token's top-k gap exceeds the fp32 bound: the fp64 comparison checked nothing"
    pk = packed.cpu().numpy().view(np.uint32)
    wb = w.cpu().to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).astype(np.uint32)
    assert np.array_equal(pk >> 16, got_ids.astype(np.uint32)) and np.array_equal(pk & 0xFFFF, wb)


def test_gate_route_logits_in_workspace_match_the_returned_ones():
    T, H, N, S, k = 2, 4096, 256, 2, 8
    x, wg, _, logits, ids, w, _, _ = run_gate(T, H, N, S, k, 1, seed=5)
    d = moe.MoeDims(T=T, H=H, I=128, E=N, k=k, n_sink=S, n_shared=0, wdtype=0, score=1, alpha=1.0, beta=0.0,
                    limit=float("inf"), route_scale=1.0)
    ws = moe.alloc_workspace(d, moe.MOE_WS_GATE_ROUTE)
    ids2 = torch.empty_like(ids)
    w2 = torch.empty_like(w)
    sw2 = torch.empty((T, S), device="cuda")
    moe.moe_gate_route(x, wg, d, None, None, ids2, w2, sw2, None, ws)  # logits kept in the workspace
    torch.cuda.synchronize()
    assert torch.equal(ids, ids2) and torch.equal(w, w2)
