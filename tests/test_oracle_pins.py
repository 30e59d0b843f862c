"""Pins of the fp64 oracle against things other than itself (CPU only).

Each test ties one oracle function to a fact the pages or the mathematics fix: a
library routine for a special case, brute force on tiny inputs, a closed form, an
invariant, or a constant the pages print (tests/golden/pages_constants.json).
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_constants.json")))


# --------------------------------------------------------------------------- E4M3

def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert nan.sum() == 2  # 0x7F and 0xFF
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9


def test_e4m3_encode_matches_torch_rne_in_range():
    rng = np.random.default_rng(1)
    v = np.concatenate([
        rng.normal(0, 50, 4000), rng.normal(0, 0.01, 2000), rng.uniform(-447, 447, 2000),
        rng.normal(0, 2 ** -7, 1000),  # subnormal range
    ]).astype(np.float32)
    ours = oracle.e4m3_encode(v)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encode_ties_to_even_and_saturation():
    grid = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    exact = mids.astype(np.float64) == (grid[:-1] + grid[1:]) / 2
    codes = oracle.e4m3_encode(mids[exact])
    assert np.all(codes % 2 == 0), "a midpoint must round to the even code"
    ref = torch.from_numpy(mids[exact]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)
    big = np.array([448.0, 449.0, 470.0, 1e6, -500.0, -448.5], dtype=np.float32)
    assert list(oracle.e4m3_encode(big)) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert oracle.e4m3_encode(np.array([-1e-6], np.float32))[0] == 0x80  # sign kept on zero
    assert oracle.e4m3_encode(np.array([np.nan], np.float32))[0] == 0x7F


def test_quant_1x128_block_properties():
    rng = np.random.default_rng(2)
    v = rng.normal(0, 3, (5, 512)).astype(np.float32)
    v[2, 128:256] = 0.0
    q, s = oracle.quant_1x128(v)
    assert s.shape == (5, 4)
    assert s[2, 1] == 1.0 and np.all(q[2, 128:256] == 0)
    deq = oracle.e4m3_decode(q) * np.repeat(s, 128, axis=1)
    for r in range(5):
        for b in range(4):
            blk = v[r, b * 128:(b + 1) * 128]
            if not np.any(blk):
                continue
            j = int(np.argmax(np.abs(blk)))
            assert q[r, b * 128 + j] & 0x7F == 0x7E  # the block maximum maps to +-448
            assert s[r, b] == np.float32(np.abs(blk).max()) / np.float32(448.0)
    # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 above the subnormal range.
    scaled = np.abs(v) / np.repeat(s, 128, axis=1)
    normal = scaled >= 2 ** -6
    err = np.abs(deq - v)
    assert np.all(err[normal] <= np.abs(v[normal]) * 2 ** -4 * (1 + 1e-6))
    assert np.all(err[~normal] <= np.repeat(s, 128, axis=1)[~normal] * 2 ** -10 * (1 + 1e-6))


# --------------------------------------------------------------------------- SwiGLU

def test_swiglu_standard_reduces_to_silu_times_up():
    rng = np.random.default_rng(3)
    g = rng.normal(0, 4, 200)
    u = rng.normal(0, 4, 200)
    p = GOLD["standard_swiglu"]
    ours = oracle.swiglu(g, u, p["alpha"], p["up_bias"], math.inf)
    ref = (torch.nn.functional.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    np.testing.assert_allclose(ours, ref, rtol=1e-14, atol=1e-300)


@pytest.mark.parametrize("params", ["oai_swiglu", "glm_clamp"])
def test_swiglu_clamp_boundaries(params):
    p = GOLD[params]
    L = p.get("clamp", p.get("limit"))
    a = p.get("alpha", 1.0)
    b = p.get("up_bias", 0.0)
    f = lambda g, u: float(oracle.swiglu(np.array([g]), np.array([u]), a, b, L)[0])
    # gate is clamped from above only
    for g in [L, L + 1e-9, L + 3.0, 1e6]:
        assert f(g, 1.5) == f(L, 1.5)
    assert f(-50.0, 1.5) != f(-L, 1.5)
    assert f(np.nextafter(L, 0), 1.5) < f(L, 1.5)
    # up is clamped on both sides
    for u in [L, L + 0.5, 1e6]:
        assert f(2.0, u) == f(2.0, L)
    for u in [-L, -L - 0.5, -1e6]:
        assert f(2.0, u) == f(2.0, -L)
    assert f(2.0, np.nextafter(L, 0)) < f(2.0, L)
    # the lower gate side stays unclamped: at alpha = 1, beta = 0 it is silu(g)*u
    if a == 1.0 and b == 0.0:
        ref = float(torch.nn.functional.silu(torch.tensor(-50.0, dtype=torch.float64)) * 1.5)
        assert f(-50.0, 1.5) == pytest.approx(ref, rel=1e-13)


@pytest.mark.parametrize("alpha", [1.0, 1.702, 0.5])
def test_swiglu_alpha_beta_identities(alpha):
    beta = GOLD["oai_swiglu"]["up_bias"]
    L = 7.0
    f = lambda g, u, b=0.0: float(oracle.swiglu(np.array([g]), np.array([u]), alpha, b, L)[0])
    # g*sigmoid(a g) + g*sigmoid(-a g) = g: f(g) - f(-g) = g with u = 1, beta = 0
    for g in [0.3, 1.0, 2.5, 6.0]:
        assert f(g, 1.0) - f(-g, 1.0) == pytest.approx(g, rel=1e-13)
    # curvature at 0 is alpha/2: (f(e) + f(-e)) / e^2 -> alpha / 2
    e = 1e-4
    assert (f(e, 1.0) + f(-e, 1.0)) / e ** 2 == pytest.approx(alpha / 2, rel=1e-6)
    # beta shifts the up value: zero at u = -beta, linear in u with slope f(g, 1)
    assert f(1.3, -beta, beta) == 0.0
    assert f(1.3, 2.0, beta) - f(1.3, 1.0, beta) == pytest.approx(f(1.3, 1.0), rel=1e-13)
    # large gate: sigmoid -> 1, output -> L_clamped gate * (u + beta)
    assert f(1e3, 2.0, beta) == pytest.approx(L * scipy.special.expit(alpha * L) * (2.0 + beta), rel=1e-14)


# --------------------------------------------------------------------------- router

def _brute_topk(row, k):
    order = sorted(range(len(row)), key=lambda e: (-float(row[e]), e))
    return order[:k]


@pytest.mark.parametrize("T,N,k", [(37, 16, 4), (20, 9, 9), (50, 12, 1), (30, 40, 6)])
def test_route_selection_brute_force_with_ties(T, N, k):
    rng = np.random.default_rng(T * 100 + N)
    logits = rng.integers(-3, 3, (T, N)).astype(np.float32)  # many exact ties
    logits[::3] += rng.normal(0, 1, (len(logits[::3]), N)).astype(np.float32)
    ids, w, _ = oracle.route(logits, N, k, oracle.SCORE_SOFTMAX)
    for t in range(T):
        assert list(ids[t]) == _brute_topk(logits[t], k)
        assert len(set(ids[t])) == k


def test_route_softmax_weights_match_torch_softmax():
    rng = np.random.default_rng(5)
    logits = rng.normal(0, 3, (64, 32)).astype(np.float32)
    ids, w, _ = oracle.route(logits, 32, 5, oracle.SCORE_SOFTMAX)
    sel = np.take_along_axis(logits.astype(np.float64), ids.astype(np.int64), 1)
    ref = torch.softmax(torch.from_numpy(sel), dim=1).numpy()
    np.testing.assert_allclose(w, ref, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("S", [0, 2])
def test_route_sigmoid_weights_are_sigma_ratios(S):
    rng = np.random.default_rng(6 + S)
    N, k = 64, 6
    logits = rng.normal(0, 3, (48, N + S)).astype(np.float32)
    ids, w, sw = oracle.route(logits, N, k, oracle.SCORE_SIGMOID, 1.0)
    sig = scipy.special.expit(logits.astype(np.float64))
    sel = np.take_along_axis(sig, ids.astype(np.int64), 1)
    den = sel.sum(1) + (sig[:, N:].sum(1) if S else 0)
    np.testing.assert_allclose(w, sel / den[:, None], rtol=1e-12)
    if S:
        np.testing.assert_allclose(sw, sig[:, N:] / den[:, None], rtol=1e-12)


@pytest.mark.parametrize("base", GOLD["all_negative_bases"]["bases"])
def test_route_all_negative_rows_finite(base):
    # Below -104 fp32 sigmoid is 0; sigmoid(x) = e^x (1 - e^x + ...), so for x << 0 the
    # weights equal a softmax over the same logits to within e^base relative.
    rng = np.random.default_rng(int(-base))
    N, S, k = GOLD["inkling_gate"]["routed"], GOLD["inkling_gate"]["sinks"], GOLD["inkling_gate"]["top_k"]
    logits = (base + rng.uniform(-5, 5, (8, N + S))).astype(np.float32)
    ids, w, sw = oracle.route(logits, N, k, oracle.SCORE_SIGMOID)
    assert np.all(np.isfinite(w)) and np.all(np.isfinite(sw))
    sel = np.take_along_axis(logits.astype(np.float64), ids.astype(np.int64), 1)
    allv = np.concatenate([sel, logits[:, N:].astype(np.float64)], 1)
    ref = torch.softmax(torch.from_numpy(allv), 1).numpy()
    np.testing.assert_allclose(np.concatenate([w, sw], 1), ref, rtol=max(1e-12, 4 * math.exp(base + 5)))


def test_route_free_invariant_and_dominating_sink():
    inv = GOLD["free_invariant"]["route_scale_times_global_scale"]
    rng = np.random.default_rng(9)
    N, S, k = 256, 2, 6
    logits = rng.normal(0, 2, (16, N + S)).astype(np.float32)
    _, w, sw = oracle.route(logits, N, k, oracle.SCORE_SIGMOID, inv)
    np.testing.assert_allclose(w.sum(1) + sw.sum(1), inv, rtol=1e-14)
    # sigmoid saturates at 1, so a sink dominates only against small routed sigmoids:
    # routed near -40 give sigma < e^-30 each, a sink at +50 gives sigma ~ 1.
    logits[:, :N] -= 40.0
    logits[:, N] = 50.0
    logits[:, N + 1] = -40.0
    _, w, sw = oracle.route(logits, N, k, oracle.SCORE_SIGMOID, 1.0)
    assert np.all(sw[:, 0] > 1 - 1e-12) and np.all(w.sum(1) < 1e-12)
    assert np.all(w > 0)


def test_route_rejects_sinks_with_softmax():
    with pytest.raises(ValueError):
        oracle.route(np.zeros((2, 10), np.float32), 8, 2, oracle.SCORE_SOFTMAX)


def test_route_zero_bias_keeps_the_raw_logit_order():
    # sigmoid is increasing, so a zero correction bias ranks exactly like the raw logit
    rng = np.random.default_rng(21)
    N, S, k = 64, 2, 6
    logits = rng.normal(0, 3, (40, N + S)).astype(np.float32)
    ids0, w0, sw0 = oracle.route(logits, N, k, oracle.SCORE_SIGMOID)
    ids1, w1, sw1 = oracle.route(logits, N, k, oracle.SCORE_SIGMOID, bias=np.zeros(N, np.float32))
    assert np.array_equal(ids0, ids1)
    np.testing.assert_array_equal(w0, w1)
    np.testing.assert_array_equal(sw0, sw1)


def test_route_dominant_bias_forces_the_selection_and_not_the_weights():
    # sigmoid lies in (0, 1): bias gaps of 10 decide the ranking whatever the logits, and
    # the weights still come from the raw logits of the selected columns.
    rng = np.random.default_rng(22)
    N, S, k = 32, 2, 5
    logits = rng.normal(0, 4, (24, N + S)).astype(np.float32)
    bias = (10.0 * rng.permutation(N)).astype(np.float32)
    ids, w, sw = oracle.route(logits, N, k, oracle.SCORE_SIGMOID, 1.0, bias=bias)
    want = np.argsort(-bias, kind="stable")[:k]
    sig = scipy.special.expit(logits.astype(np.float64))
    for t in range(len(logits)):
        assert list(ids[t]) == list(want)
        den = sig[t, want].sum() + sig[t, N:].sum()
        np.testing.assert_allclose(w[t], sig[t, want] / den, rtol=1e-12)
        np.testing.assert_allclose(sw[t], sig[t, N:] / den, rtol=1e-12)


@pytest.mark.parametrize("scale", [0.02, 0.3])
def test_route_bias_selection_is_the_top_k_of_sigmoid_plus_bias(scale):
    rng = np.random.default_rng(23)
    N, k = 48, 8
    logits = rng.normal(0, 2, (64, N)).astype(np.float32)
    bias = rng.normal(0, scale, N).astype(np.float32)
    ids, _, _ = oracle.route(logits, N, k, oracle.SCORE_SIGMOID, bias=bias)
    key = scipy.special.expit(logits.astype(np.float64)) + bias.astype(np.float64)
    for t in range(len(logits)):
        sel = key[t, ids[t]]
        rest = np.delete(key[t], ids[t])
        assert np.all(np.diff(sel) <= 0)          # descending key order
        assert sel.min() >= rest.max()            # nothing outside beats what is inside
        assert len(set(ids[t])) == k


def test_route_rejects_bias_with_softmax():
    with pytest.raises(ValueError):
        oracle.route(np.zeros((2, 8), np.float32), 8, 2, oracle.SCORE_SOFTMAX, bias=np.zeros(8, np.float32))


def test_gate_logits_match_torch_fp64_matmul():
    # bf16 values are exact in fp64; torch's own bf16 -> fp64 conversion and matmul
    rng = np.random.default_rng(24)
    x = torch.from_numpy(rng.normal(0, 1, (5, 512))).to(torch.bfloat16)
    w = torch.from_numpy(rng.normal(0, 0.05, (258, 512))).to(torch.bfloat16)
    got = oracle.gate_logits(x.view(torch.int16).numpy().view(np.uint16), w.view(torch.int16).numpy().view(np.uint16))
    ref = (x.double() @ w.double().T).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------- permute

@pytest.mark.parametrize("T,E,k,S", [(37, 8, 2, 0), (100, 16, 4, 1), (5, 300, 8, 2), (1, 4, 4, 0)])
def test_permute_brute_force(T, E, k, S):
    rng = np.random.default_rng(T + E)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    offsets, perm, inv = oracle.permute(ids, E, S)
    entries = sorted([(int(ids[t, j]), t, j) for t in range(T) for j in range(k)])
    entries += [(E + s, t, -1) for s in range(S) for t in range(T)]
    assert len(perm) == len(entries) == offsets[-1]
    for r, (e, t, j) in enumerate(entries):
        assert perm[r] == t
        assert offsets[e] <= r < offsets[e + 1]
        if j >= 0:
            assert inv[t, j] == r
    assert np.array_equal(np.sort(inv.ravel()), np.sort(np.setdiff1d(np.arange(len(perm)),
                                                                     np.arange(offsets[E], offsets[-1]))))


def test_permute_rejects_out_of_range_ids():
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 8]], np.int32), 8)
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, -1]], np.int32), 8)


# --------------------------------------------------------------------------- layer

def _bf16_bits(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _bf16_val(bits):
    return oracle.bf16_to_double(bits)


def _mk_layer(rng, T, H, I, E, k, S=0, n_shared=0, score=oracle.SCORE_SOFTMAX, alpha=1.0, beta=0.0,
              limit=math.inf, rs=1.0, gs=None, us=None, w_mult=1.0):
    G = E + n_shared
    x = _bf16_bits(rng.normal(0, 1, (T, H)))
    w1 = _bf16_bits(rng.normal(0, 0.05 * w_mult, (G, 2 * I, H)))
    w2 = _bf16_bits(rng.normal(0, 0.05, (G, H, I)))
    logits = rng.normal(0, 1, (T, E + S)).astype(np.float32)
    return dict(T=T, H=H, I=I, E=E, k=k, n_sink=S, n_shared=n_shared, wdtype=oracle.WDTYPE_BF16,
                score=score, alpha=alpha, beta=beta, limit=limit, route_scale=rs, logits=logits,
                x=x, w1=w1, w2=w2, gate_scale=gs, up_scale=us)


def _dense_mlp(x, w1, w2, I):
    xt = torch.from_numpy(x)
    g = xt @ torch.from_numpy(w1[:I]).T
    u = xt @ torch.from_numpy(w1[I:]).T
    return ((torch.nn.functional.silu(g) * u) @ torch.from_numpy(w2).T).numpy()


def test_layer_single_expert_is_dense_swiglu_mlp():
    rng = np.random.default_rng(11)
    d = _mk_layer(rng, T=6, H=128, I=64, E=1, k=1)
    L = oracle.Layer(**d)
    out = L.moe_rows(np.arange(6))
    ref = _dense_mlp(_bf16_val(d["x"]), _bf16_val(d["w1"][0]), _bf16_val(d["w2"][0]), 64)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-13)


def test_layer_all_experts_sigmoid_is_weighted_sum_of_mlps():
    rng = np.random.default_rng(12)
    E, I = 4, 32
    d = _mk_layer(rng, T=5, H=128, I=I, E=E, k=E, score=oracle.SCORE_SIGMOID)
    out = oracle.Layer(**d).moe_rows(np.arange(5))
    x = _bf16_val(d["x"])
    sig = scipy.special.expit(d["logits"].astype(np.float64))
    wts = sig / sig.sum(1, keepdims=True)
    ref = sum(wts[:, e:e + 1] * _dense_mlp(x, _bf16_val(d["w1"][e]), _bf16_val(d["w2"][e]), I) for e in range(E))
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_layer_shared_expert_adds_its_dense_mlp():
    rng = np.random.default_rng(13)
    I = 32
    d = _mk_layer(rng, T=4, H=128, I=I, E=6, k=2, n_shared=1)
    with_sh = oracle.Layer(**d).moe_rows(np.arange(4))
    d0 = dict(d, n_shared=0, w1=d["w1"][:6], w2=d["w2"][:6])
    without = oracle.Layer(**d0).moe_rows(np.arange(4))
    ref = _dense_mlp(_bf16_val(d["x"]), _bf16_val(d["w1"][6]), _bf16_val(d["w2"][6]), I)
    np.testing.assert_allclose(with_sh - without, ref, rtol=1e-9, atol=1e-12)


def test_layer_sink_gated_shared_experts_use_sink_weights():
    rng = np.random.default_rng(14)
    I, E, S = 32, 8, 2
    d = _mk_layer(rng, T=3, H=128, I=I, E=E, k=2, S=S, n_shared=S, score=oracle.SCORE_SIGMOID)
    out = oracle.Layer(**d).moe_rows(np.arange(3))
    ids, w, sw = oracle.route(d["logits"], E, 2, oracle.SCORE_SIGMOID)
    x = _bf16_val(d["x"])
    for t in range(3):
        ref = sum(w[t, j] * _dense_mlp(x[t:t + 1], _bf16_val(d["w1"][ids[t, j]]), _bf16_val(d["w2"][ids[t, j]]), I)[0] for j in range(2))
        ref = ref + sum(sw[t, s] * _dense_mlp(x[t:t + 1], _bf16_val(d["w1"][E + s]), _bf16_val(d["w2"][E + s]), I)[0] for s in range(S))
        np.testing.assert_allclose(out[t], ref, rtol=1e-9, atol=1e-12)


def test_layer_expert_relabelling_and_scale_linearity():
    rng = np.random.default_rng(15)
    E = 8
    d = _mk_layer(rng, T=7, H=128, I=64, E=E, k=3, alpha=1.702, beta=1.0, limit=7.0, w_mult=4.0,
                  gs=np.full(E, 2.0, np.float32), us=np.full(E, 0.5, np.float32))
    base = oracle.Layer(**d).moe_rows(np.arange(7))
    p = rng.permutation(E)
    relab = dict(d, logits=np.ascontiguousarray(d["logits"][:, p]), w1=d["w1"][p], w2=d["w2"][p])
    np.testing.assert_allclose(oracle.Layer(**relab).moe_rows(np.arange(7)), base, rtol=1e-12, atol=1e-14)
    # per-expert gate/up scales act on the accumulators: same as scaling the weight rows
    # (x2 and x0.5 are exact in bf16)
    I = 64
    w1s = _bf16_val(d["w1"]).copy()
    w1s[:, :I] *= 2.0
    w1s[:, I:] *= 0.5
    folded = dict(d, w1=_bf16_bits(w1s), gate_scale=None, up_scale=None)
    np.testing.assert_allclose(oracle.Layer(**folded).moe_rows(np.arange(7)), base, rtol=1e-12, atol=1e-14)
    # linear in W2 and in route_scale
    d2 = dict(d, w2=_bf16_bits(_bf16_val(d["w2"]) * 2.0), route_scale=3.0)
    np.testing.assert_allclose(oracle.Layer(**d2).moe_rows(np.arange(7)), 6.0 * base, rtol=1e-12, atol=1e-13)


def test_layer_fp8_matches_torch_e4m3_composition():
    rng = np.random.default_rng(16)
    T, H, I, E = 4, 256, 128, 2
    G = E + 1
    w1f = rng.normal(0, 0.02, (G, 2 * I, H)).astype(np.float32)
    w2f = rng.normal(0, 0.02, (G, H, I)).astype(np.float32)

    def tq(w):  # 128x128 block quantisation with torch's own E4M3 rounding
        Gn, R, C = w.shape
        blk = torch.from_numpy(w).reshape(Gn, R // 128, 128, C // 128, 128)
        s = blk.abs().amax(dim=(2, 4)) / 448.0
        q = (blk / s[:, :, None, :, None]).to(torch.float8_e4m3fn)
        return q.reshape(Gn, R, C).view(torch.uint8).numpy(), s.numpy().astype(np.float32)

    q1, s1 = tq(w1f)
    q2, s2 = tq(w2f)
    x = _bf16_bits(rng.normal(0, 1, (T, H)))
    logits = rng.normal(0, 1, (T, E)).astype(np.float32)
    L = oracle.Layer(T=T, H=H, I=I, E=E, k=1, n_sink=0, n_shared=1, wdtype=oracle.WDTYPE_FP8,
                     score=oracle.SCORE_SIGMOID, alpha=1.0, beta=0.0, limit=10.0, route_scale=1.0,
                     logits=logits, x=x, w1=q1, w2=q2, w1_scale=s1, w2_scale=s2)
    out = L.moe_rows(np.arange(T))

    def deq(q, s):
        v = torch.from_numpy(q).view(torch.float8_e4m3fn).to(torch.float64)
        return (v.reshape(q.shape[0], q.shape[1] // 128, 128, q.shape[2] // 128, 128)
                * torch.from_numpy(s).double()[:, :, None, :, None]).reshape(q.shape)

    def act_q(v):  # 1x128 activation blocks, scale amax/448 in fp32, torch's E4M3 rounding
        f = v.float().reshape(-1, 128)
        s = f.abs().amax(1, keepdim=True) / 448.0
        s = torch.where(s > 0, s, torch.ones_like(s))
        return ((f / s).to(torch.float8_e4m3fn).double() * s.double()).reshape(v.shape)

    W1, W2 = deq(q1, s1), deq(q2, s2)
    xv = act_q(torch.from_numpy(_bf16_val(x)))
    for t in range(T):
        sig = scipy.special.expit(float(logits[t].max()))
        wsel = 1.0  # k = 1: the single selected weight renormalises to 1
        assert sig > 0
        ref = torch.zeros(H, dtype=torch.float64)
        e = int(np.argmax(logits[t]))
        for ex, wt in [(e, wsel), (E, 1.0)]:
            g = torch.clamp(xv[t] @ W1[ex, :I].T, max=10.0)
            u = torch.clamp(xv[t] @ W1[ex, I:].T, -10.0, 10.0)
            h = act_q(torch.nn.functional.silu(g) * u)
            ref += wt * (h @ W2[ex].T)
        np.testing.assert_allclose(out[t], ref.numpy(), rtol=1e-9, atol=1e-12)


def test_gemm_pieces_agree_with_dense_reference():
    rng = np.random.default_rng(17)
    T, H, I, E, k = 9, 128, 64, 3, 2
    d = _mk_layer(rng, T=T, H=H, I=I, E=E, k=k)
    L = oracle.Layer(**d)
    ids, w, _ = oracle.route(d["logits"], E, k, oracle.SCORE_SOFTMAX)
    offsets, perm, inv = oracle.permute(ids, E)
    A = offsets[-1]
    xp = d["x"][perm]
    grp = np.searchsorted(offsets, np.arange(A), side="right") - 1
    h = L.gemm1_rows(A, xp, None, np.arange(A), grp)
    x = _bf16_val(d["x"])
    for r in range(A):
        e = grp[r]
        g = torch.from_numpy(x[perm[r]]) @ torch.from_numpy(_bf16_val(d["w1"][e][:I])).T
        u = torch.from_numpy(x[perm[r]]) @ torch.from_numpy(_bf16_val(d["w1"][e][I:])).T
        np.testing.assert_allclose(h[r], (torch.nn.functional.silu(g) * u).numpy(), rtol=1e-11, atol=1e-14)
    hb = _bf16_bits(h)
    row_w = np.zeros(A, np.float32)
    for t in range(T):
        for j in range(k):
            row_w[inv[t, j]] = w[t, j]
    out = L.gemm2_rows(A, hb, None, offsets, inv, row_w, np.arange(T))
    hv = _bf16_val(hb)
    for t in range(T):
        ref = sum(float(row_w[inv[t, j]]) * (torch.from_numpy(hv[inv[t, j]]) @ torch.from_numpy(_bf16_val(d["w2"][ids[t, j]])).T).numpy() for j in range(k))
        np.testing.assert_allclose(out[t], ref, rtol=1e-11, atol=1e-14)


def _dense_mlp_clamped(x, w1, w2, I, L):
    # alpha = 1, beta = 0: h = silu(min(g, L)) * clamp(u, -L, L), all torch library calls
    xt = torch.from_numpy(x)
    g = torch.clamp(xt @ torch.from_numpy(w1[:I]).T, max=L)
    u = torch.clamp(xt @ torch.from_numpy(w1[I:]).T, min=-L, max=L)
    return ((torch.nn.functional.silu(g) * u) @ torch.from_numpy(w2).T).numpy()


def test_layer_per_expert_limits_clamp_each_expert_with_its_own_value():
    # k = 1 softmax: every token goes to one expert with weight 1, so the layer output
    # is that expert's clamped MLP with that expert's limit
    rng = np.random.default_rng(31)
    E, I, T = 3, 32, 9
    limits = np.array([0.25, 0.8, np.inf], np.float32)
    d = _mk_layer(rng, T=T, H=128, I=I, E=E, k=1, w_mult=2.0)
    out = oracle.Layer(**d, limits=limits).moe_rows(np.arange(T))
    ids, _, _ = oracle.route(d["logits"], E, 1, oracle.SCORE_SOFTMAX)
    x = _bf16_val(d["x"])
    assert len(set(ids[:, 0])) == E  # every expert (and so every limit) is exercised
    for t in range(T):
        e = int(ids[t, 0])
        ref = _dense_mlp_clamped(x[t:t + 1], _bf16_val(d["w1"][e]), _bf16_val(d["w2"][e]), I, float(limits[e]))
        np.testing.assert_allclose(out[t:t + 1], ref, rtol=1e-10, atol=1e-12)
    # a uniform array is the scalar limit (0.75: the same value in fp32 and fp64)
    uni = oracle.Layer(**dict(d, limit=0.75), limits=np.full(E, 0.75, np.float32)).moe_rows(np.arange(T))
    sca = oracle.Layer(**dict(d, limit=0.75)).moe_rows(np.arange(T))
    np.testing.assert_array_equal(uni, sca)


def test_layer_router_bias_changes_only_the_selection():
    # a dominant bias routes every token to the same experts; the output then equals the
    # sigma-ratio-weighted sum of those experts' dense MLPs (raw-logit weights)
    rng = np.random.default_rng(32)
    E, I, T, k = 6, 32, 5, 2
    d = _mk_layer(rng, T=T, H=128, I=I, E=E, k=k, score=oracle.SCORE_SIGMOID)
    bias = np.array([0, 0, 50, 0, 40, 0], np.float32)
    out = oracle.Layer(**d, router_bias=bias).moe_rows(np.arange(T))
    x = _bf16_val(d["x"])
    sig = scipy.special.expit(d["logits"].astype(np.float64))
    wts = sig[:, [2, 4]] / sig[:, [2, 4]].sum(1, keepdims=True)
    ref = sum(wts[:, j:j + 1] * _dense_mlp(x, _bf16_val(d["w1"][e]), _bf16_val(d["w2"][e]), I)
              for j, e in enumerate([2, 4]))
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------------------- INT4 group-32 weights

def _torch_int4_dequant(packed, scale_bits):
    """The pages' rule with torch ops: low nibble = even K, high = odd K, (nibble - 8) * scale
    as a bf16 product (torch multiplies bf16 in fp32 and rounds to bf16 once)."""
    p = torch.from_numpy(packed.astype(np.int32))
    n = torch.stack([(p & 0xF) - 8, (p >> 4) - 8], dim=-1).reshape(p.shape[0], -1)
    s = torch.from_numpy(scale_bits.view(np.int16)).view(torch.bfloat16).repeat_interleave(32, dim=1)
    return n.to(torch.bfloat16) * s


def test_int4_dequant_follows_the_nibble_order_and_group_scale():
    rng = np.random.default_rng(41)
    packed = rng.integers(0, 256, (6, 64), dtype=np.uint8)  # K = 128: 4 groups of 32
    scales = _bf16_bits(rng.normal(0, 0.3, (6, 4)))
    packed[0, 0], packed[0, 1] = 0x2F, 0x80  # K 0..3: nibbles 15, 2, 0, 8 -> 7s, -6s, -8s, 0
    got = oracle.int4_dequant(packed, scales)
    ref = _torch_int4_dequant(packed, scales).double().numpy()
    np.testing.assert_array_equal(got, ref)
    s0 = float(_bf16_val(scales[0, 0]))
    # byte 0x2F: low nibble 15 is K 0 (+7 s), high nibble 2 is K 1 (-6 s); byte 0x80: 0 -> -8 s, 8 -> 0
    assert got[0, 2] == -8 * s0 and got[0, 3] == 0.0   # powers of two times s: exact in bf16
    np.testing.assert_allclose(got[0, :2], [7 * s0, -6 * s0], rtol=2 ** -8)


def test_layer_int4_equals_bf16_layer_with_dequantised_weights():
    # the INT4 layer must compute exactly the bf16 layer whose weights are the dequantised
    # INT4 weights (the same fp64 arithmetic on the same values)
    rng = np.random.default_rng(42)
    T, H, I, E, k, S = 6, 128, 64, 4, 2, 1
    G = E + S
    w1p = rng.integers(0, 256, (G, 2 * I, H // 2), dtype=np.uint8)
    w2p = rng.integers(0, 256, (G, H, I // 2), dtype=np.uint8)
    w1s = _bf16_bits(np.abs(rng.normal(0.01, 0.003, (G, 2 * I, H // 32))))
    w2s = _bf16_bits(np.abs(rng.normal(0.01, 0.003, (G, H, I // 32))))
    x = _bf16_bits(rng.normal(0, 1, (T, H)))
    logits = rng.normal(0, 1, (T, E)).astype(np.float32)
    common = dict(T=T, H=H, I=I, E=E, k=k, n_sink=0, n_shared=S, score=oracle.SCORE_SOFTMAX, alpha=1.702, beta=1.0,
                  limit=7.0, route_scale=1.0, logits=logits, x=x)
    q = oracle.Layer(**common, wdtype=oracle.WDTYPE_INT4, w1=w1p, w2=w2p, w1_scale=w1s, w2_scale=w2s)
    w1b = np.stack([_torch_int4_dequant(w1p[g], w1s[g]).view(torch.int16).numpy().view(np.uint16) for g in range(G)])
    w2b = np.stack([_torch_int4_dequant(w2p[g], w2s[g]).view(torch.int16).numpy().view(np.uint16) for g in range(G)])
    b = oracle.Layer(**common, wdtype=oracle.WDTYPE_BF16, w1=w1b, w2=w2b)
    np.testing.assert_array_equal(q.moe_rows(np.arange(T)), b.moe_rows(np.arange(T)))


# ------------------------------------------------------------------ NVFP4 weights
# E2M1 elements with one E4M3 scale per 16 along K (the NVFP4 checkpoints of the
# xorl-wheels FlashInfer 0.6.18 page, "Changes"); ml_dtypes implements both element
# formats independently of the oracle.

def _ml_fp4_dequant(packed, scale_codes):
    """packed uint8 [rows, K/2] (low nibble = even K), E4M3 codes [rows, K/16] -> bf16 bits
    of E2M1 * E4M3 (exact in bf16), computed with ml_dtypes and torch."""
    import ml_dtypes
    n = np.stack([packed & 0xF, packed >> 4], axis=-1).reshape(packed.shape[0], -1)
    v = n.astype(np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    s = scale_codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64).repeat(16, axis=1)
    w = torch.from_numpy(v * s).to(torch.bfloat16)
    assert torch.equal(w.double(), torch.from_numpy(v * s))  # exact: at most 6 significant bits
    return w.view(torch.int16).numpy().view(np.uint16)


def test_e2m1_decode_all_codes_match_ml_dtypes():
    import ml_dtypes
    ref = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    got = np.array([oracle.e2m1_decode(c) for c in range(16)])
    np.testing.assert_array_equal(got, ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))


def _finite_e4m3_codes(rng, shape, lo=0x20, hi=0x48):
    """positive finite E4M3 codes (no NaN pattern), exponents around 2^-4 .. 2^1"""
    return rng.integers(lo, hi, shape, dtype=np.uint8)


def test_fp4_dequant_follows_the_nibble_order_and_block_scale():
    rng = np.random.default_rng(51)
    packed = rng.integers(0, 256, (6, 64), dtype=np.uint8)  # K = 128: 8 blocks of 16
    scales = _finite_e4m3_codes(rng, (6, 8))
    packed[0, 0] = 0x2F  # K 0: low nibble 0xF = -6, K 1: high nibble 0x2 = +1
    got = oracle.fp4_dequant(packed, scales)
    ref = _bf16_val(_ml_fp4_dequant(packed, scales))
    np.testing.assert_array_equal(got, ref)
    import ml_dtypes
    s0 = float(np.array([scales[0, 0]], np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)[0])
    assert got[0, 0] == -6 * s0 and got[0, 1] == 1 * s0
    # the scale of K 16..31 is the second code of the row
    s1 = float(np.array([scales[2, 1]], np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)[0])
    b = packed[2, 8]
    assert got[2, 16] == float(np.array([b & 0xF], np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)[0]) * s1


def test_layer_nvfp4_equals_bf16_layer_with_dequantised_weights():
    # with per-expert gate/up global scales (the NVFP4 checkpoints' g1_alphas / g1_alphas_up)
    rng = np.random.default_rng(52)
    T, H, I, E, k, S = 6, 128, 64, 4, 2, 1
    G = E + S
    w1p = rng.integers(0, 256, (G, 2 * I, H // 2), dtype=np.uint8)
    w2p = rng.integers(0, 256, (G, H, I // 2), dtype=np.uint8)
    w1s = _finite_e4m3_codes(rng, (G, 2 * I, H // 16), 0x10, 0x30)
    w2s = _finite_e4m3_codes(rng, (G, H, I // 16), 0x10, 0x30)
    gs = rng.uniform(0.5, 1.3, G).astype(np.float32)
    us = rng.uniform(0.5, 1.3, G).astype(np.float32)
    x = _bf16_bits(rng.normal(0, 1, (T, H)))
    logits = rng.normal(0, 1, (T, E)).astype(np.float32)
    common = dict(T=T, H=H, I=I, E=E, k=k, n_sink=0, n_shared=S, score=oracle.SCORE_SOFTMAX, alpha=1.702, beta=1.0,
                  limit=7.0, route_scale=1.0, logits=logits, x=x, gate_scale=gs, up_scale=us)
    q = oracle.Layer(**common, wdtype=oracle.WDTYPE_NVFP4, w1=w1p, w2=w2p, w1_scale=w1s, w2_scale=w2s)
    w1b = np.stack([_ml_fp4_dequant(w1p[g], w1s[g]) for g in range(G)])
    w2b = np.stack([_ml_fp4_dequant(w2p[g], w2s[g]) for g in range(G)])
    b = oracle.Layer(**common, wdtype=oracle.WDTYPE_BF16, w1=w1b, w2=w2b)
    np.testing.assert_array_equal(q.moe_rows(np.arange(T)), b.moe_rows(np.arange(T)))
