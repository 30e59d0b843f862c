"""The whole layer (moe_forward, the launch configuration the bench times) on every
workload against the oracle: every token on the small workloads, sampled tokens on the
full-size prefill workloads; router ids and offsets bit-exact at full size."""
import numpy as np
import pytest
import torch

import oracle
import grouped_gemm_swiglu_b200 as moe
from grouped_gemm_swiglu_b200 import workloads as W
from helpers import assert_bf16_close, assert_fp8_close, f32, fp8_layout, oracle_layer, pair_layout, sample_tokens

pytestmark = pytest.mark.gpu

FULL = ["tiny", "oai_swiglu", "decode_t1", "decode_t8", "decode_t64", "decode_t1_int4", "decode_t64_int4",
        "decode_t1_nvfp4", "decode_t64_nvfp4"]
SAMPLED = {"qwen3_30b_a3b": 48, "glm_fp8": 24}


def run_forward(wl, inp):
    d = moe.MoeDims.of(wl)
    layer = moe.MoELayer(d, inp["w1"], inp["w2"], inp["w1_scale"], inp["w2_scale"], inp["gate_scale"],
                         inp["up_scale"])
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    tw = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    sw = torch.empty((wl.T, wl.n_sink), dtype=torch.float32, device="cuda") if wl.n_sink else None
    out = layer.forward(inp["logits"], inp["x"], topk_ids=ids, topk_w=tw, shared_w=sw)
    torch.cuda.synchronize()
    return out, ids, tw, sw, layer


@pytest.mark.parametrize("name", FULL + list(SAMPLED))
def test_forward_matches_oracle(name):
    wl = W.WORKLOADS[name]
    inp = W.make_inputs(wl, "cuda")
    out, ids, tw, sw, layer = run_forward(wl, inp)
    assert layer.status() == 0
    o_ids, o_w, o_sw = oracle.route(f32(inp["logits"]), wl.E, wl.k, wl.score, wl.route_scale)
    assert np.array_equal(ids.cpu().numpy(), o_ids)
    assert np.abs(tw.cpu().numpy() - o_w).max() <= 1e-6
    toks = sample_tokens(wl.T, SAMPLED.get(name, wl.T), seed=1)
    ref = oracle_layer(wl, inp).moe_rows(toks)
    got = out.float().cpu().numpy()[toks]
    if wl.wdtype == W.WDTYPE_FP8:
        assert_fp8_close(got, ref, name)
    else:
        assert_bf16_close(got, ref, name)


# FP8 at a size the oracle covers token by token, with groups of about 540 rows (several
# token blocks each, ragged tails) and the GLM parameters (sigmoid routing, L = 10, one
# shared expert), in both layouts of large-group FP8 tiles
LARGE_FP8 = W.Workload("glm_fp8_t1024", T=1024, H=1024, I=512, E=16, k=8, n_shared=1, wdtype=W.WDTYPE_FP8,
                       score=W.SCORE_SIGMOID, limit=10.0)


@pytest.mark.parametrize("pair", [False, True], ids=["cta128", "cta_pair"])
def test_forward_fp8_large_groups_every_token(pair):
    wl = LARGE_FP8
    inp = W.make_inputs(wl, "cuda")
    with fp8_layout(pair):
        out, ids, tw, sw, layer = run_forward(wl, inp)
    assert layer.status() == 0
    ref = oracle_layer(wl, inp).moe_rows(np.arange(wl.T, dtype=np.int32))
    assert_fp8_close(out.float().cpu().numpy(), ref, wl.name)


# bf16 with groups of about 500 rows (256-row token blocks, ragged tails), per-expert
# gate/up scales and a shared expert, in both layouts of 256-row bf16 tiles
LARGE_BF16 = W.Workload("bf16_t1024_large_groups", T=1024, H=1024, I=512, E=16, k=8, n_shared=1,
                        score=W.SCORE_SOFTMAX, expert_scales=(0.52, 1.22))


@pytest.mark.parametrize("pair", [False, True], ids=["cta256", "cta_pair"])
def test_forward_bf16_large_groups_every_token(pair):
    wl = LARGE_BF16
    inp = W.make_inputs(wl, "cuda")
    with pair_layout(pair):
        out, ids, tw, sw, layer = run_forward(wl, inp)
    assert layer.status() == 0
    ref = oracle_layer(wl, inp).moe_rows(np.arange(wl.T, dtype=np.int32))
    assert_bf16_close(out.float().cpu().numpy(), ref, wl.name)


def test_forward_qwen3_bf16_cta_pair_sampled():
    """The full Qwen3-shaped bf16 prefill in the token-major CTA-pair layout (sampled tokens)."""
    wl = W.WORKLOADS["qwen3_30b_a3b"]
    inp = W.make_inputs(wl, "cuda")
    with pair_layout(True):
        out, ids, tw, sw, layer = run_forward(wl, inp)
    assert layer.status() == 0
    toks = sample_tokens(wl.T, 32, seed=3)
    ref = oracle_layer(wl, inp).moe_rows(toks)
    assert_bf16_close(out.float().cpu().numpy()[toks], ref, "qwen3_30b_a3b (CTA pair)")


def test_forward_glm_fp8_cta_pair_sampled():
    """The full GLM-shaped FP8 prefill in the CTA-pair layout (sampled tokens)."""
    wl = W.WORKLOADS["glm_fp8"]
    inp = W.make_inputs(wl, "cuda")
    with fp8_layout(True):
        out, ids, tw, sw, layer = run_forward(wl, inp)
    assert layer.status() == 0
    toks = sample_tokens(wl.T, 24, seed=2)
    ref = oracle_layer(wl, inp).moe_rows(toks)
    assert_fp8_close(out.float().cpu().numpy()[toks], ref, "glm_fp8 (CTA pair)")


def test_forward_is_deterministic_and_reusable():
    wl = W.WORKLOADS["oai_swiglu"]
    inp = W.make_inputs(wl, "cuda")
    out1, *_ , layer = run_forward(wl, inp)
    out2 = layer.forward(inp["logits"], inp["x"])
    out3 = layer.forward(inp["logits"][:100], inp["x"][:100])  # fewer tokens, same workspace
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)
    ref = oracle_layer(wl.with_(T=100), {**inp, "logits": inp["logits"][:100], "x": inp["x"][:100]}).moe_rows(
        np.arange(100, dtype=np.int32))
    assert_bf16_close(out3.float().cpu().numpy(), ref, "T=100")


def test_forward_empty_batch():
    wl = W.WORKLOADS["tiny"]
    inp = W.make_inputs(wl, "cuda")
    d = moe.MoeDims.of(wl, T=0)
    ws = moe.alloc_workspace(moe.MoeDims.of(wl), moe.MOE_WS_FORWARD)
    out = torch.empty((0, wl.H), dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(inp["logits"][:0], None, inp["x"][:0], inp["w1"], None, None, None, None, inp["w2"], None, d, out,
                    ws=ws)
    assert moe.moe_read_status(ws) == 0


def test_forward_skewed_routing_one_hot_expert():
    """Every token routed to the same top-k experts (the degenerate load imbalance)."""
    wl = W.WORKLOADS["oai_swiglu"].with_(T=200)
    inp = W.make_inputs(wl, "cuda")
    inp["logits"][:, :4] += 100.0
    out, ids, *_ = run_forward(wl, inp)
    assert set(np.unique(ids.cpu().numpy()).tolist()) == {0, 1, 2, 3}
    ref = oracle_layer(wl, inp).moe_rows(np.arange(200, dtype=np.int32))
    assert_bf16_close(out.float().cpu().numpy(), ref, "skewed")


@pytest.mark.parametrize("name", ["oai_swiglu", "decode_t8", "glm_fp8", "decode_t1", "decode_t1_int4",
                                  "decode_t1_nvfp4"])
def test_public_stage_calls_reproduce_forward(name):
    """moe_route_topk -> moe_permute -> moe_experts -> moe_combine gives moe_forward's
    output bit for bit (same kernels, deterministic order), and matches the oracle."""
    wl = W.WORKLOADS[name]
    if name == "glm_fp8":
        wl = wl.with_(T=512)
    inp = W.make_inputs(wl, "cuda")
    out_f, *_ = run_forward(wl, inp)
    d = moe.MoeDims.of(wl)
    fp8 = wl.wdtype == W.WDTYPE_FP8
    A, G, T = d.A, d.G, wl.T
    dev = "cuda"
    ids = torch.empty((T, wl.k), dtype=torch.int32, device=dev)
    tw = torch.empty((T, wl.k), dtype=torch.float32, device=dev)
    sw = torch.empty((T, wl.n_sink), dtype=torch.float32, device=dev) if wl.n_sink else None
    offsets = torch.empty((G + 1,), dtype=torch.int32, device=dev)
    perm = torch.empty((A,), dtype=torch.int32, device=dev)
    inv = torch.empty((T, wl.k), dtype=torch.int32, device=dev)
    xp = torch.empty((A, wl.H), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
    xs = torch.empty((wl.H // 128, A), dtype=torch.float32, device=dev) if fp8 else None
    h = torch.empty((A, wl.I), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
    hs = torch.empty((wl.I // 128, A), dtype=torch.float32, device=dev) if fp8 else None
    y = torch.empty((A, wl.H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((T, wl.H), dtype=torch.bfloat16, device=dev)
    ws_p = moe.alloc_workspace(d, moe.MOE_WS_PERMUTE)
    ws_e = moe.alloc_workspace(d, moe.MOE_WS_EXPERTS)
    ws_c = moe.alloc_workspace(d, moe.MOE_WS_COMBINE)
    for _ in range(2):  # a second pass checks that the experts workspace is left reusable
        moe.moe_route_topk(inp["logits"], d, None, ids, tw, sw)
        moe.moe_permute(ids, inp["x"], d, offsets, perm, inv, xp, xs, ws_p)
        moe.moe_experts(xp, xs, offsets, inp["w1"], inp["w1_scale"], inp["gate_scale"], inp["up_scale"], None,
                        inp["w2"], inp["w2_scale"], d, h, hs, y, ws_e)
        moe.moe_combine(y, offsets, inv, tw, sw, d, out, ws_c)
        torch.cuda.synchronize()
        for ws in (ws_p, ws_e, ws_c):
            assert moe.moe_read_status(ws) == 0
        assert torch.equal(out, out_f)
    toks = sample_tokens(T, 16, seed=2)
    ref = oracle_layer(wl, inp).moe_rows(toks)
    got = out.float().cpu().numpy()[toks]
    (assert_fp8_close if fp8 else assert_bf16_close)(got, ref, name)


def test_forward_with_router_bias_expert_limits_and_packed_output():
    """moe_forward with a correction bias on the ranking, a clamp per expert and the packed
    routing output, against the oracle given the same bias and limits (decode shape:
    sigmoid scoring with sinks gating the shared experts)."""
    from oracle.torch_io import host_inputs, oracle_layer_from_inputs
    wl = W.WORKLOADS["decode_t64"]
    inp = W.make_inputs(wl, "cuda")
    g = torch.Generator(device="cuda").manual_seed(11)
    bias = torch.randn((wl.E,), generator=g, device="cuda") * 0.05
    limits = 0.5 + 2 * torch.rand((wl.E + wl.n_shared,), generator=g, device="cuda")  # pre-activation std ~1.3
    d = moe.MoeDims.of(wl)
    layer = moe.MoELayer(d, inp["w1"], inp["w2"], limits=limits, router_bias=bias)
    T = wl.T
    ids = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
    sw = torch.empty((T, wl.n_sink), dtype=torch.float32, device="cuda")
    packed = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
    out = layer.forward(inp["logits"], inp["x"], topk_ids=ids, topk_w=tw, shared_w=sw, packed=packed)
    torch.cuda.synchronize()
    assert layer.status() == 0
    o_ids, o_w, o_sw = oracle.route(f32(inp["logits"]), wl.E, wl.k, wl.score, wl.route_scale, bias=f32(bias))
    assert np.array_equal(ids.cpu().numpy(), o_ids)
    assert np.abs(tw.cpu().numpy() - o_w).max() <= 1e-6 and np.abs(sw.cpu().numpy() - o_sw).max() <= 1e-6
    pk = packed.cpu().numpy().view(np.uint32)
    wb = tw.cpu().to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).astype(np.uint32)
    assert np.array_equal(pk >> 16, o_ids.astype(np.uint32)) and np.array_equal(pk & 0xFFFF, wb)
    host = host_inputs(inp)
    host["router_bias"], host["limits"] = f32(bias), f32(limits)
    ref = oracle_layer_from_inputs(wl, host).moe_rows(np.arange(T, dtype=np.int32))
    assert_bf16_close(out.float().cpu().numpy(), ref, "bias + limits")
    # the limits bite: without them the output differs by more than the tolerance
    host0 = host_inputs(inp)
    host0["router_bias"] = f32(bias)
    ref0 = oracle_layer_from_inputs(wl, host0).moe_rows(np.arange(8, dtype=np.int32))
    assert np.abs(ref0 - ref[:8]).max() > 0.05 * np.abs(ref[:8]).max()
