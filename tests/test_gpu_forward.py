"""The whole layer (moe_forward, the launch configuration the bench times) on every
workload against the oracle: every token on the small workloads, sampled tokens on the
full-size prefill workloads; router ids and offsets bit-exact at full size."""
import numpy as np
import pytest
import torch

import oracle
import grouped_gemm_swiglu_b200 as moe
from grouped_gemm_swiglu_b200 import workloads as W
from helpers import assert_bf16_close, assert_fp8_close, f32, oracle_layer, sample_tokens

pytestmark = pytest.mark.gpu

FULL = ["tiny", "oai_swiglu", "decode_t1", "decode_t8", "decode_t64"]
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
    moe.moe_forward(inp["logits"][:0], inp["x"][:0], inp["w1"], None, None, None, inp["w2"], None, d, out, ws=ws)
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
