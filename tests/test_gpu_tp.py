"""Tensor parallelism over I on one GPU: R = 2 and 4 ranks as threads of this process
(LocalExchange; the ranks meet on the host for the all-reduce, no kernel waits for
another rank). Each rank runs moe_forward on every token with its slice of every expert;
after the all-reduce every rank holds the same output, which must match the oracle's
one-rank layer within the layer's tolerance."""
import threading

import numpy as np
import pytest
import torch

import grouped_gemm_swiglu_b200 as moe
from grouped_gemm_swiglu_b200 import ep, tp
from grouped_gemm_swiglu_b200 import workloads as W
from helpers import assert_bf16_close, assert_fp8_close, oracle_layer

pytestmark = pytest.mark.gpu

CASES = [
    (W.Workload("tp_bf16_sinks", T=37, H=512, I=512, E=16, k=4, n_sink=2, n_shared=2, score=W.SCORE_SIGMOID), 4),
    (W.Workload("tp_oai_params", T=64, H=512, I=256, E=16, k=4, score=W.SCORE_SOFTMAX, alpha=1.702, beta=1.0,
                limit=7.0, gate_up_mult=4.0, expert_scales=(0.52, 1.22)), 2),
    (W.Workload("tp_fp8", T=37, H=512, I=256, E=8, k=2, n_shared=1, wdtype=W.WDTYPE_FP8, score=W.SCORE_SIGMOID,
                limit=10.0), 2),
    (W.Workload("tp_int4", T=29, H=512, I=512, E=8, k=2, n_sink=2, n_shared=2, wdtype=W.WDTYPE_INT4,
                score=W.SCORE_SIGMOID), 4),
    (W.Workload("tp_nvfp4", T=40, H=512, I=256, E=8, k=2, n_shared=1, wdtype=W.WDTYPE_NVFP4,
                score=W.SCORE_SIGMOID, expert_scales=(0.52, 1.22)), 2),
]


@pytest.mark.parametrize("wl,world", CASES, ids=[f"{w.name}-r{r}" for w, r in CASES])
def test_tensor_parallel_layer_matches_the_oracle(wl, world):
    inp = W.make_inputs(wl, "cuda")
    d = moe.MoeDims.of(wl)
    hub = ep.LocalExchange(world)
    outs, errs, status = [None] * world, [], [None] * world

    def run(r):
        try:
            layer = tp.TensorParallelMoE(d, r, world, tp.shard_w1(inp["w1"], r, world),
                                         tp.shard_w2(inp["w2"], r, world), tp.shard_w1(inp["w1_scale"], r, world),
                                         tp.shard_w2(inp["w2_scale"], r, world), inp["gate_scale"], inp["up_scale"],
                                         exchange=hub.for_rank(r))
            outs[r] = layer.forward(inp["logits"], inp["x"])
            torch.cuda.synchronize()
            status[r] = layer.status()
        except Exception as e:  # noqa: BLE001 (reported below)
            errs.append(e)
            hub._barrier.abort()

    ts = [threading.Thread(target=run, args=(r,)) for r in range(world)]
    for t in ts:
        t.start()
    for t in ts:
        t.join(timeout=300)
    assert not errs, errs
    assert status == [0] * world
    for r in range(1, world):
        assert torch.equal(outs[r], outs[0])
    ref = oracle_layer(wl, inp).moe_rows(np.arange(wl.T, dtype=np.int32))
    (assert_fp8_close if wl.wdtype == W.WDTYPE_FP8 else assert_bf16_close)(outs[0].float().cpu().numpy(), ref,
                                                                          f"{wl.name} on {world} ranks")
