"""Expert parallelism on one GPU: the two index kernels checked exactly, and the whole
expert-parallel layer with R = 2 and 4 ranks run as threads of this process
(LocalExchange: the ranks meet on the host and copy their rows between buffers; no
kernel waits for another rank). Each rank holds only its routed experts and the shared
ones, serves its own slice of the tokens, and its output must match the oracle's rows
for those tokens within the layer's tolerance."""
import threading

import numpy as np
import pytest
import torch

import grouped_gemm_swiglu_b200 as moe
from grouped_gemm_swiglu_b200 import ep
from grouped_gemm_swiglu_b200 import workloads as W
from helpers import assert_bf16_close, assert_fp8_close, oracle_layer

pytestmark = pytest.mark.gpu

MOE_ERR_EXPERT_ID = -5


def test_row_ids_follow_the_offsets():
    wl = W.Workload("rows", T=53, H=256, I=128, E=16, k=4, n_sink=2, n_shared=2, score=W.SCORE_SIGMOID)
    inp = W.make_inputs(wl, "cuda")
    d = moe.MoeDims.of(wl)
    ids = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    tw = torch.empty((wl.T, wl.k), dtype=torch.float32, device="cuda")
    sw = torch.empty((wl.T, wl.n_sink), dtype=torch.float32, device="cuda")
    moe.moe_route_topk(inp["logits"], d, None, ids, tw, sw)
    offsets = torch.empty((d.G + 1,), dtype=torch.int32, device="cuda")
    perm = torch.empty((d.A,), dtype=torch.int32, device="cuda")
    inv = torch.empty((wl.T, wl.k), dtype=torch.int32, device="cuda")
    xp = torch.empty((d.A, wl.H), dtype=torch.bfloat16, device="cuda")
    ws = moe.alloc_workspace(d, moe.MOE_WS_PERMUTE)
    moe.moe_permute(ids, inp["x"], d, offsets, perm, inv, xp, None, ws)
    row_ids = torch.full((d.A,), -7, dtype=torch.int32, device="cuda")
    moe.moe_ep_row_ids(offsets, d, row_ids)
    o = offsets.cpu().numpy()
    want = np.repeat(np.arange(d.G, dtype=np.int32), np.diff(o))
    assert np.array_equal(row_ids.cpu().numpy(), want)
    # the routed rows' ids are the experts the router chose for their tokens
    got_routed = row_ids[:o[wl.E]].cpu().numpy()
    chosen = ids.cpu().numpy()
    tok = perm[:o[wl.E]].cpu().numpy()
    assert all(e in chosen[t] for e, t in zip(got_routed, tok))


def test_rebase_maps_local_shared_and_foreign_ids():
    E, S, off, n_local = 16, 2, 8, 4  # this rank: experts 8..11
    g = np.array([8, 9, 11, 12, 7, 0, 15, 16, 17, 18, -1, 1 << 20, 10, -(1 << 20)], dtype=np.int32)
    want = np.array([0, 1, 3, -1, -1, -1, -1, 4, 5, -1, -1, -1, 2, -1], dtype=np.int32)
    ids = torch.from_numpy(g).cuda()
    out = torch.full_like(ids, 99)
    moe.moe_ep_rebase(ids, ids.numel(), E, S, off, n_local, out)
    assert np.array_equal(out.cpu().numpy(), want)
    moe.moe_ep_rebase(ids, ids.numel(), E, S, off, n_local, ids)  # in place
    assert np.array_equal(ids.cpu().numpy(), want)


def test_a_foreign_id_is_reported_by_the_local_permutation():
    E, S, off, n_local, H = 8, 0, 4, 4, 256
    g = torch.tensor([4, 5, 1, 7, 6], dtype=torch.int32, device="cuda")  # expert 1 is rank 0's
    loc = torch.empty((5, 1), dtype=torch.int32, device="cuda")
    moe.moe_ep_rebase(g, 5, E, S, off, n_local, loc)
    d = moe.MoeDims()
    d.T, d.H, d.I, d.E, d.k, d.n_sink, d.n_shared = 5, H, 128, n_local, 1, 0, 0
    d.wdtype, d.score, d.alpha, d.beta, d.limit, d.route_scale = 0, 0, 1.0, 0.0, float("inf"), 1.0
    x = torch.randn((5, H), device="cuda").to(torch.bfloat16)
    offsets = torch.empty((n_local + 1,), dtype=torch.int32, device="cuda")
    perm = torch.empty((5,), dtype=torch.int32, device="cuda")
    inv = torch.empty((5, 1), dtype=torch.int32, device="cuda")
    xp = torch.empty((5, H), dtype=torch.bfloat16, device="cuda")
    ws = moe.alloc_workspace(d, moe.MOE_WS_PERMUTE)
    moe.moe_permute(loc, x, d, offsets, perm, inv, xp, None, ws)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws) == MOE_ERR_EXPERT_ID
    assert offsets[-1].item() == 4  # the foreign row is dropped


CASES = [  # (workload, ranks)
    (W.Workload("ep_bf16_sinks", T=45, H=512, I=256, E=16, k=4, n_sink=2, n_shared=2, score=W.SCORE_SIGMOID), 2),
    (W.Workload("ep_bf16_sinks", T=45, H=512, I=256, E=16, k=4, n_sink=2, n_shared=2, score=W.SCORE_SIGMOID), 4),
    (W.Workload("ep_oai_params", T=64, H=512, I=256, E=16, k=4, score=W.SCORE_SOFTMAX, alpha=1.702, beta=1.0,
                limit=7.0, gate_up_mult=4.0), 4),
    (W.Workload("ep_fp8", T=37, H=512, I=256, E=8, k=2, n_shared=1, wdtype=W.WDTYPE_FP8, score=W.SCORE_SIGMOID,
                limit=10.0), 2),
    (W.Workload("ep_int4", T=29, H=512, I=256, E=8, k=2, n_sink=2, n_shared=2, wdtype=W.WDTYPE_INT4,
                score=W.SCORE_SIGMOID), 2),
    (W.Workload("ep_nvfp4", T=40, H=512, I=256, E=8, k=2, n_shared=1, wdtype=W.WDTYPE_NVFP4,
                score=W.SCORE_SIGMOID, expert_scales=(0.52, 1.22)), 4),
    (W.WORKLOADS["oai_swiglu"], 4),
]


@pytest.mark.parametrize("wl,world", CASES, ids=[f"{w.name}-r{r}" for w, r in CASES])
def test_expert_parallel_layer_matches_the_oracle(wl, world):
    inp = W.make_inputs(wl, "cuda")
    d = moe.MoeDims.of(wl)
    E, S = wl.E, wl.n_shared
    # uneven token slices, one of them empty when there are four ranks
    cuts = np.linspace(0, wl.T, world + 1).astype(int)
    if world == 4:
        cuts[2] = cuts[1]
    hub = ep.LocalExchange(world)
    outs, errs, status = [None] * world, [], [None] * world

    def run(r):
        try:
            sh = lambda t: ep.shard(t, r, world, E, S)  # noqa: E731
            layer = ep.ExpertParallelMoE(d, r, world, sh(inp["w1"]), sh(inp["w2"]), sh(inp["w1_scale"]),
                                         sh(inp["w2_scale"]), sh(inp["gate_scale"]), sh(inp["up_scale"]),
                                         exchange=hub.for_rank(r))
            a, b = cuts[r], cuts[r + 1]
            outs[r] = layer.forward(inp["logits"][a:b].contiguous(), inp["x"][a:b].contiguous())
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
    got = torch.cat(outs).float().cpu().numpy()
    ref = oracle_layer(wl, inp).moe_rows(np.arange(wl.T, dtype=np.int32))
    (assert_fp8_close if wl.wdtype == W.WDTYPE_FP8 else assert_bf16_close)(got, ref, f"{wl.name} on {world} ranks")
