"""Failure detection on the GPU without a fault: a wait that can never complete runs out,
the kernel records MOE_ERR_TIMEOUT in the workspace's status word and returns, and the
context stays usable.

The planted failure is a flag that nothing sets: the experts workspace's per-block GEMM1
completion counters (the first words after the 256-byte header) start a million below
zero, so the GEMM1 tiles' release-adds never bring them to the count the GEMM2 tiles wait
for. Each GEMM2 tile's bounded wait (about a second) gives up, its CTA drains its copies
and MMAs, frees tensor memory and leaves. No trap, no invalid address: the same workspace
then runs the layer normally. Three kernel layouts: the single-CTA bf16 tile, and the FP8
and bf16 CTA pairs (two CTAs of a cluster sharing each MMA), whose CTAs also wait on each
other."""
import time

import numpy as np
import pytest
import torch

import grouped_gemm_swiglu_b200 as moe
from grouped_gemm_swiglu_b200 import workloads as W
from helpers import assert_bf16_close, assert_fp8_close, oracle_layer, pair_layout

pytestmark = pytest.mark.gpu

HEADER = 256        # workspace header bytes (status word and counters)
MOE_ERR_TIMEOUT = -6

CASES = [
    W.WORKLOADS["tiny"],
    # about 180 rows per group: FP8 in the CTA-pair layout (256-row token blocks; the
    # test selects it with moe_set_option)
    W.Workload("fp8_pair", T=300, H=512, I=256, E=4, k=2, n_shared=1, wdtype=W.WDTYPE_FP8,
               score=W.SCORE_SIGMOID, limit=10.0),
    # the same groups in bf16: the token-major bf16 CTA pair
    W.Workload("bf16_pair", T=300, H=512, I=256, E=4, k=2, n_shared=1, score=W.SCORE_SIGMOID),
]


@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_a_wait_that_never_completes_reports_timeout_and_the_context_survives(wl):
    with pair_layout(pair=wl.name.endswith("_pair")):  # the *_pair cases in the CTA-pair layouts
        _check_timeout(wl)


def _check_timeout(wl):
    inp = W.make_inputs(wl, "cuda")
    d = moe.MoeDims.of(wl)
    fp8 = wl.wdtype == W.WDTYPE_FP8
    T, k, A, G, H, I = wl.T, wl.k, d.A, d.G, wl.H, wl.I
    dev = "cuda"
    adt = torch.uint8 if fp8 else torch.bfloat16
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    tw = torch.empty((T, k), dtype=torch.float32, device=dev)
    offsets = torch.empty((G + 1,), dtype=torch.int32, device=dev)
    perm = torch.empty((A,), dtype=torch.int32, device=dev)
    inv = torch.empty((T, k), dtype=torch.int32, device=dev)
    xp = torch.empty((A, H), dtype=adt, device=dev)
    xs = torch.empty((H // 128, A), dtype=torch.float32, device=dev) if fp8 else None
    h = torch.empty((A, I), dtype=adt, device=dev)
    hs = torch.empty((I // 128, A), dtype=torch.float32, device=dev) if fp8 else None
    y = torch.empty((A, H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    ws_p = moe.alloc_workspace(d, moe.MOE_WS_PERMUTE)
    ws_e = moe.alloc_workspace(d, moe.MOE_WS_EXPERTS)
    ws_c = moe.alloc_workspace(d, moe.MOE_WS_COMBINE)
    moe.moe_route_topk(inp["logits"], d, None, ids, tw)
    moe.moe_permute(ids, inp["x"], d, offsets, perm, inv, xp, xs, ws_p)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws_p) == 0

    nblk_max = min(A, G) + A // 16 + 1  # block counters the workspace holds for these sizes
    counters = ws_e[HEADER:HEADER + 4 * nblk_max].view(torch.int32)
    counters.fill_(-1_000_000)
    args = (inp["w1"], inp["w1_scale"], inp["gate_scale"], inp["up_scale"], None, inp["w2"], inp["w2_scale"])
    t0 = time.perf_counter()
    moe.moe_experts(xp, xs, offsets, *args, d, h, hs, y, ws_e)  # the launch itself succeeds
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert moe.moe_read_status(ws_e) == MOE_ERR_TIMEOUT
    assert waited < 60.0

    # the context and the workspace are usable again (the test undoes its own planting:
    # counters past the launch's token blocks are not the kernel's to reset)
    counters.zero_()
    moe.moe_clear_status(ws_e)
    moe.moe_experts(xp, xs, offsets, *args, d, h, hs, y, ws_e)
    moe.moe_combine(y, offsets, inv, tw, None, d, out, ws_c)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws_e) == 0 and moe.moe_read_status(ws_c) == 0
    ref = oracle_layer(wl, inp).moe_rows(np.arange(T, dtype=np.int32))
    got = out.float().cpu().numpy()
    if fp8:
        assert_fp8_close(got, ref, "after a timed-out launch")
    else:
        assert_bf16_close(got, ref, "after a timed-out launch")
