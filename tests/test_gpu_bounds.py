"""Out-of-bounds writes (the stand-in for a memory sanitizer): every output buffer of
moe_forward and of the stage calls, and each workspace, sits inside a larger allocation
whose head and tail hold a canary byte pattern. After the calls every canary is intact and
the results match the oracle. Tiny and odd shapes: one expert with k = 1, one token with
sinks and shared experts, T = 3 and T = 37 with ragged groups, FP8 (all three tile layouts:
narrow, token-major, CTA pair) and INT4 weights."""
import math

import numpy as np
import pytest
import torch

import grouped_gemm_swiglu_b200 as moe
from grouped_gemm_swiglu_b200 import workloads as W
from helpers import assert_bf16_close, assert_fp8_close, oracle_layer, pair_layout

pytestmark = pytest.mark.gpu

GUARD = 4096      # canary bytes on each side (a multiple of 256 keeps every view aligned)
CANARY = 0xA5

SHAPES = [
    W.Workload("one_expert_k1", T=37, H=256, I=128, E=1, k=1, score=W.SCORE_SOFTMAX),
    W.Workload("t1_sinks_shared", T=1, H=512, I=256, E=16, k=4, n_sink=2, n_shared=2, score=W.SCORE_SIGMOID),
    W.Workload("t3_ragged", T=3, H=384, I=128, E=8, k=2, score=W.SCORE_SIGMOID, alpha=1.702, beta=1.0, limit=7.0),
    W.Workload("t37_oai_params", T=37, H=512, I=256, E=16, k=4, score=W.SCORE_SOFTMAX, alpha=1.702, beta=1.0,
               limit=7.0, gate_up_mult=4.0),
    W.Workload("t37_fp8_shared", T=37, H=512, I=256, E=8, k=2, n_shared=1, wdtype=W.WDTYPE_FP8,
               score=W.SCORE_SIGMOID, limit=10.0),
    W.Workload("t3_int4", T=3, H=512, I=256, E=8, k=2, n_sink=2, n_shared=2, wdtype=W.WDTYPE_INT4,
               score=W.SCORE_SIGMOID),
    W.Workload("t37_nvfp4_scales", T=37, H=512, I=256, E=8, k=2, n_shared=1, wdtype=W.WDTYPE_NVFP4,
               score=W.SCORE_SIGMOID, expert_scales=(0.52, 1.22)),
    # about 100 rows per group: the token-major 128-token FP8 tile, with ragged tails
    W.Workload("t300_fp8_wide", T=300, H=512, I=384, E=8, k=2, n_shared=1, wdtype=W.WDTYPE_FP8,
               score=W.SCORE_SIGMOID, limit=10.0),
    # about 180 rows per group: the FP8 CTA pair (256-row blocks, 128 rows per CTA); the
    # shared group's second block has 44 rows, so one CTA of that pair holds none
    W.Workload("t300_fp8_pair", T=300, H=512, I=384, E=4, k=2, n_shared=1, wdtype=W.WDTYPE_FP8,
               score=W.SCORE_SIGMOID, limit=10.0),
    # the same groups in bf16 (256-row token blocks): the token-major bf16 CTA pair, with
    # the OAI SwiGLU parameters
    W.Workload("t300_bf16_pair", T=300, H=512, I=384, E=4, k=2, n_shared=1, score=W.SCORE_SOFTMAX,
               alpha=1.702, beta=1.0, limit=7.0),
]


class Guarded:
    """A tensor view with canary bands before and after it."""

    def __init__(self, shape, dtype):
        n = math.prod(shape) * torch.empty((), dtype=dtype).element_size()
        self.n = n
        self.raw = torch.full((2 * GUARD + ((n + 255) // 256) * 256,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(shape) if n else torch.empty(shape, dtype=dtype,
                                                                                          device="cuda")

    def intact(self) -> bool:
        r = self.raw.cpu().numpy()
        return bool(np.all(r[:GUARD] == CANARY) and np.all(r[GUARD + self.n:] == CANARY))


def guarded_ws(d, kind):
    n = moe.moe_workspace_size(d, kind)
    g = Guarded((n,), torch.uint8)
    g.t.zero_()
    return g


@pytest.mark.parametrize("wl", SHAPES, ids=[w.name for w in SHAPES])
def test_outputs_stay_in_bounds_and_match_the_oracle(wl):
    with pair_layout(pair=wl.name.endswith("_pair")):  # the *_pair shapes in the CTA-pair layouts
        _check_bounds(wl)


def _check_bounds(wl):
    inp = W.make_inputs(wl, "cuda")
    d = moe.MoeDims.of(wl)
    T, k, S, A, G, H, I = wl.T, wl.k, wl.n_sink, d.A, d.G, wl.H, wl.I
    fp8 = wl.wdtype == W.WDTYPE_FP8
    act = torch.uint8 if fp8 else torch.bfloat16

    # the whole layer
    out = Guarded((T, H), torch.bfloat16)
    ids = Guarded((T, k), torch.int32)
    tw = Guarded((T, k), torch.float32)
    sw = Guarded((T, S), torch.float32) if S else None
    packed = Guarded((T, k), torch.int32)
    ws_f = guarded_ws(d, moe.MOE_WS_FORWARD)
    args = (inp["w1"], inp["w1_scale"], inp["gate_scale"], inp["up_scale"], None, inp["w2"], inp["w2_scale"])
    moe.moe_forward(inp["logits"], None, inp["x"], *args, d, out.t, ids.t, tw.t, sw.t if sw else None, packed.t,
                    ws_f.t)
    torch.cuda.synchronize()
    assert moe.moe_read_status(ws_f.t) == 0
    ref = oracle_layer(wl, inp).moe_rows(np.arange(T, dtype=np.int32))
    (assert_fp8_close if fp8 else assert_bf16_close)(out.t.float().cpu().numpy(), ref, wl.name)

    # the stage calls, every output guarded
    offsets = Guarded((G + 1,), torch.int32)
    perm = Guarded((A,), torch.int32)
    inv = Guarded((T, k), torch.int32)
    xp = Guarded((A, H), act)
    xs = Guarded((H // 128, A), torch.float32) if fp8 else None
    h = Guarded((A, I), act)
    hs = Guarded((I // 128, A), torch.float32) if fp8 else None
    y = Guarded((A, H), torch.bfloat16)
    out2 = Guarded((T, H), torch.bfloat16)
    ws_p = guarded_ws(d, moe.MOE_WS_PERMUTE)
    ws_e = guarded_ws(d, moe.MOE_WS_EXPERTS)
    ws_c = guarded_ws(d, moe.MOE_WS_COMBINE)
    moe.moe_permute(ids.t, inp["x"], d, offsets.t, perm.t, inv.t, xp.t, xs.t if xs else None, ws_p.t)
    moe.moe_experts(xp.t, xs.t if xs else None, offsets.t, *args, d, h.t, hs.t if hs else None, y.t, ws_e.t)
    moe.moe_combine(y.t, offsets.t, inv.t, tw.t, sw.t if sw else None, d, out2.t, ws_c.t)
    torch.cuda.synchronize()
    for ws in (ws_p, ws_e, ws_c):
        assert moe.moe_read_status(ws.t) == 0
    assert torch.equal(out2.t, out.t)  # same kernels, same order: the same bits

    named = dict(out=out, ids=ids, tw=tw, sw=sw, packed=packed, ws_forward=ws_f, offsets=offsets, perm=perm,
                 inv=inv, x_perm=xp, x_scale=xs, h=h, h_scale=hs, y=y, out_staged=out2, ws_permute=ws_p,
                 ws_experts=ws_e, ws_combine=ws_c)
    broken = [name for name, g in named.items() if g is not None and not g.intact()]
    assert not broken, f"{wl.name}: writes outside {broken}"
