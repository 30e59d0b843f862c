"""Grouped GEMM1 (+ SwiGLU epilogue) and GEMM2 (+ weighted combine) on the GPU against
the oracle, on synthetic permuted inputs that span several tiles, every token-tile width
(16/32/64/128/256 rows, and the FP8 and bf16 two-CTA 256-row pairs), ragged group tails,
empty groups and shared groups."""
import math

import numpy as np
import pytest
import torch

import oracle
import grouped_gemm_swiglu_b200 as moe
from grouped_gemm_swiglu_b200 import workloads as W
from helpers import assert_bf16_close, assert_fp8_close, bits16, e4m3_to_np, f32, fp8_layout, pair_layout, u8

pytestmark = pytest.mark.gpu


def make_case(T, E, k, S, H, I, fp8, seed, gate_up_mult=1.0, scales=False, sinks=False, skew=0.0, limits=False,
              int4=False, fp4=False):
    ids = W.random_topk_ids(T, E, k, seed=seed, skew=skew)
    offsets, perm, inv = oracle.permute(ids.numpy(), E, S)
    A = T * (k + S)
    G = E + S
    g = torch.Generator(device="cuda").manual_seed(seed)
    w1f = torch.randn((G, 2 * I, H), generator=g, device="cuda") * 0.02 * gate_up_mult
    w2f = torch.randn((G, H, I), generator=g, device="cuda") * 0.02
    xf = torch.randn((A, H), generator=g, device="cuda")
    hf = torch.randn((A, I), generator=g, device="cuda")
    c = dict(T=T, E=E, k=k, S=S, H=H, I=I, A=A, G=G, fp8=fp8, int4=int4, fp4=fp4, ids=ids, offsets=offsets,
             perm=perm, inv=inv)
    if int4 or fp4:  # INT4 group-32 or NVFP4 weights, bf16 activations
        make = W.random_nvfp4_weights if fp4 else W.random_int4_weights
        c["w1"], c["w1_scale"] = make(g, (G, 2 * I, H), "cuda", 0.02 * gate_up_mult)
        c["w2"], c["w2_scale"] = make(g, (G, H, I), "cuda", 0.02)
        c["xs"] = c["hs"] = None
        c["xp"], c["hp"] = xf.to(torch.bfloat16), hf.to(torch.bfloat16)
    elif fp8:
        c["w1"], c["w1_scale"] = W.fp8_block_quantize_weights(w1f)
        c["w2"], c["w2_scale"] = W.fp8_block_quantize_weights(w2f)
        q, s = oracle.quant_1x128(xf.cpu().numpy())
        c["xp"], c["xs"] = torch.from_numpy(q).cuda(), torch.from_numpy(np.ascontiguousarray(s.T)).cuda()
        q, s = oracle.quant_1x128(hf.cpu().numpy())
        c["hp"], c["hs"] = torch.from_numpy(q).cuda(), torch.from_numpy(np.ascontiguousarray(s.T)).cuda()
    else:
        c["w1"], c["w2"] = w1f.to(torch.bfloat16), w2f.to(torch.bfloat16)
        c["w1_scale"] = c["w2_scale"] = c["xs"] = c["hs"] = None
        c["xp"], c["hp"] = xf.to(torch.bfloat16), hf.to(torch.bfloat16)
    c["gate_scale"] = (0.52 + 0.7 * torch.rand((G,), generator=g, device="cuda")) if scales else None
    c["up_scale"] = (0.52 + 0.7 * torch.rand((G,), generator=g, device="cuda")) if scales else None
    # a clamp per expert: small enough to bite on the pre-activations (std ~0.45), one group unclamped
    c["limits"] = None
    if limits:
        lim = 0.2 + 0.8 * torch.rand((G,), generator=g, device="cuda")
        lim[G // 2] = float("inf")
        c["limits"] = lim
    c["topk_w"] = torch.rand((T, k), generator=g, device="cuda")
    c["shared_w"] = torch.rand((T, S), generator=g, device="cuda") if (sinks and S) else None
    return c


def dims_of(c, alpha=1.0, beta=0.0, limit=math.inf):
    return moe.MoeDims(T=c["T"], H=c["H"], I=c["I"], E=c["E"], k=c["k"], n_sink=c["S"] if c["shared_w"] is not None else 0,
                       n_shared=c["S"], wdtype=3 if c.get("fp4") else (2 if c.get("int4") else (1 if c["fp8"] else 0)),
                       score=1, alpha=alpha,
                       beta=beta,
                       limit=limit, route_scale=1.0)


def oracle_of(c, d):
    fp8 = c["fp8"]
    if c.get("int4") or c.get("fp4"):
        scl = u8 if c.get("fp4") else bits16  # NVFP4: E4M3 scale codes; INT4: bf16 scale bits
        return oracle.Layer(T=c["T"], H=c["H"], I=c["I"], E=c["E"], k=c["k"], n_sink=d.n_sink, n_shared=c["S"],
                            wdtype=oracle.WDTYPE_NVFP4 if c.get("fp4") else oracle.WDTYPE_INT4, score=1,
                            alpha=d.alpha, beta=d.beta, limit=d.limit,
                            route_scale=1.0, logits=np.zeros((c["T"], c["E"] + d.n_sink), np.float32),
                            x=np.zeros((c["T"], c["H"]), np.uint16), w1=u8(c["w1"]), w2=u8(c["w2"]),
                            w1_scale=scl(c["w1_scale"]), w2_scale=scl(c["w2_scale"]),
                            gate_scale=f32(c["gate_scale"]), up_scale=f32(c["up_scale"]), limits=f32(c.get("limits")))
    return oracle.Layer(T=c["T"], H=c["H"], I=c["I"], E=c["E"], k=c["k"], n_sink=d.n_sink, n_shared=c["S"],
                        wdtype=1 if fp8 else 0, score=1, alpha=d.alpha, beta=d.beta, limit=d.limit,
                        route_scale=1.0, logits=np.zeros((c["T"], c["E"] + d.n_sink), np.float32),
                        x=np.zeros((c["T"], c["H"]), np.uint16),
                        w1=u8(c["w1"]) if fp8 else bits16(c["w1"]), w2=u8(c["w2"]) if fp8 else bits16(c["w2"]),
                        w1_scale=f32(c["w1_scale"]), w2_scale=f32(c["w2_scale"]),
                        gate_scale=f32(c["gate_scale"]), up_scale=f32(c["up_scale"]), limits=f32(c.get("limits")))


GEMM1_CASES = [
    # T, E, k, S, H, I, fp8, extra
    (8, 64, 4, 0, 256, 256, False, {}),                         # token tile 16, most groups empty
    (64, 16, 4, 0, 512, 256, False, {}),                        # tile 32
    (128, 8, 2, 0, 512, 384, False, {"scales": True}),          # tile 64, per-group gate/up scales
    (512, 8, 2, 0, 512, 256, False, {"skew": 3.0}),             # tile 128, several blocks, ragged tails
    (300, 16, 4, 1, 512, 256, False, {}),                       # a shared group of T rows
    (1024, 8, 2, 0, 512, 256, False, {"skew": 2.0}),            # tile 256, several blocks, ragged tails
    (600, 4, 2, 1, 512, 384, False, {"scales": True}),          # tile 256, shared group of 600 rows
    (96, 32, 4, 0, 2048, 768, False, {"oai": True}),            # OAI-SwiGLU shape and parameters
    (512, 8, 2, 0, 512, 256, True, {}),                         # FP8, tile 128 (register split)
    (256, 8, 2, 0, 512, 256, True, {}),                         # FP8, tile 64
    (1024, 8, 2, 1, 512, 384, True, {"skew": 2.0, "scales": True, "limits": True}),  # FP8 tile 128, ragged, shared
    (40, 32, 4, 1, 512, 256, True, {"glm": True}),              # FP8, tile 16, shared group, L = 10
    (200, 8, 2, 0, 1024, 512, True, {"oai": True, "scales": True}),
    # FP8 with groups above 128 rows on average (both layouts: 128-token tiles, and the
    # CTA pair's 256-row token blocks, 128 per CTA); heavy skew leaves some groups under
    # 128 rows (the pair's odd CTA holds none of them) and some over 256 (several
    # blocks); a shared group of T rows
    (1500, 16, 2, 1, 512, 256, True, {"skew": 4.0, "oai": True}),
    (700, 4, 2, 0, 1024, 384, True, {"scales": True, "limits": True}),
    # bf16 with groups above 128 rows on average (256-row token blocks: one CTA, or the
    # token-major CTA pair), heavy skew, a shared group of T rows, OAI parameters
    (1500, 16, 2, 1, 512, 256, False, {"skew": 4.0, "oai": True}),
    (700, 4, 2, 0, 1024, 384, False, {"scales": True, "limits": True}),
    (128, 8, 2, 1, 512, 384, False, {"limits": True}),          # a clamp per expert (shared group too)
    (300, 16, 4, 0, 512, 256, True, {"limits": True, "scales": True}),  # FP8, tile 32, clamp per expert
    (8, 64, 4, 0, 256, 256, False, {"int4": True}),            # INT4 group-32 weights: tile 16, split-K
    (64, 16, 4, 0, 512, 256, False, {"int4": True}),           # INT4, tile 32
    (300, 16, 4, 1, 512, 384, False, {"int4": True, "oai": True, "scales": True}),  # INT4, shared group
    (512, 8, 2, 0, 512, 256, False, {"int4": True, "skew": 3.0, "limits": True}),   # INT4, tile 128
    # NVFP4 weights (E2M1, E4M3 scale per 16 K), per-group global scales on gate and up
    (8, 64, 4, 0, 256, 256, False, {"fp4": True}),                           # tile 16, split-K
    (64, 16, 4, 0, 512, 256, False, {"fp4": True, "scales": True}),          # tile 32, global scales
    (300, 16, 4, 1, 512, 384, False, {"fp4": True, "oai": True, "scales": True}),  # shared group, OAI params
    (512, 8, 2, 0, 512, 256, False, {"fp4": True, "skew": 3.0, "limits": True}),   # tile 64, ragged, clamps
    # decode-sized batches (at most 16 routed rows): one-row groups, split-K of GEMM1
    (2, 64, 4, 1, 512, 256, False, {}),                         # 10 rows, a shared group of 2
    (1, 32, 4, 0, 512, 384, False, {"scales": True, "limits": True}),  # one token, scales, clamp per expert
    (8, 2, 2, 0, 512, 256, False, {"oai": True}),               # 2 groups of 8 rows
    (2, 64, 4, 1, 512, 256, False, {"int4": True}),            # INT4, 10 rows
    (3, 4, 2, 1, 512, 384, False, {"int4": True, "scales": True}),  # INT4, groups of several rows
]


def _pairable(T, E, k, S, fp8):
    """FP8 cases whose groups average more than 128 rows (the layouts differ there)."""
    return fp8 is True and T * (k + S) / (E + S) > 128


GEMM1_PAIR = [c for c in GEMM1_CASES if _pairable(*c[:4], c[6])]


def _bf16_pairable(T, E, k, S, fp8, extra=None):
    """bf16 cases whose groups average more than 128 rows (256-row token blocks)."""
    extra = extra or {}
    return fp8 is False and not extra.get("int4") and not extra.get("fp4") and T * (k + S) / (E + S) > 128


GEMM1_BF16_PAIR = [c for c in GEMM1_CASES if _bf16_pairable(*c[:4], c[6], c[7])]


@pytest.mark.parametrize("T,E,k,S,H,I,fp8,extra", GEMM1_BF16_PAIR)
def test_gemm1_swiglu_bf16_cta_pair(T, E, k, S, H, I, fp8, extra):
    with pair_layout(True):
        test_gemm1_swiglu(T, E, k, S, H, I, fp8, extra)


@pytest.mark.parametrize("T,E,k,S,H,I,fp8,extra", GEMM1_PAIR)
def test_gemm1_swiglu_fp8_cta_pair(T, E, k, S, H, I, fp8, extra):
    with fp8_layout(pair=True):
        test_gemm1_swiglu(T, E, k, S, H, I, fp8, extra)


@pytest.mark.parametrize("T,E,k,S,H,I,fp8,extra", GEMM1_CASES)
def test_gemm1_swiglu(T, E, k, S, H, I, fp8, extra):
    oai, glm = extra.get("oai", False), extra.get("glm", False)
    c = make_case(T, E, k, S, H, I, fp8, seed=T + E + H, gate_up_mult=4.0 if oai else 1.0,
                  scales=extra.get("scales", False), skew=extra.get("skew", 0.0), limits=extra.get("limits", False),
                  int4=extra.get("int4", False), fp4=extra.get("fp4", False))
    d = dims_of(c, alpha=1.702 if oai else 1.0, beta=1.0 if oai else 0.0,
                limit=7.0 if oai else (10.0 if glm else math.inf))
    A = c["A"]
    h = torch.zeros((A, I), dtype=torch.uint8 if fp8 else torch.bfloat16, device="cuda")
    hs = torch.zeros((I // 128, A), dtype=torch.float32, device="cuda") if fp8 else None
    ws = moe.alloc_workspace(d, moe.MOE_WS_GEMM1)
    offsets = torch.from_numpy(c["offsets"]).cuda()
    moe.moe_gemm1_swiglu(c["xp"], c["xs"], offsets, c["w1"], c["w1_scale"], c["gate_scale"], c["up_scale"],
                         c["limits"], d,
                         h, hs, ws)
    assert moe.moe_read_status(ws) == 0
    n = int(c["offsets"][-1])
    rows = np.arange(n, dtype=np.int32)
    grp = (np.searchsorted(c["offsets"], rows, side="right") - 1).astype(np.int32)
    L = oracle_of(c, d)
    xp_host = u8(c["xp"]) if fp8 else bits16(c["xp"])
    ref = L.gemm1_rows(A, xp_host, f32(c["xs"]), rows, grp)
    if not fp8:
        assert_bf16_close(h[:n].float().cpu().numpy(), ref, "h")
    else:
        got = e4m3_to_np(h[:n]) * np.repeat(f32(hs)[:, :n].T, 128, axis=1)
        q, s = oracle.quant_1x128(ref.astype(np.float32))
        mirrored = oracle.e4m3_decode(q) * np.repeat(s, 128, axis=1)
        assert_fp8_close(got, mirrored, "h (E4M3)")


GEMM2_CASES = [
    (8, 64, 4, 0, 256, 256, False, False),
    (64, 16, 4, 0, 512, 256, False, False),
    (128, 8, 2, 0, 384, 512, False, False),
    (512, 8, 2, 0, 512, 256, False, False),
    (300, 16, 4, 2, 512, 256, False, True),     # two sink-gated shared groups
    (300, 16, 4, 1, 512, 256, False, False),    # one shared group with weight 1
    (1024, 8, 2, 0, 512, 256, False, False),    # tile 256
    (600, 4, 2, 1, 384, 256, False, True),      # tile 256, odd number of 128-row chunks of H
    (1500, 16, 2, 1, 384, 256, False, False),   # tile 256, skewless large groups, odd chunk count of H
    (512, 8, 2, 0, 512, 256, True, False),      # FP8, tile 128
    (256, 8, 2, 0, 512, 256, True, False),      # FP8, tile 64
    (600, 4, 2, 1, 384, 256, True, True),       # FP8 large groups, odd chunk count of H, sink-gated shared
    (1500, 16, 2, 1, 384, 256, True, False),    # FP8 large groups, odd chunk count of H
    (300, 8, 2, 1, 512, 256, True, False),      # FP8, tile 128 (single CTA), shared group
    (40, 32, 4, 1, 512, 256, True, False),
    (8, 64, 4, 0, 256, 256, "int4", False),     # INT4 weights, tile 16
    (300, 16, 4, 2, 512, 256, "int4", True),    # INT4, sink-gated shared groups
    (512, 8, 2, 0, 384, 256, "int4", False),    # INT4, tile 128, odd chunk count of H
    (2, 64, 4, 1, 512, 256, False, False),      # decode-sized: 10 routed rows
    (2, 16, 4, 2, 512, 256, False, True),       # decode-sized, sink-gated shared groups
    (8, 2, 2, 0, 384, 256, "int4", False),      # INT4, 2 groups of 8 rows
    (8, 64, 4, 0, 256, 256, "fp4", False),      # NVFP4, tile 16
    (300, 16, 4, 2, 512, 256, "fp4", True),     # NVFP4, sink-gated shared groups
    (512, 8, 2, 0, 384, 256, "fp4", False),     # NVFP4, tile 64, odd chunk count of H
    # many token blocks, an odd count of 128-row chunks of H (the last GEMM2 tile has one)
    (4096, 128, 2, 0, 384, 256, False, False),
    (4096, 128, 2, 0, 384, 256, True, False),   # FP8, tile 64
]


GEMM2_PAIR = [c for c in GEMM2_CASES if _pairable(*c[:4], c[6])]
GEMM2_BF16_PAIR = [c for c in GEMM2_CASES if _bf16_pairable(*c[:4], c[6])]


@pytest.mark.parametrize("T,E,k,S,H,I,fp8,sinks", GEMM2_BF16_PAIR)
def test_gemm2_combine_bf16_cta_pair(T, E, k, S, H, I, fp8, sinks):
    with pair_layout(True):
        test_gemm2_combine(T, E, k, S, H, I, fp8, sinks)


@pytest.mark.parametrize("T,E,k,S,H,I,fp8,sinks", GEMM2_PAIR)
def test_gemm2_combine_fp8_cta_pair(T, E, k, S, H, I, fp8, sinks):
    with fp8_layout(pair=True):
        test_gemm2_combine(T, E, k, S, H, I, fp8, sinks)


@pytest.mark.parametrize("T,E,k,S,H,I,fp8,sinks", GEMM2_CASES)
def test_gemm2_combine(T, E, k, S, H, I, fp8, sinks):
    int4, fp4 = fp8 == "int4", fp8 == "fp4"
    fp8 = fp8 is True
    c = make_case(T, E, k, S, H, I, fp8, seed=3 * T + E, sinks=sinks, int4=int4, fp4=fp4)
    d = dims_of(c)
    out = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    ws = moe.alloc_workspace(d, moe.MOE_WS_GEMM2_COMBINE)
    offsets = torch.from_numpy(c["offsets"]).cuda()
    inv = torch.from_numpy(c["inv"]).cuda()
    moe.moe_gemm2_combine(c["hp"], c["hs"], offsets, inv, c["topk_w"], c["shared_w"], c["w2"], c["w2_scale"], d,
                          out, ws)
    assert moe.moe_read_status(ws) == 0
    A = c["A"]
    row_w = np.zeros(A, np.float32)
    tw = f32(c["topk_w"])
    for t in range(T):
        for j in range(k):
            row_w[c["inv"][t, j]] = tw[t, j]
        for s in range(S):
            row_w[c["offsets"][E + s] + t] = f32(c["shared_w"])[t, s] if c["shared_w"] is not None else 1.0
    L = oracle_of(c, d)
    hp_host = u8(c["hp"]) if fp8 else bits16(c["hp"])
    ref = L.gemm2_rows(A, hp_host, f32(c["hs"]), c["offsets"], c["inv"], row_w, np.arange(T, dtype=np.int32))
    got = out.float().cpu().numpy()
    if fp8:
        assert_fp8_close(got, ref, "out")
    assert_bf16_close(got, ref, "out")
