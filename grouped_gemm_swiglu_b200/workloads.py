"""Seeded synthetic inputs for the MoE expert layer, shaped like the pages' workloads.

This module holds input recipes only (random draws, the gate GEMV that produces the
router's input logits, the offline FP8 weight format). None of the layer's own
arithmetic (routing, permutation, GEMMs, activation, combine) lives here; both the
CUDA path and the fp64 oracle receive the exact same bytes from it.

Workloads (synthetic stand-ins; no checkpoint or evaluation data is used):
  tiny          T=16,   H=256,  I=128,  E=8,   top-2, sigmoid+LSE, plain SwiGLU, bf16.
  oai_swiglu    T=256,  H=2048, I=768,  E=32,  top-4, softmax, alpha=1.702, beta=1, L=7,
                gate and up weight rows x4 so that the clamp fires (MiniMax-M3 parameters,
                DeepGEMM PR #445 "Summary").
  qwen3_30b_a3b T=4096, H=2048, I=768,  E=128, top-8, softmax, per-expert gate/up scales
                U[0.52, 1.22] (xorl-wheels release notes, "Changes": up/gate ratios).
  glm_fp8       T=8192, H=4096, I=1536, E=288 + 1 shared, top-8, sigmoid+LSE, L=10,
                E4M3 weights with 128x128 fp32 block scales (sglang PR #39920, "Motivation").
  decode_t{1,8,64}  H=4096, I=1024, 256 routed + 2 sink-gated shared experts, top-8,
                sigmoid+LSE with sinks, Zipf(1.2) expert popularity, row 0 all logits
                below -104 with exact ties at the top-8 boundary (sglang PR #36385, item 2).
  decode_t{1,64}_int4  the decode shapes with INT4 group-32 weights (batchgen PR #239 commit
                notes: packed nibbles, one bf16 scale per 32 K); uniform nibbles and scales
                drawn so that the weights' spread matches the bf16 workloads (std ~0.02).
  decode_t{1,64}_nvfp4  the decode shapes with NVFP4 weights (E2M1, one E4M3 scale per 16 K)
                and per-expert gate/up global scales U[0.52, 1.22] (xorl-wheels release
                notes, "Changes": NVFP4 checkpoints with distinct gate and up scales).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

WDTYPE_BF16 = 0
WDTYPE_FP8 = 1
WDTYPE_INT4 = 2
WDTYPE_NVFP4 = 3
SCORE_SOFTMAX = 0
SCORE_SIGMOID = 1

INF = float("inf")


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    n_sink: int = 0
    n_shared: int = 0
    wdtype: int = WDTYPE_BF16
    score: int = SCORE_SOFTMAX
    alpha: float = 1.0
    beta: float = 0.0
    limit: float = INF
    route_scale: float = 1.0
    wr_std: float = 0.05
    w_std: float = 0.02
    gate_up_mult: float = 1.0
    expert_scales: tuple | None = None
    zipf_s: float = 0.0
    special_row: bool = False
    seed: int = 0
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def G(self) -> int:
        return self.E + self.n_shared

    @property
    def A(self) -> int:
        return self.T * self.k + self.T * self.n_shared

    @property
    def n_cols(self) -> int:
        return self.E + self.n_sink

    def flops(self) -> float:
        """Useful GEMM FLOPs of one layer pass: 2*A*H*2I + 2*A*I*H."""
        return 2.0 * self.A * self.H * 2 * self.I + 2.0 * self.A * self.I * self.H

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", T=16, H=256, I=128, E=8, k=2, score=SCORE_SIGMOID, wr_std=0.1),
    "oai_swiglu": Workload("oai_swiglu", T=256, H=2048, I=768, E=32, k=4, score=SCORE_SOFTMAX,
                           alpha=1.702, beta=1.0, limit=7.0, gate_up_mult=4.0),
    "qwen3_30b_a3b": Workload("qwen3_30b_a3b", T=4096, H=2048, I=768, E=128, k=8,
                              score=SCORE_SOFTMAX, expert_scales=(0.52, 1.22)),
    "glm_fp8": Workload("glm_fp8", T=8192, H=4096, I=1536, E=288, k=8, n_shared=1,
                        wdtype=WDTYPE_FP8, score=SCORE_SIGMOID, limit=10.0),
    "decode_t1": Workload("decode_t1", T=1, H=4096, I=1024, E=256, k=8, n_sink=2, n_shared=2,
                          score=SCORE_SIGMOID, zipf_s=1.2, special_row=True),
    "decode_t8": Workload("decode_t8", T=8, H=4096, I=1024, E=256, k=8, n_sink=2, n_shared=2,
                          score=SCORE_SIGMOID, zipf_s=1.2, special_row=True),
    "decode_t64": Workload("decode_t64", T=64, H=4096, I=1024, E=256, k=8, n_sink=2, n_shared=2,
                           score=SCORE_SIGMOID, zipf_s=1.2, special_row=True),
    "decode_t1_int4": Workload("decode_t1_int4", T=1, H=4096, I=1024, E=256, k=8, n_sink=2, n_shared=2,
                               wdtype=WDTYPE_INT4, score=SCORE_SIGMOID, zipf_s=1.2, special_row=True),
    "decode_t64_int4": Workload("decode_t64_int4", T=64, H=4096, I=1024, E=256, k=8, n_sink=2, n_shared=2,
                                wdtype=WDTYPE_INT4, score=SCORE_SIGMOID, zipf_s=1.2, special_row=True),
    "decode_t1_nvfp4": Workload("decode_t1_nvfp4", T=1, H=4096, I=1024, E=256, k=8, n_sink=2, n_shared=2,
                                wdtype=WDTYPE_NVFP4, score=SCORE_SIGMOID, zipf_s=1.2, special_row=True,
                                expert_scales=(0.52, 1.22)),
    "decode_t64_nvfp4": Workload("decode_t64_nvfp4", T=64, H=4096, I=1024, E=256, k=8, n_sink=2, n_shared=2,
                                 wdtype=WDTYPE_NVFP4, score=SCORE_SIGMOID, zipf_s=1.2, special_row=True,
                                 expert_scales=(0.52, 1.22)),
}


def _randn(gen, shape, device, std=1.0):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std


def fp8_block_quantize_weights(w: torch.Tensor):
    """Offline E4M3 weight format with one fp32 scale per 128x128 block (the input
    format of the GLM FP8 workload, not a step of the layer): s = amax/448 (1 for an
    all-zero block), codes = E4M3(w/s). Returns (codes uint8 [..,R,C], scales [..,R/128,C/128])."""
    *lead, R, C = w.shape
    blk = w.reshape(*lead, R // 128, 128, C // 128, 128)
    amax = blk.abs().amax(dim=(-3, -1))
    s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    q = (blk / s[..., :, None, :, None]).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)
    return q.reshape(*lead, R, C).view(torch.uint8), s.to(torch.float32).contiguous()


def random_int4_weights(gen, shape, device, std: float):
    """Offline INT4 group-32 weight format (an input format, not a step of the layer):
    uniform random bytes [.., R, C/2] (two nibbles each, low nibble = even column) and one
    bf16 scale per row and 32 columns [.., R, C/32], drawn around std / 4.6 (the standard
    deviation of nibble - 8 for uniform nibbles) so the weights have std close to `std`."""
    *lead, R, C = shape
    packed = torch.randint(0, 256, (*lead, R, C // 2), generator=gen, device=device, dtype=torch.int32)
    scale = (std / 4.6) * (0.75 + 0.5 * torch.rand((*lead, R, C // 32), generator=gen, device=device))
    return packed.to(torch.uint8).contiguous(), scale.to(torch.bfloat16).contiguous()


def random_nvfp4_weights(gen, shape, device, std: float):
    """Offline NVFP4 weight format (an input format, not a step of the layer): uniform random
    bytes [.., R, C/2] (two E2M1 codes each, low nibble = even column) and one E4M3 scale per
    row and 16 columns [.., R, C/16] (uint8 codes), drawn around std / 2.93 (the root mean
    square of the 16 E2M1 values) so the weights have std close to `std`."""
    *lead, R, C = shape
    packed = torch.randint(0, 256, (*lead, R, C // 2), generator=gen, device=device, dtype=torch.int32)
    scale = (std / 2.926) * (0.75 + 0.5 * torch.rand((*lead, R, C // 16), generator=gen, device=device))
    codes = scale.to(torch.float8_e4m3fn).view(torch.uint8)
    return packed.to(torch.uint8).contiguous(), codes.contiguous()


def _special_row(gen, n_cols: int, k: int, device) -> torch.Tensor:
    """Every logit below -104 (where fp32 sigmoid flushes to zero), drawn from
    {-105, -110, -150, -200}, with an exact tie straddling the top-k boundary:
    k-3 columns at -105 and 6 columns at -110, the rest at -150 / -200."""
    vals = torch.full((n_cols,), -150.0, dtype=torch.float64, device=device)
    perm = torch.randperm(n_cols, generator=gen, device=device)
    top = perm[: k - 3]
    tie = perm[k - 3: k + 3]
    low = perm[k + 3: k + 3 + n_cols // 3]
    vals[top] = -105.0
    vals[tie] = -110.0
    vals[low] = -200.0
    return vals


def make_inputs(wl: Workload, device="cpu", seed: int | None = None) -> dict:
    """Draw every input of one layer pass on `device` with a seeded torch generator.

    Returns torch tensors: x bf16 [T,H]; logits fp32 [T,E+n_sink]; w1 [G,2I,H] and
    w2 [G,H,I] (bf16, or uint8 E4M3 codes with w1_scale/w2_scale fp32 block scales, or
    INT4 packed bytes [G,2I,H/2] / [G,H,I/2] with bf16 group scales [G,2I,H/32] / [G,H,I/32],
    or NVFP4 packed bytes with E4M3 scale codes [G,2I,H/16] / [G,H,I/16]);
    gate_scale/up_scale fp32 [G] or None. Gate logits are x.W_r in fp64 rounded to fp32.
    """
    seed = wl.seed if seed is None else seed
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    T, H, I, E, G = wl.T, wl.H, wl.I, wl.E, wl.G

    x = _randn(gen, (T, H), dev).to(torch.bfloat16)
    w_r = _randn(gen, (H, wl.n_cols), dev, wl.wr_std).to(torch.float64)
    logits = x.to(torch.float64) @ w_r
    if wl.zipf_s > 0.0:
        # Popularity ~ rank^-s: add -s * std(logit) * ln(rank_e) to routed column e,
        # with a seeded random rank per expert. Sink columns take no offset.
        rank = torch.randperm(E, generator=gen, device=dev).to(torch.float64) + 1.0
        sd = float(logits[:, :E].std()) if T > 1 else wl.wr_std * math.sqrt(H)
        logits[:, :E] += -wl.zipf_s * sd * torch.log(rank)[None, :]
    if wl.special_row:
        logits[0] = _special_row(gen, wl.n_cols, wl.k, dev)
    logits = logits.to(torch.float32).contiguous()

    # Expert weights: rows [0, I) of W1 are the gate half, [I, 2I) the up half.
    chunk = max(1, min(G, (1 << 28) // (2 * I * H)))
    w1_parts, w2_parts, s1_parts, s2_parts = [], [], [], []
    for g0 in range(0, G, chunk):
        n = min(chunk, G - g0)
        w1 = _randn(gen, (n, 2 * I, H), dev, wl.w_std)
        if wl.gate_up_mult != 1.0:
            w1 = w1 * wl.gate_up_mult
        w2 = _randn(gen, (n, H, I), dev, wl.w_std)
        if wl.wdtype == WDTYPE_FP8:
            q1, s1 = fp8_block_quantize_weights(w1)
            q2, s2 = fp8_block_quantize_weights(w2)
            w1_parts.append(q1); w2_parts.append(q2); s1_parts.append(s1); s2_parts.append(s2)
        elif wl.wdtype == WDTYPE_INT4:
            q1, s1 = random_int4_weights(gen, (n, 2 * I, H), dev, wl.w_std * wl.gate_up_mult)
            q2, s2 = random_int4_weights(gen, (n, H, I), dev, wl.w_std)
            w1_parts.append(q1); w2_parts.append(q2); s1_parts.append(s1); s2_parts.append(s2)
        elif wl.wdtype == WDTYPE_NVFP4:
            q1, s1 = random_nvfp4_weights(gen, (n, 2 * I, H), dev, wl.w_std * wl.gate_up_mult)
            q2, s2 = random_nvfp4_weights(gen, (n, H, I), dev, wl.w_std)
            w1_parts.append(q1); w2_parts.append(q2); s1_parts.append(s1); s2_parts.append(s2)
        else:
            w1_parts.append(w1.to(torch.bfloat16)); w2_parts.append(w2.to(torch.bfloat16))
        del w1, w2
    out = dict(x=x.contiguous(), logits=logits,
               w1=torch.cat(w1_parts).contiguous(), w2=torch.cat(w2_parts).contiguous(),
               w1_scale=torch.cat(s1_parts).contiguous() if s1_parts else None,
               w2_scale=torch.cat(s2_parts).contiguous() if s2_parts else None,
               gate_scale=None, up_scale=None)
    if wl.expert_scales is not None:
        lo, hi = wl.expert_scales
        out["gate_scale"] = (lo + (hi - lo) * torch.rand((G,), generator=gen, device=dev)).contiguous()
        out["up_scale"] = (lo + (hi - lo) * torch.rand((G,), generator=gen, device=dev)).contiguous()
    return out


def random_topk_ids(T: int, E: int, k: int, seed: int = 0, skew: float = 0.0) -> torch.Tensor:
    """Distinct expert ids per token (CPU int32 [T,k]); skew > 0 favours low ids."""
    gen = torch.Generator().manual_seed(seed)
    keys = torch.rand((T, E), generator=gen)
    if skew > 0:
        keys = keys * (torch.arange(E, dtype=torch.float32) + 1.0)[None, :] ** skew
    return torch.argsort(keys, dim=1)[:, :k].to(torch.int32).contiguous()


def random_activations(rows: int, cols: int, seed: int = 0, device="cpu", std=1.0) -> torch.Tensor:
    gen = torch.Generator(device=torch.device(device)).manual_seed(seed)
    return _randn(gen, (rows, cols), torch.device(device), std)
