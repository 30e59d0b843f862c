"""Shared test utilities: moving seeded inputs to the oracle, error metrics, tolerances."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from oracle.torch_io import host_inputs, oracle_layer_from_inputs
from grouped_gemm_swiglu_b200 import workloads as W

# Tolerances of the layer output (fixed by the problem statement of the layer):
#   ids, permutation, offsets: bit-exact; routing weights: 1e-6 absolute (fp32);
#   bf16 output: rel-L2 <= 1e-2 and max-abs <= 2e-2 * max|ref|; FP8 output: rel-L2 <= 3e-2.
TOL_WEIGHTS = 1e-6
TOL_BF16_RELL2 = 1e-2
TOL_BF16_MAXABS = 2e-2
TOL_FP8_RELL2 = 3e-2


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 numpy bits (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().view(np.uint8)


def f32(t):
    return None if t is None else t.detach().float().cpu().numpy()


def oracle_layer(wl: W.Workload, inp: dict) -> oracle.Layer:
    return oracle_layer_from_inputs(wl, host_inputs(inp))


def rel_l2(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = math.sqrt(float((ref * ref).sum()))
    return math.sqrt(float(((got - ref) ** 2).sum())) / max(den, 1e-300)


def assert_bf16_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    r = rel_l2(got, ref)
    m = float(np.abs(got - ref).max()) if got.size else 0.0
    lim = TOL_BF16_MAXABS * float(np.abs(ref).max()) if ref.size else 0.0
    assert r <= TOL_BF16_RELL2, f"{what}: rel-L2 {r:.3e} > {TOL_BF16_RELL2}"
    assert m <= lim, f"{what}: max-abs {m:.3e} > {lim:.3e}"
    return r, m


def assert_fp8_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    r = rel_l2(got, ref)
    assert r <= TOL_FP8_RELL2, f"{what}: rel-L2 {r:.3e} > {TOL_FP8_RELL2}"
    return r


def bf16_to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def e4m3_to_np(codes: torch.Tensor) -> np.ndarray:
    return codes.detach().contiguous().view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.float64)


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    """First, last and random tokens (sorted, unique)."""
    if T <= n:
        return np.arange(T, dtype=np.int32)
    rng = np.random.default_rng(seed)
    pick = set([0, T - 1, T // 2]) | set(rng.choice(T, n - 3, replace=False).tolist())
    return np.array(sorted(pick)[:n], dtype=np.int32)


class fp8_layout:
    """Within the block, FP8 layers with groups above 128 rows run in the given layout:
    pair=True selects the two-CTA tile (moe_set_option(MOE_OPT_FP8_CTA_PAIR, 1))."""

    def __init__(self, pair: bool):
        self.pair = pair

    def __enter__(self):
        import grouped_gemm_swiglu_b200 as moe
        self.old = moe.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, 1 if self.pair else 0)
        return self

    def __exit__(self, *exc):
        import grouped_gemm_swiglu_b200 as moe
        moe.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, self.old)
        return False


class pair_layout:
    """Within the block, layers whose groups average more than 128 rows run in the given
    layout, FP8 and bf16 alike: pair=True selects the two-CTA tiles
    (MOE_OPT_FP8_CTA_PAIR and MOE_OPT_BF16_CTA_PAIR)."""

    def __init__(self, pair: bool):
        self.pair = pair

    def __enter__(self):
        import grouped_gemm_swiglu_b200 as moe
        v = 1 if self.pair else 0
        self.old = (moe.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, v), moe.moe_set_option(moe.MOE_OPT_BF16_CTA_PAIR, v))
        return self

    def __exit__(self, *exc):
        import grouped_gemm_swiglu_b200 as moe
        moe.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, self.old[0])
        moe.moe_set_option(moe.MOE_OPT_BF16_CTA_PAIR, self.old[1])
        return False
