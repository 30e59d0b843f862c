"""moe_permute_noalloc: the permutation for callers that cannot allocate device memory
(a framework that has already planned all of the GPU's memory, a plugin interface that
passes only inputs and outputs, latency-critical code that must not call cudaMalloc).

It is checked against moe_permute, the workspace entry point, through the C ABI, on two
calls in a row: the scratch array inside the library is shared and keeps the previous
call's contents, so the second call must not depend on them. Collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import grouped_gemm_swiglu_b200 as moe
from grouped_gemm_swiglu_b200 import _lib
from grouped_gemm_swiglu_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _dims(T, E, k, S, H, fp8, wdtype=None):
    wd = (1 if fp8 else 0) if wdtype is None else wdtype
    return moe.MoeDims(T=T, H=H, I=128, E=E, k=k, n_sink=0, n_shared=S, wdtype=wd, score=0,
                       alpha=1.0, beta=0.0, limit=float("inf"), route_scale=1.0)


def _outputs(d, fp8, dev="cuda"):
    A, G = d.A, d.G
    return dict(offsets=torch.full((G + 1,), -3, dtype=torch.int32, device=dev),
                perm=torch.full((A,), -3, dtype=torch.int32, device=dev),
                inv=torch.full((d.T, d.k), -3, dtype=torch.int32, device=dev),
                xp=torch.zeros((A, d.H), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev),
                xs=torch.zeros((d.H // 128, A), dtype=torch.float32, device=dev) if fp8 else None)


def _case(T, E, k, S, H, fp8, seed, skew=0.0, wdtype=None):
    ids = W.random_topk_ids(T, E, k, seed=seed, skew=skew).cuda()
    x = W.random_activations(T, H, seed=seed + 1, device="cuda").to(torch.bfloat16)
    d = _dims(T, E, k, S, H, fp8, wdtype)
    ref = _outputs(d, fp8)
    ws = moe.alloc_workspace(d, moe.MOE_WS_PERMUTE)
    moe.moe_permute(ids, x, d, ref["offsets"], ref["perm"], ref["inv"], ref["xp"], ref["xs"], ws)
    assert moe.moe_read_status(ws) == 0
    return ids, x, d, ref


def _call_noalloc(ids, x, d, out, status):
    fn = _lib.lib().moe_permute_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(moe.MoeDims)] + [ctypes.c_void_p] * 7
    fn.restype = ctypes.c_int
    p = lambda t: None if t is None else t.data_ptr()
    return fn(p(ids), p(x), ctypes.byref(d), p(out["offsets"]), p(out["perm"]), p(out["inv"]), p(out["xp"]),
              p(out["xs"]), p(status), torch.cuda.current_stream().cuda_stream)


def _assert_same(got, ref, fp8):
    torch.cuda.synchronize()
    for key in ("offsets", "perm", "inv"):
        assert torch.equal(got[key], ref[key]), key
    assert torch.equal(got["xp"].view(torch.uint8), ref["xp"].view(torch.uint8)), "x_perm"
    if fp8:
        assert torch.equal(got["xs"], ref["xs"]), "x_scale"


def test_noalloc_matches_workspace_entry_on_two_calls_in_a_row():
    cases = [(1000, 288, 8, 1, 512, True, 11, 0.0),   # FP8, several counting chunks, a shared group
             (300, 64, 8, 0, 384, False, 12, 2.0)]    # bf16, skewed, smaller than the first
    for T, E, k, S, H, fp8, seed, skew in cases:
        ids, x, d, ref = _case(T, E, k, S, H, fp8, seed, skew)
        got = _outputs(d, fp8)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert _call_noalloc(ids, x, d, got, status) == 0
        _assert_same(got, ref, fp8)
        assert int(status.item()) == 0
    # the first case again, after the second one left its data in the shared scratch
    T, E, k, S, H, fp8, seed, skew = cases[0]
    ids, x, d, ref = _case(T, E, k, S, H, fp8, seed, skew)
    got = _outputs(d, fp8)
    assert _call_noalloc(ids, x, d, got, None) == 0
    _assert_same(got, ref, fp8)


def test_noalloc_reports_bad_ids_in_the_callers_status_word():
    ids, x, d, _ = _case(64, 16, 2, 0, 256, False, 5)
    ids[3, 1] = 16
    got = _outputs(d, False)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _call_noalloc(ids, x, d, got, status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == -5
    assert int(got["inv"][3, 1].item()) == -1


def test_noalloc_refuses_sizes_beyond_its_scratch():
    d = _dims(40000, 288, 8, 1, 512, False)
    fake = 1 << 20  # never dereferenced: the size check comes first
    fn = _lib.lib().moe_permute_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(moe.MoeDims)] + [ctypes.c_void_p] * 7
    fn.restype = ctypes.c_int
    assert fn(fake, fake, ctypes.byref(d), fake, fake, fake, fake, None, None, None) == -4


def test_noalloc_runs_at_its_largest_size_and_with_4bit_weight_types():
    """T = 28688 at k = 8, E = 288 is the largest problem the static scratch holds (the
    next size is refused: tests/test_abi.py); INT4 and NVFP4 layers permute bf16 rows
    exactly as moe_permute does for them."""
    cases = [(28688, 288, 8, 1, 128, False, 21, 0.0, None),
             (500, 64, 4, 0, 256, False, 22, 0.0, 2),
             (500, 64, 4, 2, 256, False, 23, 1.0, 3)]
    for T, E, k, S, H, fp8, seed, skew, wd in cases:
        ids, x, d, ref = _case(T, E, k, S, H, fp8, seed, skew, wd)
        got = _outputs(d, fp8)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        assert _call_noalloc(ids, x, d, got, status) == 0
        _assert_same(got, ref, fp8)
        assert int(status.item()) == 0
