"""Permutation by expert on the GPU against the oracle: offsets, perm and inv_perm
bit-exact; the gathered rows are exact copies (bf16) or bit-exact E4M3 codes and scales
(FP8, 1x128 blocks, decided in fp32 on both sides)."""
import numpy as np
import pytest
import torch

import oracle
import grouped_gemm_swiglu_b200 as moe
from grouped_gemm_swiglu_b200 import workloads as W
from helpers import bits16

pytestmark = pytest.mark.gpu


def gpu_permute(ids: torch.Tensor, x: torch.Tensor, E: int, n_shared: int, fp8: bool):
    T, k = ids.shape
    H = x.shape[1]
    d = moe.MoeDims(T=T, H=H, I=128, E=E, k=k, n_sink=0, n_shared=n_shared, wdtype=1 if fp8 else 0,
                    score=0, alpha=1.0, beta=0.0, limit=float("inf"), route_scale=1.0)
    A = d.A
    dev = x.device
    offsets = torch.full((E + n_shared + 1,), -9, dtype=torch.int32, device=dev)
    perm = torch.full((A,), -9, dtype=torch.int32, device=dev)
    inv = torch.full((T, k), -9, dtype=torch.int32, device=dev)
    xp = torch.zeros((A, H), dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev)
    xs = torch.zeros((H // 128, A), dtype=torch.float32, device=dev) if fp8 else None
    ws = moe.alloc_workspace(d, moe.MOE_WS_PERMUTE, device=dev)
    moe.moe_permute(ids, x, d, offsets, perm, inv, xp, xs, ws)
    status = moe.moe_read_status(ws)
    return offsets.cpu().numpy(), perm.cpu().numpy(), inv.cpu().numpy(), xp, xs, status


@pytest.mark.parametrize("T,E,k,S,H,fp8,skew", [
    (16, 8, 2, 0, 256, False, 0.0),
    (37, 16, 4, 1, 256, False, 0.0),
    (300, 64, 8, 0, 384, False, 2.0),     # two counting chunks, skewed, H/8 not a multiple of 32
    (1000, 288, 8, 1, 512, True, 0.0),    # several chunks, FP8 with a shared group
    (777, 256, 8, 2, 1024, True, 3.0),
    (1, 256, 8, 2, 4096, False, 0.0),     # decode token
    (513, 4, 4, 0, 128, True, 0.0),       # k = E: every group holds every token
])
def test_permute_matches_oracle(T, E, k, S, H, fp8, skew):
    ids = W.random_topk_ids(T, E, k, seed=T + E, skew=skew)
    x = W.random_activations(T, H, seed=T, device="cuda").to(torch.bfloat16)
    offsets, perm, inv, xp, xs, status = gpu_permute(ids.cuda(), x, E, S, fp8)
    assert status == 0
    o_off, o_perm, o_inv = oracle.permute(ids.numpy(), E, S)
    assert np.array_equal(offsets, o_off)
    assert np.array_equal(perm, o_perm)
    assert np.array_equal(inv, o_inv)
    xb = bits16(x)
    if not fp8:
        assert np.array_equal(bits16(xp), xb[o_perm])
    else:
        xf = (xb.astype(np.uint32) << 16).view(np.float32)[o_perm]
        q, s = oracle.quant_1x128(xf)
        assert np.array_equal(xp.cpu().numpy(), q), "E4M3 codes differ"
        assert np.array_equal(xs.cpu().numpy(), s.T), "block scales differ"


def test_permute_empty_and_all_to_one_expert():
    offsets, perm, inv, xp, xs, status = gpu_permute(torch.zeros((0, 4), dtype=torch.int32, device="cuda"),
                                                      torch.zeros((0, 256), dtype=torch.bfloat16, device="cuda"),
                                                      8, 1, False)
    assert status == 0 and np.all(offsets == 0)
    T, E, k = 200, 32, 4
    ids = torch.arange(k, dtype=torch.int32).repeat(T, 1)  # every token to experts 0..3
    x = W.random_activations(T, 256, seed=1, device="cuda").to(torch.bfloat16)
    offsets, perm, inv, xp, xs, status = gpu_permute(ids.cuda(), x, E, 0, False)
    o_off, o_perm, o_inv = oracle.permute(ids.numpy(), E, 0)
    assert status == 0 and np.array_equal(offsets, o_off) and np.array_equal(perm, o_perm)
    assert offsets[4] == offsets[-1] == T * k


def test_permute_flags_bad_ids_without_writing_out_of_range():
    T, E, k = 64, 16, 2
    ids = W.random_topk_ids(T, E, k, seed=5)
    ids[3, 1] = E          # out of range
    ids[9, 0] = -1
    ids[11, 1] = ids[11, 0]  # repeated within a token
    x = W.random_activations(T, 256, seed=2, device="cuda").to(torch.bfloat16)
    offsets, perm, inv, xp, xs, status = gpu_permute(ids.cuda(), x, E, 0, False)
    assert status == moe.MoeError("x", -5).status
    assert inv[3, 1] == -1 and inv[9, 0] == -1
    assert offsets[-1] <= T * k and np.all(np.diff(offsets) >= 0)
