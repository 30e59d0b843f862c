"""Routed mixture-of-experts expert layer for NVIDIA B200 (sm_100a).

The hot path (router -> permute -> grouped GEMM1 + clamped SwiGLU -> grouped GEMM2 ->
weighted combine) runs in hand-written CUDA kernels of libmoe_b200.so behind the C ABI
of include/moe_b200.h. This package is the thin Python binding: the functions below
carry the C names and only marshal torch tensors (device memory) and streams.
"""
from __future__ import annotations

import torch

from ._lib import (MOE_OK, MOE_SCORE_SIGMOID, MOE_SCORE_SOFTMAX, MOE_WDTYPE_BF16, MOE_WDTYPE_FP8_E4M3_BLOCK128,
                   MOE_WDTYPE_INT4_G32, MOE_WDTYPE_NVFP4,
                   MOE_WS_COMBINE, MOE_WS_EXPERTS, MOE_WS_FORWARD, MOE_WS_GEMM1, MOE_WS_GEMM2_COMBINE,
                   MOE_WS_GATE_ROUTE, MOE_WS_PERMUTE, MoeDims, MoeError, alloc_workspace, header_functions, lib,
                   MOE_OPT_FP8_CTA_PAIR, MOE_OPT_BF16_CTA_PAIR, moe_abi_version, moe_clear_status, moe_set_option, moe_combine, moe_ep_rebase, moe_ep_row_ids, moe_experts,
                   moe_forward, moe_gate_route, moe_gemm1_swiglu, moe_gemm2_combine,
                   moe_permute, moe_permute_noalloc, moe_read_status, moe_route_topk, moe_workspace_size,
                   status_string)

__all__ = ["MoeDims", "MoeError", "MoELayer", "moe_abi_version", "moe_set_option", "MOE_OPT_FP8_CTA_PAIR", "MOE_OPT_BF16_CTA_PAIR", "moe_workspace_size", "moe_read_status",
           "moe_clear_status", "moe_route_topk", "moe_gate_route", "moe_permute", "moe_permute_noalloc", "moe_gemm1_swiglu",
           "moe_gemm2_combine", "moe_experts", "moe_combine", "moe_forward", "moe_ep_row_ids", "moe_ep_rebase",
           "alloc_workspace", "status_string", "lib",
           "header_functions", "MOE_OK",
           "MOE_SCORE_SIGMOID", "MOE_SCORE_SOFTMAX", "MOE_WDTYPE_BF16", "MOE_WDTYPE_FP8_E4M3_BLOCK128",
           "MOE_WDTYPE_INT4_G32", "MOE_WDTYPE_NVFP4",
           "MOE_WS_FORWARD", "MOE_WS_GEMM1", "MOE_WS_GEMM2_COMBINE", "MOE_WS_PERMUTE", "MOE_WS_EXPERTS",
           "MOE_WS_COMBINE", "MOE_WS_GATE_ROUTE"]


class MoELayer:
    """Weights resident on the GPU plus a reusable workspace; `forward` runs moe_forward.

    w1 [G,2I,H] and w2 [G,H,I] are bf16, or uint8 E4M3 codes with w1_scale/w2_scale
    fp32 block scales; gate_scale/up_scale are optional fp32 [G]; limits is an optional
    fp32 [G] clamp per expert (else dims.limit); router_bias an optional fp32 [E]
    correction bias of the ranking. The workspace is sized for `max_tokens` tokens and
    reused by every call with T <= max_tokens.
    """

    def __init__(self, dims: MoeDims, w1, w2, w1_scale=None, w2_scale=None, gate_scale=None, up_scale=None,
                 max_tokens: int | None = None, limits=None, router_bias=None):
        self.dims = dims
        self.w1, self.w2, self.w1_scale, self.w2_scale = w1, w2, w1_scale, w2_scale
        self.gate_scale, self.up_scale = gate_scale, up_scale
        self.limits, self.router_bias = limits, router_bias
        self.max_tokens = dims.T if max_tokens is None else max_tokens
        sized = MoeDims.from_buffer_copy(dims)
        sized.T = self.max_tokens
        self.ws = alloc_workspace(sized, MOE_WS_FORWARD, device=w1.device)

    def forward(self, logits, x, out=None, topk_ids=None, topk_w=None, shared_w=None, packed=None, stream=None):
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError(f"T={T} exceeds the workspace size ({self.max_tokens} tokens)")
        d = MoeDims.from_buffer_copy(self.dims)
        d.T = T
        if out is None:
            out = torch.empty((T, d.H), dtype=torch.bfloat16, device=x.device)
        moe_forward(logits, self.router_bias, x, self.w1, self.w1_scale, self.gate_scale, self.up_scale, self.limits,
                    self.w2, self.w2_scale, d, out, topk_ids, topk_w, shared_w, packed, self.ws, stream)
        return out

    def status(self, stream=None) -> int:
        return moe_read_status(self.ws, stream)
