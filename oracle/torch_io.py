"""Marshalling of the seeded torch inputs into the oracle's host formats.

TEST INFRASTRUCTURE (tests, smoke check, the bench's CPU-baseline and reference legs).
No arithmetic of the layer: only device-to-host copies and dtype views.
"""
from __future__ import annotations

import numpy as np

from . import Layer


def _bits16(t):
    return t.detach().contiguous().view(__import__("torch").int16).cpu().numpy().view(np.uint16)


def host_inputs(inp: dict) -> dict:
    """torch input dict (any device) -> numpy dict: bf16 as uint16 bits, E4M3 as uint8."""
    import torch
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif v.dtype == torch.bfloat16:
            out[k] = _bits16(v)
        elif v.dtype == torch.uint8:
            out[k] = v.detach().contiguous().cpu().numpy()
        else:
            out[k] = v.detach().float().contiguous().cpu().numpy()
    return out


def oracle_layer_from_inputs(wl, host: dict) -> Layer:
    """oracle.Layer over a workload's host inputs (see grouped_gemm_swiglu_b200.workloads)."""
    return Layer(T=wl.T, H=wl.H, I=wl.I, E=wl.E, k=wl.k, n_sink=wl.n_sink, n_shared=wl.n_shared,
                 wdtype=wl.wdtype, score=wl.score, alpha=wl.alpha, beta=wl.beta, limit=wl.limit,
                 route_scale=wl.route_scale, logits=host["logits"], x=host["x"], w1=host["w1"], w2=host["w2"],
                 w1_scale=host.get("w1_scale"), w2_scale=host.get("w2_scale"),
                 gate_scale=host.get("gate_scale"), up_scale=host.get("up_scale"),
                 limits=host.get("limits"), router_bias=host.get("router_bias"))
