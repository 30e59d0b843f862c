"""ctypes binding of libmoe_b200.so: same names and arguments as include/moe_b200.h.

Argument marshalling only: torch tensors are passed as device pointers, every step
runs in the library's CUDA kernels. There is no CPU fallback; if the library is
missing or the device is not sm_100, calls raise.
"""
from __future__ import annotations

import ctypes
import math
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libmoe_b200.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "moe_b200.h")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_ARCH",
                -4: "MOE_ERR_WORKSPACE", -5: "MOE_ERR_EXPERT_ID", -6: "MOE_ERR_TIMEOUT", -7: "MOE_ERR_CUDA"}
MOE_WS_PERMUTE, MOE_WS_GEMM1, MOE_WS_GEMM2_COMBINE, MOE_WS_FORWARD, MOE_WS_EXPERTS, MOE_WS_COMBINE = 0, 1, 2, 3, 4, 5
MOE_WS_GATE_ROUTE = 6
MOE_SCORE_SOFTMAX, MOE_SCORE_SIGMOID = 0, 1
MOE_WDTYPE_BF16, MOE_WDTYPE_FP8_E4M3_BLOCK128, MOE_WDTYPE_INT4_G32, MOE_WDTYPE_NVFP4 = 0, 1, 2, 3


class MoeError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {STATUS_NAMES.get(status, status)}: {status_string(status)}")


class MoeDims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32), ("E", ctypes.c_int32),
                ("k", ctypes.c_int32), ("n_sink", ctypes.c_int32), ("n_shared", ctypes.c_int32),
                ("wdtype", ctypes.c_int32), ("score", ctypes.c_int32),
                ("alpha", ctypes.c_float), ("beta", ctypes.c_float), ("limit", ctypes.c_float),
                ("route_scale", ctypes.c_float)]

    @classmethod
    def of(cls, wl, T: int | None = None) -> "MoeDims":
        """From a workloads.Workload (or anything with the same attribute names)."""
        return cls(T=wl.T if T is None else T, H=wl.H, I=wl.I, E=wl.E, k=wl.k, n_sink=wl.n_sink,
                   n_shared=wl.n_shared, wdtype=wl.wdtype, score=wl.score, alpha=wl.alpha, beta=wl.beta,
                   limit=wl.limit if math.isfinite(wl.limit) else float("inf"), route_scale=wl.route_scale)

    @property
    def G(self) -> int:
        return self.E + self.n_shared

    @property
    def A(self) -> int:
        return self.T * (self.k + self.n_shared)


_lib = None
_VP = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m grouped_gemm_swiglu_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(MoeDims)
        sig = {
            "moe_abi_version": ([], ctypes.c_int),
            "moe_set_option": ([ctypes.c_int, ctypes.c_int], ctypes.c_int),
            "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
            "moe_workspace_size": ([P, ctypes.c_int, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
            "moe_read_status": ([_VP, ctypes.POINTER(ctypes.c_int32), _VP], ctypes.c_int),
            "moe_clear_status": ([_VP, _VP], ctypes.c_int),
            "moe_route_topk": ([_VP, P, _VP, _VP, _VP, _VP, _VP, _VP], ctypes.c_int),
            "moe_permute": ([_VP, _VP, P, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_size_t, _VP], ctypes.c_int),
            "moe_gemm1_swiglu": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, P, _VP, _VP, _VP, ctypes.c_size_t, _VP],
                                 ctypes.c_int),
            "moe_gemm2_combine": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, P, _VP, _VP, ctypes.c_size_t, _VP],
                                  ctypes.c_int),
            "moe_forward": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, P, _VP, _VP, _VP, _VP, _VP, _VP,
                             ctypes.c_size_t, _VP], ctypes.c_int),
            "moe_experts": ([_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, P, _VP, _VP, _VP, _VP,
                             ctypes.c_size_t, _VP], ctypes.c_int),
            "moe_combine": ([_VP, _VP, _VP, _VP, _VP, P, _VP, _VP, ctypes.c_size_t, _VP], ctypes.c_int),
            "moe_gate_route": ([_VP, _VP, P, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_size_t, _VP], ctypes.c_int),
            "moe_ep_row_ids": ([_VP, P, _VP, _VP], ctypes.c_int),
            "moe_ep_rebase": ([_VP, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                               _VP, _VP], ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = res
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/moe_b200.h declares."""
    text = open(HEADER_PATH).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(moe_\w+)\s*\(", text, flags=re.M)


def status_string(status: int) -> str:
    try:
        return lib().moe_status_string(int(status)).decode()
    except Exception:  # library missing: still give a message
        return STATUS_NAMES.get(status, str(status))


def _p(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _s(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, rc: int):
    if rc != MOE_OK:
        raise MoeError(fn, rc)


def moe_abi_version() -> int:
    return int(lib().moe_abi_version())


MOE_OPT_FP8_CTA_PAIR = 1
MOE_OPT_BF16_CTA_PAIR = 2


def moe_set_option(option: int, value: int) -> int:
    """Process-wide kernel-layout option (see moe_set_option in the header); returns the
    previous value."""
    rc = int(lib().moe_set_option(int(option), int(value)))
    if rc < 0:
        raise MoeError("moe_set_option", rc)
    return rc


def moe_workspace_size(dims: MoeDims, kind: int) -> int:
    n = ctypes.c_size_t(0)
    _check("moe_workspace_size", lib().moe_workspace_size(ctypes.byref(dims), kind, ctypes.byref(n)))
    return int(n.value)


def moe_read_status(ws, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check("moe_read_status", lib().moe_read_status(_p(ws), ctypes.byref(v), _s(stream)))
    return int(v.value)


def moe_clear_status(ws, stream=None) -> None:
    _check("moe_clear_status", lib().moe_clear_status(_p(ws), _s(stream)))


def moe_route_topk(logits, dims: MoeDims, bias, topk_ids, topk_w, shared_w=None, packed=None, stream=None) -> None:
    _check("moe_route_topk", lib().moe_route_topk(_p(logits), ctypes.byref(dims), _p(bias), _p(topk_ids),
                                                  _p(topk_w), _p(shared_w), _p(packed), _s(stream)))


def moe_gate_route(x, w_gate, dims: MoeDims, bias, logits, topk_ids, topk_w, shared_w, packed, ws,
                   stream=None) -> None:
    _check("moe_gate_route", lib().moe_gate_route(_p(x), _p(w_gate), ctypes.byref(dims), _p(bias), _p(logits),
                                                  _p(topk_ids), _p(topk_w), _p(shared_w), _p(packed), _p(ws),
                                                  _nbytes(ws), _s(stream)))


def moe_permute(topk_ids, x, dims: MoeDims, offsets, perm, inv_perm, x_perm, x_scale, ws, stream=None) -> None:
    _check("moe_permute", lib().moe_permute(_p(topk_ids), _p(x), ctypes.byref(dims), _p(offsets), _p(perm),
                                            _p(inv_perm), _p(x_perm), _p(x_scale), _p(ws), _nbytes(ws),
                                            _s(stream)))


def moe_gemm1_swiglu(x_perm, x_scale, offsets, w1, w1_scale, gate_scale, up_scale, limits, dims: MoeDims, h,
                     h_scale, ws, stream=None) -> None:
    _check("moe_gemm1_swiglu", lib().moe_gemm1_swiglu(_p(x_perm), _p(x_scale), _p(offsets), _p(w1), _p(w1_scale),
                                                      _p(gate_scale), _p(up_scale), _p(limits), ctypes.byref(dims),
                                                      _p(h), _p(h_scale), _p(ws), _nbytes(ws), _s(stream)))


def moe_gemm2_combine(h, h_scale, offsets, inv_perm, topk_w, shared_w, w2, w2_scale, dims: MoeDims, out, ws,
                      stream=None) -> None:
    _check("moe_gemm2_combine", lib().moe_gemm2_combine(_p(h), _p(h_scale), _p(offsets), _p(inv_perm), _p(topk_w),
                                                        _p(shared_w), _p(w2), _p(w2_scale), ctypes.byref(dims),
                                                        _p(out), _p(ws), _nbytes(ws), _s(stream)))


def moe_forward(logits, bias, x, w1, w1_scale, gate_scale, up_scale, limits, w2, w2_scale, dims: MoeDims, out,
                topk_ids=None, topk_w=None, shared_w=None, packed=None, ws=None, stream=None) -> None:
    _check("moe_forward", lib().moe_forward(_p(logits), _p(bias), _p(x), _p(w1), _p(w1_scale), _p(gate_scale),
                                            _p(up_scale), _p(limits), _p(w2), _p(w2_scale), ctypes.byref(dims),
                                            _p(out), _p(topk_ids), _p(topk_w), _p(shared_w), _p(packed), _p(ws),
                                            _nbytes(ws), _s(stream)))


def moe_experts(x_perm, x_scale, offsets, w1, w1_scale, gate_scale, up_scale, limits, w2, w2_scale, dims: MoeDims,
                h, h_scale, y, ws, stream=None) -> None:
    _check("moe_experts", lib().moe_experts(_p(x_perm), _p(x_scale), _p(offsets), _p(w1), _p(w1_scale),
                                            _p(gate_scale), _p(up_scale), _p(limits), _p(w2), _p(w2_scale),
                                            ctypes.byref(dims), _p(h), _p(h_scale), _p(y), _p(ws), _nbytes(ws),
                                            _s(stream)))


def moe_combine(y, offsets, inv_perm, topk_w, shared_w, dims: MoeDims, out, ws, stream=None) -> None:
    _check("moe_combine", lib().moe_combine(_p(y), _p(offsets), _p(inv_perm), _p(topk_w), _p(shared_w),
                                            ctypes.byref(dims), _p(out), _p(ws), _nbytes(ws), _s(stream)))


def moe_ep_row_ids(offsets, dims: MoeDims, row_ids, stream=None) -> None:
    _check("moe_ep_row_ids", lib().moe_ep_row_ids(_p(offsets), ctypes.byref(dims), _p(row_ids), _s(stream)))


def moe_ep_rebase(ids, n: int, E: int, n_shared: int, local_offset: int, n_local: int, out, stream=None) -> None:
    _check("moe_ep_rebase", lib().moe_ep_rebase(_p(ids), int(n), int(E), int(n_shared), int(local_offset),
                                                int(n_local), _p(out), _s(stream)))


def _nbytes(t) -> int:
    if t is None:
        return 0
    return t.numel() * t.element_size()


def alloc_workspace(dims: MoeDims, kind: int, device="cuda") -> torch.Tensor:
    """A zeroed, 256-byte aligned workspace (uint8) for the given call."""
    n = moe_workspace_size(dims, kind)
    ws = torch.zeros(n + 256, dtype=torch.uint8, device=device)
    off = (-ws.data_ptr()) % 256
    return ws[off:off + n]


def moe_permute_noalloc(topk_ids, x, dims: MoeDims, offsets, perm, inv_perm, x_perm, x_scale, status=None,
                        stream=None) -> None:
    """moe_permute without a workspace: the scratch is a fixed array inside the library
    (for callers that cannot allocate device memory; see include/moe_b200.h)."""
    fn = lib().moe_permute_noalloc
    if fn.restype is not ctypes.c_int:
        fn.argtypes = [_VP, _VP, ctypes.POINTER(MoeDims), _VP, _VP, _VP, _VP, _VP, _VP, _VP]
        fn.restype = ctypes.c_int
    _check("moe_permute_noalloc", fn(_p(topk_ids), _p(x), ctypes.byref(dims), _p(offsets), _p(perm),
                                     _p(inv_perm), _p(x_perm), _p(x_scale), _p(status), _s(stream)))
