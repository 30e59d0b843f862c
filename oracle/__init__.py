"""fp64 CPU oracle of the routed MoE expert layer (ctypes wrapper over oracle.c).

TEST INFRASTRUCTURE. Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product library
(``grouped_gemm_swiglu_b200``) never imports it and has no CPU fallback.

The arithmetic lives in ``oracle.c``; each C function there names the passage of
the pages it follows. This module only marshals numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
# ORACLE_LIB selects another build of oracle.c (the mutation tests load planted-mistake
# builds this way); it is used as given, never rebuilt.
_LIB = os.environ.get("ORACLE_LIB") or os.path.join(_HERE, "liboracle.so")

WDTYPE_BF16 = 0
WDTYPE_FP8 = 1
WDTYPE_INT4 = 2
WDTYPE_NVFP4 = 3
SCORE_SOFTMAX = 0
SCORE_SIGMOID = 1


def compile_library(out: str, defines=()) -> str:
    """gcc (OpenMP, IEEE float: no fast-math, no FMA contraction) of oracle.c into `out`;
    `defines` are extra -D flags (the mutation tests plant mistakes with ORACLE_MUTANT)."""
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-fno-fast-math",
           "-ffp-contract=off", *[f"-D{d}" for d in defines], "-o", out, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it."""
    if os.environ.get("ORACLE_LIB"):
        return _LIB
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        compile_library(_LIB)
    return _LIB


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        c_i32p = ctypes.POINTER(ctypes.c_int32)
        lib.oracle_e4m3_decode.restype = ctypes.c_double
        lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_encode.restype = ctypes.c_uint8
        lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        lib.oracle_bf16_to_double.restype = ctypes.c_double
        lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
        lib.oracle_swiglu.restype = ctypes.c_double
        lib.oracle_swiglu.argtypes = [ctypes.c_double] * 5
        lib.oracle_quant_1x128.restype = None
        lib.oracle_quant_1x128.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_route.restype = ctypes.c_int
        lib.oracle_route.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                     ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_gate_logits.restype = ctypes.c_int
        lib.oracle_gate_logits.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_void_p]
        lib.oracle_e2m1_decode.restype = ctypes.c_double
        lib.oracle_e2m1_decode.argtypes = [ctypes.c_uint8]
        lib.oracle_fp4_at.restype = ctypes.c_double
        lib.oracle_fp4_at.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_int64]
        lib.oracle_int4_at.restype = ctypes.c_double
        lib.oracle_int4_at.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                       ctypes.c_int64]
        lib.oracle_permute.restype = ctypes.c_int
        lib.oracle_permute.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.oracle_moe_rows.restype = ctypes.c_int
        lib.oracle_moe_rows.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
        lib.oracle_gemm1_rows.restype = ctypes.c_int
        lib.oracle_gemm1_rows.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_int, ctypes.c_void_p]
        lib.oracle_gemm2_rows.restype = ctypes.c_int
        lib.oracle_gemm2_rows.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                          ctypes.c_void_p]
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
        del c_i32p
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


class _Layer(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("k", ctypes.c_int32), ("n_sink", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("wdtype", ctypes.c_int32), ("score", ctypes.c_int32),
                ("pad_", ctypes.c_int32),
                ("alpha", ctypes.c_double), ("beta", ctypes.c_double), ("limit", ctypes.c_double),
                ("route_scale", ctypes.c_double),
                ("logits", ctypes.c_void_p), ("x", ctypes.c_void_p), ("w1", ctypes.c_void_p),
                ("w1_scale", ctypes.c_void_p), ("w2", ctypes.c_void_p), ("w2_scale", ctypes.c_void_p),
                ("gate_scale", ctypes.c_void_p), ("up_scale", ctypes.c_void_p),
                ("limits", ctypes.c_void_p), ("router_bias", ctypes.c_void_p)]


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def e4m3_decode(codes) -> np.ndarray:
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.oracle_e4m3_decode(int(c)) for c in codes.ravel()]).reshape(codes.shape)


def e4m3_encode(values) -> np.ndarray:
    lib = _load()
    v = np.asarray(values, dtype=np.float32)
    return np.array([lib.oracle_e4m3_encode(float(f)) for f in v.ravel()], dtype=np.uint8).reshape(v.shape)


def bf16_to_double(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def swiglu(gate, up, alpha=1.0, beta=0.0, limit=float("inf")):
    lib = _load()
    g = np.asarray(gate, dtype=np.float64)
    u = np.broadcast_to(np.asarray(up, dtype=np.float64), g.shape)
    out = np.empty(g.shape, dtype=np.float64)
    for idx in np.ndindex(g.shape):
        out[idx] = lib.oracle_swiglu(float(g[idx]), float(u[idx]), alpha, beta, limit)
    return out


def quant_1x128(values):
    """values [rows, cols] float32 -> (codes uint8 [rows, cols], scales float32 [rows, cols/128])."""
    v = _c(values, np.float32)
    rows, cols = v.shape
    assert cols % 128 == 0
    q = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty((rows, cols // 128), dtype=np.float32)
    _load().oracle_quant_1x128(_ptr(v), rows, cols, _ptr(q), _ptr(s))
    return q, s


def route(logits, n_routed: int, k: int, score: int, route_scale: float = 1.0, bias=None):
    """logits [T, n_routed + n_sink] float32 (+ optional correction bias float32 [n_routed])
    -> (ids int32 [T,k], w f64 [T,k], shared_w f64 [T,n_sink])."""
    lg = _c(logits, np.float32)
    b = _c(bias, np.float32)
    T, cols = lg.shape
    S = cols - n_routed
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    sw = np.empty((T, max(S, 0)), dtype=np.float64)
    rc = _load().oracle_route(_ptr(lg), _ptr(b), T, n_routed, S, k, score, route_scale, _ptr(ids), _ptr(w),
                              _ptr(sw) if S > 0 else None)
    if rc != 0:
        raise ValueError("oracle_route: invalid arguments")
    return ids, w, sw


def int4_dequant(packed, scale_bits):
    """INT4 group-32 weights: packed uint8 [rows, K/2], bf16 scale bits [rows, K/32] -> fp64 [rows, K]."""
    p = _c(packed, np.uint8)
    s = _c(scale_bits, np.uint16)
    rows, K = p.shape[0], p.shape[1] * 2
    lib = _load()
    out = np.empty((rows, K), dtype=np.float64)
    for r in range(rows):
        for c in range(K):
            out[r, c] = lib.oracle_int4_at(_ptr(p), _ptr(s), K, r, c)
    return out


def e2m1_decode(code: int) -> float:
    return _load().oracle_e2m1_decode(int(code))


def fp4_dequant(packed, scale_codes):
    """NVFP4 weights: packed uint8 [rows, K/2], E4M3 scale codes uint8 [rows, K/16] -> fp64 [rows, K]."""
    p = _c(packed, np.uint8)
    s = _c(scale_codes, np.uint8)
    rows, K = p.shape[0], p.shape[1] * 2
    lib = _load()
    out = np.empty((rows, K), dtype=np.float64)
    for r in range(rows):
        for c in range(K):
            out[r, c] = lib.oracle_fp4_at(_ptr(p), _ptr(s), K, r, c)
    return out


def gate_logits(x_bits, w_bits):
    """Gate GEMV: x bf16 bits [T,H], w bf16 bits [C,H] -> fp64 logits [T,C]."""
    x = _c(x_bits, np.uint16)
    w = _c(w_bits, np.uint16)
    T, H = x.shape
    C = w.shape[0]
    out = np.empty((T, C), dtype=np.float64)
    if _load().oracle_gate_logits(_ptr(x), _ptr(w), T, H, C, _ptr(out)) != 0:
        raise ValueError("oracle_gate_logits: invalid sizes")
    return out


def permute(ids, E: int, n_shared: int = 0):
    """ids int32 [T,k] -> (offsets [E+n_shared+1], perm [A], inv [T,k]) all int32."""
    ids = _c(ids, np.int32)
    T, k = ids.shape
    A = T * k + T * n_shared
    offsets = np.empty(E + n_shared + 1, dtype=np.int32)
    perm = np.empty(A, dtype=np.int32)
    inv = np.empty((T, k), dtype=np.int32)
    rc = _load().oracle_permute(_ptr(ids), T, k, E, n_shared, _ptr(offsets), _ptr(perm), _ptr(inv))
    if rc != 0:
        raise ValueError("oracle_permute: expert id out of range")
    return offsets, perm, inv


class Layer:
    """Host copies of one layer's inputs, in the raw formats the kernels consume.

    x: uint16 bf16 bits [T,H]; logits float32 [T,E+n_sink];
    w1: [G,2I,H] uint16 (bf16 bits) or uint8 (E4M3); w2: [G,H,I] likewise;
    w1_scale [G,2I/128,H/128] and w2_scale [G,H/128,I/128] float32 for E4M3;
    gate_scale / up_scale float32 [G] or None; limits float32 [G] (a clamp per
    expert) or None; router_bias float32 [E] or None.
    """

    def __init__(self, *, T, H, I, E, k, n_sink, n_shared, wdtype, score, alpha, beta, limit,
                 route_scale, logits, x, w1, w2, w1_scale=None, w2_scale=None,
                 gate_scale=None, up_scale=None, limits=None, router_bias=None):
        wt = np.uint16 if wdtype == WDTYPE_BF16 else np.uint8
        # INT4 group scales are bf16 bits, NVFP4 block scales E4M3 codes
        st = {WDTYPE_INT4: np.uint16, WDTYPE_NVFP4: np.uint8}.get(wdtype, np.float32)
        self._keep = dict(
            logits=_c(logits, np.float32), x=_c(x, np.uint16), w1=_c(w1, wt), w2=_c(w2, wt),
            w1_scale=_c(w1_scale, st), w2_scale=_c(w2_scale, st),
            gate_scale=_c(gate_scale, np.float32), up_scale=_c(up_scale, np.float32),
            limits=_c(limits, np.float32), router_bias=_c(router_bias, np.float32))
        k_ = self._keep
        self.dims = dict(T=T, H=H, I=I, E=E, k=k, n_sink=n_sink, n_shared=n_shared,
                         wdtype=wdtype, score=score)
        self.s = _Layer(T, H, I, E, k, n_sink, n_shared, wdtype, score, 0,
                        float(alpha), float(beta), float(limit), float(route_scale),
                        _ptr(k_["logits"]), _ptr(k_["x"]), _ptr(k_["w1"]), _ptr(k_["w1_scale"]),
                        _ptr(k_["w2"]), _ptr(k_["w2_scale"]), _ptr(k_["gate_scale"]),
                        _ptr(k_["up_scale"]), _ptr(k_["limits"]), _ptr(k_["router_bias"]))

    def moe_rows(self, tokens) -> np.ndarray:
        tok = _c(tokens, np.int32)
        out = np.empty((len(tok), self.dims["H"]), dtype=np.float64)
        rc = _load().oracle_moe_rows(ctypes.byref(self.s), _ptr(tok), len(tok), _ptr(out))
        if rc != 0:
            raise ValueError("oracle_moe_rows: invalid arguments")
        return out

    def gemm1_rows(self, A, xp, xs, rows, row_expert) -> np.ndarray:
        rows = _c(rows, np.int32)
        row_expert = _c(row_expert, np.int32)
        xp = np.ascontiguousarray(xp)
        xs = _c(xs, np.float32)
        h = np.empty((len(rows), self.dims["I"]), dtype=np.float64)
        rc = _load().oracle_gemm1_rows(ctypes.byref(self.s), int(A), _ptr(xp), _ptr(xs), _ptr(rows),
                                       _ptr(row_expert), len(rows), _ptr(h))
        if rc != 0:
            raise ValueError("oracle_gemm1_rows: invalid arguments")
        return h

    def gemm2_rows(self, A, hp, hs, offsets, inv, row_w, tokens) -> np.ndarray:
        tok = _c(tokens, np.int32)
        hp = np.ascontiguousarray(hp)
        out = np.empty((len(tok), self.dims["H"]), dtype=np.float64)
        rc = _load().oracle_gemm2_rows(ctypes.byref(self.s), int(A), _ptr(hp), _ptr(_c(hs, np.float32)),
                                       _ptr(_c(offsets, np.int32)), _ptr(_c(inv, np.int32)),
                                       _ptr(_c(row_w, np.float32)), _ptr(tok), len(tok), _ptr(out))
        if rc != 0:
            raise ValueError("oracle_gemm2_rows: invalid arguments")
        return out
