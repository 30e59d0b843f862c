"""The C ABI library on the host (CPU only): it builds, loads, exports every function the
header declares, and rejects bad arguments before touching a GPU."""
import ctypes
import math

import pytest

import grouped_gemm_swiglu_b200 as moe
from grouped_gemm_swiglu_b200 import build as B
from grouped_gemm_swiglu_b200 import workloads as W


@pytest.fixture(scope="module")
def L():
    B.build()
    return moe.lib()


def test_every_header_function_is_exported(L):
    names = moe.header_functions()
    assert set(names) >= {"moe_route_topk", "moe_permute", "moe_gemm1_swiglu", "moe_gemm2_combine", "moe_forward",
                          "moe_workspace_size", "moe_status_string", "moe_abi_version", "moe_read_status",
                          "moe_clear_status"}
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/moe_b200.h but not exported"


def test_version_and_status_strings(L):
    assert moe.moe_abi_version() == 7
    for code in range(-7, 1):
        assert moe.status_string(code)
    assert "unknown" in moe.status_string(-99)


def _dims(**kw):
    d = moe.MoeDims.of(W.WORKLOADS["tiny"])
    for k, v in kw.items():
        setattr(d, k, v)
    return d


@pytest.mark.parametrize("bad", [dict(H=200), dict(I=64), dict(E=0), dict(E=2000), dict(k=0), dict(k=9),
                                 dict(k=33, E=64), dict(n_sink=1, score=moe.MOE_SCORE_SOFTMAX),
                                 dict(n_sink=2, n_shared=1, score=moe.MOE_SCORE_SIGMOID), dict(T=-1),
                                 dict(limit=0.0), dict(limit=float("nan")), dict(alpha=float("inf")),
                                 dict(wdtype=4), dict(wdtype=5), dict(score=3),
                                 dict(k=8, n_sink=25, score=moe.MOE_SCORE_SIGMOID)])
def test_invalid_dims_rejected(L, bad):
    d = _dims(**bad)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_workspace_size(d, moe.MOE_WS_FORWARD)
    assert ei.value.status == -1
    # the entry points reject the same dims before any CUDA call
    assert L.moe_route_topk(None, ctypes.byref(d), None, None, None, None, None, None) == -1


def test_null_pointers_and_small_workspace_rejected(L):
    d = _dims()
    assert L.moe_route_topk(None, ctypes.byref(d), None, None, None, None, None, None) == -1
    assert L.moe_forward(*([None] * 10), ctypes.byref(d), None, None, None, None, None, None, 0, None) == -1
    fake = 1 << 20  # never dereferenced: the checks fail first
    n = moe.moe_workspace_size(d, moe.MOE_WS_PERMUTE)
    rc = L.moe_permute(fake, fake, ctypes.byref(d), fake, fake, fake, fake, None, fake, n - 1, None)
    assert rc == -4
    rc = L.moe_permute(fake, fake, ctypes.byref(d), fake, fake, fake, fake, None, fake + 8, n, None)
    assert rc == -4  # misaligned workspace
    rc = L.moe_permute(fake, fake + 2, ctypes.byref(d), fake, fake, fake, fake, None, fake, n, None)
    assert rc == -1  # x not 16-byte aligned
    # sink weights pointer must match n_sink
    rc = L.moe_route_topk(fake, ctypes.byref(d), None, fake, fake, fake, None, None)
    assert rc == -1


@pytest.mark.parametrize("args", [
    (-1, 8, 0, 0, 4),     # negative row count
    (16, 0, 0, 0, 1),     # no routed experts
    (16, 8, -1, 0, 4),    # negative shared count
    (16, 8, 0, -1, 4),    # negative local offset
    (16, 8, 0, 4, 5),     # local range past E
    (16, 8, 0, 0, 0),     # no local experts
    (16, 2000, 0, 0, 4),  # E beyond the library's limit
])
def test_ep_rebase_rejects_bad_ranges(L, args):
    n, E, n_shared, off, n_local = args
    fake = 1 << 20  # never dereferenced: the checks fail first
    assert L.moe_ep_rebase(fake, n, E, n_shared, off, n_local, fake, None) == -1


def test_ep_calls_reject_null_pointers(L):
    d = _dims()
    assert L.moe_ep_rebase(None, 16, 8, 0, 0, 4, None, None) == -1
    assert L.moe_ep_row_ids(None, ctypes.byref(d), None, None) == -1
    bad = _dims(k=0)
    assert L.moe_ep_row_ids(1 << 20, ctypes.byref(bad), 1 << 20, None) == -1


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_workspace_sizes_cover_the_intermediates(L, name):
    wl = W.WORKLOADS[name]
    d = moe.MoeDims.of(wl)
    A, H, I = d.A, d.H, d.I
    elt = 1 if wl.wdtype == W.WDTYPE_FP8 else 2
    fwd = moe.moe_workspace_size(d, moe.MOE_WS_FORWARD)
    need = A * H * elt + A * I * elt + A * H * 2  # x_perm, h, y
    if elt == 1:
        need += (H // 128 + I // 128) * A * 4
    assert fwd >= need + 256
    assert fwd % 256 == 0
    assert moe.moe_workspace_size(d, moe.MOE_WS_GEMM1) >= 256
    assert moe.moe_workspace_size(d, moe.MOE_WS_GEMM2_COMBINE) >= A * H * 2
    assert moe.moe_workspace_size(d, moe.MOE_WS_PERMUTE) >= d.T * d.k * 4


def test_no_clamp_is_infinite_limit():
    d = moe.MoeDims.of(W.WORKLOADS["tiny"])
    assert math.isinf(d.limit) and d.limit > 0
    assert moe.MoeDims.of(W.WORKLOADS["oai_swiglu"]).limit == pytest.approx(7.0)


def test_router_bias_needs_sigmoid_scoring(L):
    """A correction bias is defined for the sigmoid ranking only: rejected before any CUDA call."""
    fake = 1 << 20
    d = _dims(score=moe.MOE_SCORE_SOFTMAX, n_sink=0)
    assert L.moe_route_topk(fake, ctypes.byref(d), fake, fake, fake, None, None, None) == -2
    ws_n = moe.moe_workspace_size(d, moe.MOE_WS_FORWARD)
    assert L.moe_forward(fake, fake, fake, fake, None, None, None, None, fake, None, ctypes.byref(d), fake,
                         None, None, None, None, fake, ws_n, None) == -2


def test_gate_route_checks(L):
    """The fused gate GEMV + router takes T <= 16 and sizes its workspace for the logits."""
    fake = 1 << 20
    d = _dims(T=17)
    n = moe.moe_workspace_size(d, moe.MOE_WS_GATE_ROUTE)
    assert n >= 256 + 17 * (d.E + d.n_sink) * 4
    assert L.moe_gate_route(fake, fake, ctypes.byref(d), None, None, fake, fake, None, None, fake, n, None) == -2
    d = _dims(T=4)
    assert L.moe_gate_route(fake, fake + 8, ctypes.byref(d), None, None, fake, fake, None, None, fake, n,
                            None) == -1  # w_gate not 16-byte aligned


@pytest.mark.parametrize("wdtype", [moe.MOE_WDTYPE_INT4_G32, moe.MOE_WDTYPE_NVFP4])
def test_4bit_weights_need_aligned_scales(L, wdtype):
    """INT4 and NVFP4 layers size their workspaces like bf16 ones (bf16 activations) and
    reject a missing or misaligned scale array before any CUDA call."""
    d = _dims(wdtype=wdtype)
    assert moe.moe_workspace_size(d, moe.MOE_WS_GEMM1) == moe.moe_workspace_size(_dims(), moe.MOE_WS_GEMM1)
    fake = 1 << 20
    n = moe.moe_workspace_size(d, moe.MOE_WS_GEMM1)
    # x_perm, x_scale, offsets, w1, w1_scale, gate_scale, up_scale, limits, dims, h, h_scale, ws, ws_bytes, stream
    assert L.moe_gemm1_swiglu(fake, None, fake, fake, None, None, None, None, ctypes.byref(d), fake, None, fake, n,
                              None) == -1
    assert L.moe_gemm1_swiglu(fake, None, fake, fake, fake + 2, None, None, None, ctypes.byref(d), fake, None, fake,
                              n, None) == -1


def _noalloc(L):
    fn = L.moe_permute_noalloc
    fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(moe.MoeDims)] + [ctypes.c_void_p] * 7
    fn.restype = ctypes.c_int
    return fn


def test_noalloc_size_limit_is_where_the_header_says(L):
    """The static scratch holds 1 MiB - 256 bytes of counts and ranks; at k = 8, E = 288
    the first size that does not fit is T = 28689. The refusal comes before any CUDA call,
    so fake (never dereferenced) pointers are enough here; T = 28688 runs on the GPU."""
    al = lambda b: (b + 255) & ~255
    need = lambda T: al(((T + 255) // 256) * 288 * 4) + al(T * 8 * 4)
    assert need(28688) <= (1 << 20) - 256 < need(28689)
    fake = 1 << 20
    for wd in (0, 1, 2, 3):  # the four weight types are accepted alike
        d = _dims(T=28689, H=512, E=288, k=8, n_shared=1, n_sink=0, wdtype=wd, score=moe.MOE_SCORE_SIGMOID)
        assert _noalloc(L)(fake, fake, ctypes.byref(d), fake, fake, fake, fake, fake, None, None) == -4
    d = _dims(T=28689, H=512, E=288, k=8, n_shared=1, n_sink=0, wdtype=4)
    assert _noalloc(L)(fake, fake, ctypes.byref(d), fake, fake, fake, fake, fake, None, None) == -1


def test_set_option_returns_the_previous_value_and_rejects_unknown_ones(L):
    """moe_set_option is host-only: it never touches a GPU."""
    old = moe.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, 1)
    try:
        assert old in (0, 1)
        assert moe.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, 0) == 1
        assert moe.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, 0) == 0
        assert L.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, 2) == -1
        assert L.moe_set_option(99, 0) == -1
        assert moe.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, 0) == 0  # the refusals changed nothing
    finally:
        moe.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, old)
    old_b = moe.moe_set_option(moe.MOE_OPT_BF16_CTA_PAIR, 1)
    try:  # the two options are independent
        assert old_b in (0, 1)
        assert moe.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, old) == old
        assert moe.moe_set_option(moe.MOE_OPT_BF16_CTA_PAIR, 0) == 1
        assert L.moe_set_option(moe.MOE_OPT_BF16_CTA_PAIR, -1) == -1
        assert moe.moe_set_option(moe.MOE_OPT_BF16_CTA_PAIR, 0) == 0
    finally:
        moe.moe_set_option(moe.MOE_OPT_BF16_CTA_PAIR, old_b)


@pytest.mark.parametrize("name", ["qwen3_30b_a3b", "glm_fp8", "oai_swiglu", "decode_t64"])
def test_layout_options_need_no_other_workspace(L, name):
    """The CTA-pair layouts run inside the workspace sized without them (their second
    GEMM1 completion counter per 256-row block fits the block flags; otherwise the
    single-CTA tile runs): moe_workspace_size does not depend on the options."""
    d = moe.MoeDims.of(W.WORKLOADS[name])
    kinds = [moe.MOE_WS_FORWARD, moe.MOE_WS_EXPERTS, moe.MOE_WS_GEMM1, moe.MOE_WS_GEMM2_COMBINE]
    base = [moe.moe_workspace_size(d, k) for k in kinds]
    old = (moe.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, 1), moe.moe_set_option(moe.MOE_OPT_BF16_CTA_PAIR, 1))
    try:
        assert [moe.moe_workspace_size(d, k) for k in kinds] == base
    finally:
        moe.moe_set_option(moe.MOE_OPT_FP8_CTA_PAIR, old[0])
        moe.moe_set_option(moe.MOE_OPT_BF16_CTA_PAIR, old[1])
