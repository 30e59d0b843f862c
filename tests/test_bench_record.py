"""The bench's link to the committed ncu capture (CPU): the traffic record is keyed on the
grouped-GEMM kernel's code without comments, so a comment edit keeps the captured
counters and any code edit retires them."""
import importlib.util
import json
import os

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_record", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_comments_are_stripped_but_literals_are_kept():
    b = _bench()
    src = 'int a = 1; // note\n/* block\n comment */ const char* s = "x // y /* z */"; char q = \'"\';\n'
    assert b.strip_comments(src) == 'int a = 1; const char* s = "x // y /* z */"; char q = \'"\';'
    assert b.strip_comments("a  =\n\tb; // c") == b.strip_comments("a = b;")
    assert b.strip_comments("a = b;") != b.strip_comments("a = c;")


def test_the_committed_record_is_used_only_while_the_kernel_code_matches():
    """traffic.json's counters are reported while the kernel's code (comments aside) is the
    captured code, and retired (null) as soon as it differs."""
    b = _bench()
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    assert tuple(rec["kernel_code_files"]) == b.KERNEL_SOURCES
    assert rec["workloads"] and all(isinstance(v, int) and v > 0 for v in rec["workloads"].values())
    same = rec["kernel_code_sha1"] == b.kernel_code_digest()
    for w, v in rec["workloads"].items():
        assert b.profiled_traffic(w) == (v if same else None)
    assert b.profiled_traffic("no_such_workload") is None


def test_kernel_work_counts_touched_experts_once():
    """The roofline's algorithmic work, against hand counts: FLOPs 6*A*H*I (GEMM1 2*A*H*2I
    plus GEMM2 2*A*I*H), bytes = each touched group's W1 and W2 read once (plus FP8
    block scales), empty groups not counted; the implementation's intermediates apart."""
    import numpy as np
    from grouped_gemm_swiglu_b200 import workloads as W
    b = _bench()
    glm = W.WORKLOADS["glm_fp8"]  # E4M3 weights, 128x128 fp32 block scales
    G = glm.E + glm.n_shared
    A = glm.T * (glm.k + glm.n_shared)
    off = np.linspace(0, A, G + 1).astype(np.int64)  # every group holds rows
    flops, wb, ib = b.kernel_work(glm, off)
    H, I = glm.H, glm.I
    assert flops == 6.0 * A * H * I == 2783138807808.0
    per_expert = 3 * I * H + (2 * I // 128 * H // 128 + H // 128 * I // 128) * 4
    assert wb == G * per_expert == 5456024064
    assert ib == A * H + 2 * A * I + A * H * 2 + A * (H // 128 + 2 * (I // 128)) * 4
    # three empty groups: their weights are not algorithmic bytes; the rows are unchanged
    sizes = np.diff(off)
    sizes[[3, 17, 200]] = 0
    sizes[0] += A - sizes.sum()
    off2 = np.concatenate([[0], np.cumsum(sizes)])
    f2, wb2, ib2 = b.kernel_work(glm, off2)
    assert (f2, ib2) == (flops, ib) and wb2 == (G - 3) * per_expert
    # bf16 and INT4 group-32 weights: 2 bytes, and half a byte plus a bf16 scale per 32
    q = W.WORKLOADS["qwen3_30b_a3b"]
    Aq = q.T * q.k
    offq = np.linspace(0, Aq, q.E + 1).astype(np.int64)
    fq, wq, iq = b.kernel_work(q, offq)
    assert wq == q.E * 3 * q.I * q.H * 2 and iq == Aq * q.H * 2 + 2 * Aq * q.I * 2 + Aq * q.H * 2
    d4 = W.WORKLOADS["decode_t1_int4"]
    G4 = d4.E + d4.n_shared
    off4 = np.zeros(G4 + 1, np.int64)
    off4[1:] = np.minimum(np.arange(1, G4 + 1), d4.T * (d4.k + d4.n_shared))  # the first 10 groups, one row each
    f4, w4, _ = b.kernel_work(d4, off4)
    assert w4 == 10 * 3 * d4.I * d4.H * (0.5 + 2 / 32) and f4 == 6.0 * 10 * d4.H * d4.I
