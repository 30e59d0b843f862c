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
