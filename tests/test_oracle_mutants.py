"""Mutation checks of the oracle's pins (CPU only). Each case builds oracle.c with one
planted, plausible mistake (-DORACLE_MUTANT=n: a flipped tie rule, sigma carried out of the
top-k loop instead of the raw logit, a dropped clamp, a wrong sign, a transposed operand,
...) and runs the pin named for it in a child process that loads that build (ORACLE_LIB);
the pin must fail. The pins themselves pass on the normal build (test_oracle_pins.py)."""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PINS = os.path.join("tests", "test_oracle_pins.py")

MUTANTS = [
    (1, "equal keys go to the higher expert id", "test_route_selection_brute_force_with_ties"),
    (2, "sigmoid(logit) carried out of the top-k loop instead of the raw logit",
     "test_route_softmax_weights_match_torch_softmax"),
    (3, "gate not clamped at L", "test_swiglu_clamp_boundaries"),
    (4, "up not clamped from below at -L", "test_swiglu_clamp_boundaries"),
    (5, "sigmoid of -alpha*g instead of alpha*g", "test_swiglu_standard_reduces_to_silu_times_up"),
    (6, "up bias beta dropped", "test_swiglu_alpha_beta_identities"),
    (7, "sink columns left out of the logsumexp", "test_route_sigmoid_weights_are_sigma_ratios"),
    (8, "softmax renormalised over every column, not the selected k",
     "test_route_softmax_weights_match_torch_softmax"),
    (9, "rows of an expert in reverse token order", "test_permute_brute_force"),
    (10, "E4M3 ties rounded to the larger code, not the even one", "test_e4m3_encode_ties_to_even_and_saturation"),
    (11, "activation scale amax/240 instead of amax/448", "test_quant_1x128_block_properties"),
    (12, "FP8 weight block scale dropped", "test_layer_fp8_matches_torch_e4m3_composition"),
    (13, "INT4 nibbles in the wrong order", "test_int4_dequant_follows_the_nibble_order_and_group_scale"),
    (14, "shared expert weighted 1 instead of its sink weight",
     "test_layer_sink_gated_shared_experts_use_sink_weights"),
    (15, "route_scale not applied", "test_layer_expert_relabelling_and_scale_linearity"),
    (16, "per-expert clamp ignored", "test_layer_per_expert_limits_clamp_each_expert_with_its_own_value"),
    (17, "gate and up scales swapped", "test_layer_expert_relabelling_and_scale_linearity"),
    (18, "W2 read transposed", "test_layer_single_expert_is_dense_swiglu_mlp"),
    (19, "gate and up halves of W1 swapped", "test_layer_single_expert_is_dense_swiglu_mlp"),
    (20, "correction bias added to the weights, not only the ranking",
     "test_route_dominant_bias_forces_the_selection_and_not_the_weights"),
    (21, "E2M1 exponent bias 2 instead of 1", "test_e2m1_decode_all_codes_match_ml_dtypes"),
    (22, "NVFP4 block scale per 32 weights instead of 16", "test_fp4_dequant_follows_the_nibble_order_and_block_scale"),
]


@pytest.fixture(scope="module")
def verdicts(tmp_path_factory):
    """Builds every mutant and runs each one's pin in a child process, six at a time;
    returns {n: (exit code, output)}."""
    import concurrent.futures as cf
    d = tmp_path_factory.mktemp("mutants")

    def run(case):
        n, _, pin = case
        lib = oracle.compile_library(str(d / f"liboracle_m{n}.so"), defines=[f"ORACLE_MUTANT={n}"])
        env = dict(os.environ, ORACLE_LIB=lib, OMP_NUM_THREADS="2")
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                            f"{PINS}::{pin}"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
        return n, (r.returncode, r.stdout[-3000:] + r.stderr[-2000:])

    with cf.ThreadPoolExecutor(max_workers=6) as ex:
        return dict(ex.map(run, MUTANTS))


@pytest.mark.parametrize("n,what,pin", MUTANTS, ids=[f"m{m[0]}" for m in MUTANTS])
def test_pin_catches_the_planted_mistake(n, what, pin, verdicts):
    code, out = verdicts[n]
    # exit code 1: the collected tests ran and at least one failed (2+ would be an error)
    assert code == 1, f"mutant {n} ({what}) not caught by {pin}:\n{out}"
