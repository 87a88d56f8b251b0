"""The oracle's pins catch planted mistakes.

Each case rebuilds the C oracle with one deliberate mistake (a dropped bias,
a reversed code order, a sign flip, a transposed operand, ...) and checks that
at least one of the listed pin tests fails against it.  CPU only.
"""
import pytest

import oracle as O
import importlib

OB = importlib.import_module("oracle.build")
import test_oracle_pins as P

MUTANTS = {
    1: ("dequant drops the bias", [P.test_hand_packed_dequant]),
    2: ("codes read in reversed order", [P.test_hand_packed_dequant]),
    3: ("silu sign flipped", [P.test_expert_ffn_matches_numpy, P.test_expert_ffn_hand_worked]),
    4: ("ties go to the higher index", [P.test_topk_bruteforce_with_ties]),
    5: ("residual dropped", [P.test_one_hot_routing_is_single_expert]),
    6: ("eps added outside the square root", [P.test_rmsnorm_closed_form]),
    7: ("scale divides by 2^b instead of 2^b - 1", [P.test_quantizer_picks_nearest_code]),
    8: ("shared down projection transposed", [P.test_shared_ffn_matches_numpy, P.test_shared_ffn_hand_worked]),
    9: ("gate and up swapped in SwiGLU", [P.test_expert_ffn_matches_numpy, P.test_expert_ffn_hand_worked]),
    10: ("router reads Wr transposed", [P.test_router_hand_worked]),
    11: ("router drops the bias", [P.test_router_hand_worked]),
    12: ("silu replaced by the plain sigmoid", [P.test_expert_ffn_hand_worked, P.test_shared_ffn_hand_worked]),
    13: ("pre-norm divides by the sum, not the mean", [P.test_prenorm_hand_worked, P.test_prenorm_closed_forms]),
    14: ("pre-norm drops gamma", [P.test_prenorm_hand_worked, P.test_prenorm_closed_forms]),
    15: ("shared gate uses silu, not the sigmoid", [P.test_shared_gate_closed_forms]),
    16: ("shared gate ignored", [P.test_shared_gate_closed_forms]),
    17: ("packed shared expert ignored for the bf16 weights", [P.test_packed_shared_is_an_expert]),
}


def _run_pin(fn):
    import inspect
    params = inspect.signature(fn).parameters
    if "case" in params:
        for case in P._hand_cases():
            fn(case)
    elif "bits" in params:
        for bits in (4, 2):
            fn(bits)
    else:
        fn()


@pytest.mark.parametrize("n", sorted(MUTANTS))
def test_pins_catch_planted_mistake(n, tmp_path):
    what, pins = MUTANTS[n]
    path = OB.build_mutant(n, str(tmp_path))
    prev = O.oracle.use_library(path)
    try:
        caught = 0
        for fn in pins:
            try:
                _run_pin(fn)
            except AssertionError:
                caught += 1
        assert caught == len(pins), "planted mistake not caught by every listed pin: " + what
    finally:
        O.oracle.restore_library(prev)


def test_unmutated_oracle_passes_same_pins():
    for _, pins in MUTANTS.values():
        for fn in pins:
            _run_pin(fn)
