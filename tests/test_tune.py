"""Depth auto-tune: the decision rule (host logic, no GPU)."""
import itertools

import pytest

from verify_step_lm_b200 import tune


@pytest.mark.parametrize("alpha", [0.0, 0.3, 0.75, 0.999, 1.0])
@pytest.mark.parametrize("K", [1, 2, 3, 5])
def test_expected_tokens_matches_enumeration(alpha, K):
    # enumerate accept/reject outcomes of the K drafts; emission stops at the
    # first rejection (n accepted drafts + one token from the target)
    total = 0.0
    for outcome in itertools.product([True, False], repeat=K):
        p = 1.0
        for a in outcome:
            p *= alpha if a else 1.0 - alpha
        n = next((i for i, a in enumerate(outcome) if not a), K)
        total += p * (n + 1)
    assert tune.expected_tokens_constant(alpha, K) == pytest.approx(total, rel=1e-12, abs=1e-12)


def test_choose_depth_takes_the_fastest():
    table = {0: {"tokens_per_cycle": 1.0, "cycle_ms": 0.30},
             1: {"tokens_per_cycle": 1.8, "cycle_ms": 0.50},
             2: {"tokens_per_cycle": 2.4, "cycle_ms": 0.60},
             3: {"tokens_per_cycle": 2.7, "cycle_ms": 0.75}}
    # tokens/s: 3333, 3600, 4000, 3600
    assert tune.choose_depth(table) == 2


def test_choose_depth_turns_drafting_off_when_it_does_not_pay():
    table = {0: {"tokens_per_cycle": 1.0, "cycle_ms": 0.25},
             1: {"tokens_per_cycle": 1.2, "cycle_ms": 0.45},
             3: {"tokens_per_cycle": 1.5, "cycle_ms": 0.70}}
    assert tune.choose_depth(table) == 0


def test_choose_depth_ties_go_to_the_smaller_depth():
    table = {0: {"tokens_per_cycle": 1.0, "cycle_ms": 0.5},
             2: {"tokens_per_cycle": 2.0, "cycle_ms": 1.0}}
    assert tune.choose_depth(table) == 0


def test_decide_adds_the_body_to_every_cycle():
    res = {"depths": {2: {"tokens_per_cycle": 2.5, "cycle_ms": 0.75}},
           "ar": {"tokens_per_cycle": 1.0, "cycle_ms": 0.28}}
    assert tune.decide(res, 0.0)["choice"] == 0          # heads only: drafting does not pay
    d = tune.decide(res, 2.0)                            # a 2 ms body per pass: it does
    assert d["choice"] == 2
    assert d["tokens_per_s"][0] == pytest.approx(1e3 / 2.28)
    assert d["tokens_per_s"][2] == pytest.approx(1e3 * 2.5 / 2.75)
