"""Depth auto-tune measured on the GPU (small head, few steps)."""
import pytest

from verify_step_lm_b200 import synth, tune

pytestmark = pytest.mark.gpu


def test_tune_table_and_choice():
    W = synth.make_head(4096, 512, 0.05, seed=12345, device="cuda")
    Wq, S = synth.quantize_int4_g64(W)
    res = tune.measure(W, Wq, S, [1, 2, 3], 0.6, 0.95, 0.3, steps=8, warmup=2)
    rows = res["depths"]
    assert sorted(rows) == [1, 2, 3]
    for K, r in rows.items():
        assert 0.0 <= r["mean_accepted"] <= K
        assert r["draft_ms"] > 0 and r["verify_ms"] > 0
        assert r["tokens_per_cycle"] == pytest.approx(r["mean_accepted"] + 1.0)
    table = {K: {"tokens_per_cycle": r["tokens_per_cycle"], "cycle_ms": r["cycle_ms"]}
             for K, r in rows.items()}
    table[0] = {"tokens_per_cycle": 1.0, "cycle_ms": res["ar"]["cycle_ms"]}
    best = max(table, key=lambda k: tune.throughput(table[k]["tokens_per_cycle"], table[k]["cycle_ms"]))
    assert res["choice"] == best


def test_identical_draft_head_accepts_everything():
    # sigma = 0: the draft rows equal the target rows; with the bf16 head's
    # int4 copy the draft distribution differs a little, so most (not all)
    # drafts are accepted
    W = synth.make_head(4096, 512, 0.05, seed=12345, device="cuda")
    Wq, S = synth.quantize_int4_g64(W)
    res = tune.measure(W, Wq, S, [3], 0.6, 0.95, 0.0, steps=8, warmup=1)
    assert res["depths"][3]["acceptance_rate"] > 0.5
