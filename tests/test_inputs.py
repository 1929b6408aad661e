"""The seeded input generator: deterministic, right shapes, and the long_skewed
bias gives expert 0 about 40% of the slots (fixture written by the oracle-only
calibration script)."""
import json
import os

import torch

from workloads import (CONFIGS, LONG_SKEWED_BETA, bias_vector, make_inputs, small_case,
                       worked_example_a)


def test_deterministic_and_shapes():
    a = small_case("s", T=37, d=64, E=5, k=2, F=128, act="swiglu")
    b = small_case("s", T=37, d=64, E=5, k=2, F=128, act="swiglu")
    assert a.x.dtype == torch.bfloat16 and a.x.shape == (37, 64)
    assert a.w1.shape == (5, 64, 128) and a.w3.shape == (5, 64, 128) and a.w2.shape == (5, 128, 64)
    for t in ("x", "wg", "w1", "w3", "w2"):
        assert torch.equal(getattr(a, t), getattr(b, t))
    c = small_case("s", T=37, d=64, E=5, k=2, F=128, act="swiglu", seed=8)
    assert not torch.equal(a.x, c.x)


def test_bias_recipes():
    b = bias_vector(CONFIGS["capacity_skew"])
    assert b.shape == (64,) and b[0] == 0.0 and b[1] < b[0] and torch.all(b[1:] < b[:-1])
    b5 = bias_vector(CONFIGS["long_skewed"])
    assert b5[0] == LONG_SKEWED_BETA and torch.all(b5[1:] == 0)
    assert bias_vector(CONFIGS["mixtral"]) is None


def test_long_skewed_fixture_matches_constant():
    with open(os.path.join(os.path.dirname(__file__), "golden", "long_skewed_bias.json")) as f:
        g = json.load(f)
    assert g["beta"] == LONG_SKEWED_BETA
    assert 0.39 <= g["expert0_share"] <= 0.41


def test_worked_example_a_shape():
    a = worked_example_a()
    assert a.x.shape == (8, 4) and a.extra["ids"] == [2, 0, 2, 3, 0, 2, 0, 2]


def test_tiny_config_draws():
    inp = make_inputs(CONFIGS["tiny_fp32"])
    assert inp.x.dtype == torch.float32 and inp.w1.shape == (4, 64, 128)
    assert 0.05 < float(inp.w1.std()) < 0.15
