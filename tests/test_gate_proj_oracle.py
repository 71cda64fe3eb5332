"""Pins for the five-gate projection oracle (Muir review §2.3).

What the page fixes: the gate order and ranks, the 2 d R_tot parameter count
(printed 2.10M at d = 2048) and the FFN width it frees; what the mathematics
fixes: a low-rank product equals the dense product of its factors, and the
activations' ranges and limits, with the logistic taken from scipy.
"""
import json
import os

import numpy as np
import pytest
from scipy.special import expit

from oracle import gate_proj as gp

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "gate_projection_budget.json")


def _rand(N=37, d=256, ranks=gp.RANKS, seed=0):
    r = np.random.default_rng(seed)
    R = sum(ranks)
    return (r.standard_normal((N, d)), r.standard_normal((d, R)) / np.sqrt(d),
            r.standard_normal((R, d)) / 8.0, r.standard_normal((5, d)))


def test_budget_matches_the_printed_figures():
    with open(GOLDEN) as f:
        g = json.load(f)
    assert tuple(g["ranks"]) == gp.RANKS and gp.GATES == ("f", "b", "g", "w", "q")
    n = gp.parameter_count(g["d"])
    assert round(n / 1e6, 2) == g["muir_params_millions"]
    assert 4 * g["d"] - sum(gp.RANKS) == g["muir_ffn_width"]
    # the same 12 d^2 budget rule gives GDN-2's printed FFN width from its printed gate parameters
    r_gdn2 = g["gdn2_params_millions"] * 1e6 / (2 * g["d"])
    assert abs(4 * g["d"] - r_gdn2 - g["gdn2_ffn_width"]) < 0.01 * g["d"]


def test_low_rank_logits_equal_the_dense_product_of_the_factors():
    x, wd, wu, bias = _rand()
    lg = gp.logits(x, wd, wu, bias)
    off = 0
    for i, (name, r) in enumerate(zip(gp.GATES, gp.RANKS)):
        dense = wd[:, off:off + r] @ wu[off:off + r]          # d x d, formed first
        want = x @ dense + bias[i]
        assert np.max(np.abs(lg[name] - want)) <= 1e-12 * np.max(np.abs(want))
        off += r


def test_each_gate_reads_only_its_own_code_block():
    """Weights that are zero outside one gate's block leave every other gate at its bias."""
    x, wd, wu, bias = _rand(seed=1)
    off = 0
    for i, (name, r) in enumerate(zip(gp.GATES, gp.RANKS)):
        wu_one = np.zeros_like(wu)
        wu_one[off:off + r] = wu[off:off + r]
        lg = gp.logits(x, wd, wu_one, bias)
        for j, other in enumerate(gp.GATES):
            if other != name:
                assert np.array_equal(lg[other], np.broadcast_to(bias[j], lg[other].shape))
        assert np.max(np.abs(lg[name] - bias[i])) > 0.1
        off += r


def test_activation_ranges_and_limits():
    v = np.linspace(-40.0, 40.0, 2001)[None, :]
    a = gp.activate({k: v for k in gp.GATES})
    s = expit(v)
    assert np.max(np.abs(a["b"] - 2 * s)) < 1e-15 and np.max(np.abs(a["g"] - s)) < 1e-15
    assert np.array_equal(a["g"], a["w"]) and np.array_equal(a["z"], v)
    assert np.max(np.abs(np.exp(a["log_alpha"]) - s)) < 1e-15          # alpha = sigmoid(f)
    assert np.all(a["log_alpha"] < 0) and np.all((a["b"] > 0) & (a["b"] < 2) | (np.abs(v) > 36))
    mid = v.shape[1] // 2                                                # logit 0
    assert a["b"][0, mid] == 1.0 and a["g"][0, mid] == 0.5 and abs(a["log_alpha"][0, mid] + np.log(2)) < 1e-15
    assert abs(a["log_alpha"][0, 0] + 40.0) < 1e-15                    # log sigmoid(-40) ~ -40
    assert -1e-17 < a["log_alpha"][0, -1] < 0                            # log sigmoid(40) ~ -4e-18


@pytest.mark.parametrize("mutant", ["swap_gates", "no_bias", "sigmoid_for_b", "alpha_not_log"])
def test_planted_mistakes_fail_a_pin(mutant):
    """Each planted mistake in a copy of the oracle is caught by one of the checks above."""
    x, wd, wu, bias = _rand(seed=2)
    lg = gp.logits(x, wd, wu, bias)
    a = gp.activate(lg)
    if mutant == "swap_gates":                       # g and w up-projections swapped
        bad = dict(lg)
        bad["g"], bad["w"] = lg["w"], lg["g"]
        off = 64 + 64
        dense_g = wd[:, off:off + 128] @ wu[off:off + 128]
        assert np.max(np.abs(bad["g"] - (x @ dense_g + bias[2]))) > 1e-3
    elif mutant == "no_bias":
        bad = lg["f"] - bias[0]
        assert np.max(np.abs(bad - (x @ (wd[:, :64] @ wu[:64]) + bias[0]))) > 1e-3
    elif mutant == "sigmoid_for_b":
        assert np.max(np.abs(expit(lg["b"]) - 2 * expit(lg["b"]))) > 0.1
        assert np.max(np.abs(a["b"] - 2 * expit(lg["b"]))) < 1e-14
    else:                                            # alpha itself instead of its log
        assert np.max(np.abs(expit(lg["f"]) - a["log_alpha"])) > 0.1
