"""Pins for the oracle's Chunk-Aware Growth budget solver and the
sparsity-to-block-count mapping.

Source: Light Forcing (paper.rainbus.top), execution flow, stage 1; gist.science
Technical Summary 2.1; 163.com article section 2. Readings: alpha_i = 1/sqrt(T_i);
the FLOP constraint is sum_i w_i s_i = s_target * sum_i w_i over all chunks
(optionally chunks 2..n); infeasible budgets are errors, not clamped.
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_cag_hand_worked():
    g = json.load(open(os.path.join(GOLDEN, "cag_hand.json")))
    for c in g["cases"]:
        rc, s, beta = oracle.cag(c["T"], c["w"], c["s_base"], c["s_target"], c["over_all"])
        assert (rc == 0) == c["ok"], c
        if c["ok"]:
            assert beta == pytest.approx(c["beta"], abs=1e-14)
            np.testing.assert_allclose(s, c["s"], atol=1e-14)


def test_blocks_for_sparsity_hand_worked():
    g = json.load(open(os.path.join(GOLDEN, "cag_hand.json")))["blocks_for_sparsity"]
    for sp, nkv, nsel, bpf, expect in g["cases"]:
        assert oracle.blocks_for_sparsity(sp, nkv, nsel, bpf) == expect


@pytest.mark.parametrize("seed", range(20))
def test_cag_budget_identity_and_growth(seed):
    """For random feasible inputs: s_1 = 0, the weighted sparsity equals the
    target, and s_i grows with i when T_i grows (alpha_i falls)."""
    rng = np.random.default_rng(seed)
    n = int(rng.integers(2, 12))
    T = np.cumsum(rng.uniform(0.5, 3.0, n))
    w = rng.uniform(0.5, 5.0, n)
    s_base = rng.uniform(0.85, 0.99)
    over_all = bool(seed % 2)
    # choose a target inside the feasible range for this (T, w, s_base)
    s_target = rng.uniform(0.3, 0.7) * s_base
    rc, s, beta = oracle.cag(T, w, s_base, s_target, over_all)
    if rc != 0:
        assert beta < 0 or (s[1:] < 0).any() or (s[1:] >= 1).any()
        return
    assert s[0] == 0.0
    idx = slice(0, n) if over_all else slice(1, n)
    assert (w[idx] * s[idx]).sum() == pytest.approx(s_target * w[idx].sum(), rel=1e-12)
    assert np.all(np.diff(s[1:]) >= -1e-15)
    np.testing.assert_allclose(s[1:], s_base - beta / np.sqrt(T[1:]), rtol=1e-14)


def test_cag_rollout_defaults_are_feasible():
    """The 7-chunk rollout with T_i = i, w_i = i, s_base 0.95, target 0.8 is
    feasible and progressive (a sanity check of the readings, not a pin of
    specific numbers)."""
    rc, s, beta = oracle.cag(np.arange(1, 8), np.arange(1, 8), 0.95, 0.80, True)
    assert rc == 0 and beta > 0
    assert s[0] == 0 and np.all(np.diff(s[1:]) > 0) and s[-1] < 0.95
