"""Block-wise greedy per-matrix sparsity allocation (TopK-Guided, Appendix D, Table 4): the oracle
pinned to the pages' two-matrix toy block, and the library's host implementation against the oracle.

The pages give the toy block's endpoint, not its error values. The pin therefore uses an error
model of the kind the appendix describes (the large matrix B absorbs sparsity first, the small
matrix A is protected until B's cost rises). Under that model the step rule and the
compute-weighted budget accounting must land exactly on Table 4: pA = 0.5 and pB = 0.25 at P = 0.3,
after one switch from B to A. A wrong step size (not inversely proportional to the parameter
count) or a wrong budget measure cannot reach that point.
"""
import json
import os

import numpy as np
import pytest

import oracle
from tiered_weight_gemv_b200 import spax

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "pages_facts.json")


def toy_error(p):
    # linear cost per unit of sparsity, plus a steep penalty once B passes 0.25
    return float(p[0] + p[1] + 100.0 * max(0.0, p[1] - 0.25 - 1e-9))


@pytest.mark.parametrize("step_base", ["mean", "sum"])
def test_table4_toy_block(step_base):
    t4 = json.load(open(GOLDEN))["greedy_toy_table4"]
    p, order, ok = oracle.greedy_allocation([t4["f_A"], t4["f_B"]], t4["alpha"], t4["P"], toy_error,
                                            step_base=step_base)
    assert ok
    assert p[0] == pytest.approx(t4["p_A"], abs=1e-12) and p[1] == pytest.approx(t4["p_B"], abs=1e-12)
    P = (t4["f_A"] * p[0] + t4["f_B"] * p[1]) / (t4["f_A"] + t4["f_B"])
    assert P == pytest.approx(t4["P"], abs=1e-12)
    # B (index 1) first, then a single switch to A (index 0)
    assert order[0] == 1 and order[-1] == 0
    assert sum(1 for a, b in zip(order, order[1:]) if a != b) == 1


def test_each_increment_moves_the_budget_equally():
    f = [16.8, 16.8, 16.8, 16.8, 45.1, 45.1, 45.1]
    rng = np.random.default_rng(5)
    w = rng.uniform(0.5, 3.0, len(f))
    err = lambda p: float(np.sum(w * p ** 2))
    alpha = 0.025
    p, order, ok = oracle.greedy_allocation(f, alpha, 0.5, err)
    assert ok
    steps = [alpha * np.mean(f) / fm for fm in f]
    counts = np.bincount(order, minlength=len(f))
    assert np.allclose(p, counts * np.array(steps), atol=1e-12)
    # every increment moves sum f p / sum f by alpha / n, so the step count is fixed by the budget
    assert len(order) == int(np.ceil(0.5 / (alpha / len(f)) - 1e-9))


def test_library_matches_oracle():
    rng = np.random.default_rng(11)
    cases = [([100.0, 400.0], 0.1, 0.3, toy_error, 1.0)]
    for _ in range(25):
        n = int(rng.integers(1, 8))
        f = rng.uniform(1.0, 50.0, n)
        w = rng.uniform(0.1, 5.0, n)
        c = rng.uniform(0.0, 0.5, n)
        err = (lambda w, c: (lambda p: float(np.sum(w * p ** 2 + c * p))))(w, c)
        cases.append((list(f), float(rng.uniform(0.01, 0.1)), float(rng.uniform(0.0, 0.8)), err, 0.95))
    for f, alpha, target, err, pmax in cases:
        po, oo, ok = oracle.greedy_allocation(f, alpha, target, err, p_max=pmax)
        assert ok
        pl, ol = spax.spax_greedy_allocation(f, alpha, target, err, p_max=pmax)
        assert list(ol) == oo
        assert np.allclose(pl, po, rtol=0, atol=1e-12)  # same steps, rounding order may differ


def test_library_reports_an_unreachable_budget():
    with pytest.raises(spax.SpaxError):
        spax.spax_greedy_allocation([1.0, 1.0], 0.1, 0.9, lambda p: float(p.sum()), p_max=0.5)
    with pytest.raises(spax.SpaxError):
        spax.spax_greedy_allocation([1.0, -1.0], 0.1, 0.5, lambda p: 0.0)
    with pytest.raises(spax.SpaxError):
        spax.spax_greedy_allocation([1.0], 0.0, 0.5, lambda p: 0.0)
