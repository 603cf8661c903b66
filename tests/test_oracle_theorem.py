"""Brute-force check of the (n+1)*eps <= 1 statement through the oracle's own
decode loop (vocab 8, n <= 3)."""
import numpy as np
import pytest

from oracle.decode import generate
from oracle.theorem import (JointTableModel, all_orders, joint_argmax, marginals,
                            planted_table, sequential_greedy)

VOCAB = 8


def _tables(n, eps, count, seed):
    rng = np.random.default_rng(seed)
    out = []
    tries = 0
    while len(out) < count and tries < 200_000:
        tries += 1
        t = planted_table(rng, n, VOCAB, concentration=0.3, mode_mass=rng.uniform(0.6, 0.999))
        if all(m.max() > 1 - eps for m in marginals(t)):
            out.append(t)
    assert len(out) == count
    return out


@pytest.mark.parametrize("n", [1, 2, 3])
def test_parallel_equals_sequential_when_condition_holds(n):
    eps = 1.0 / (n + 1)                      # (n+1) * eps = 1, the boundary case
    for t in _tables(n, eps, 40, seed=n):
        a = tuple(int(np.argmax(m)) for m in marginals(t))
        assert joint_argmax(t) == a
        for order in all_orders(n):
            assert sequential_greedy(t, order) == a
        model = JointTableModel(t)
        par = generate(model, [], n, n, 1 - eps, "none")
        assert par.steps == 1                # all n tokens pass the threshold together
        assert tuple(par.tokens) == a
        seq = generate(model, [], n, n, 1.01, "none")
        assert seq.steps == n
        assert tuple(seq.tokens) == a


def test_counterexample_when_condition_fails():
    # n = 2, eps slightly above 1/3: both marginals exceed 1 - eps but the
    # marginal argmax pair is not the joint argmax.
    d = 0.01
    t = np.zeros((VOCAB, VOCAB))
    t[0, 1] = 1 / 3
    t[1, 0] = 1 / 3
    t[0, 0] = 1 / 3 - d
    t[2, 2] = d
    m = marginals(t)
    eps = 1 / 3 + 2 * d
    assert all(mm.max() > 1 - eps for mm in m) and 3 * eps > 1
    a = tuple(int(np.argmax(mm)) for mm in m)
    assert a == (0, 0)
    assert joint_argmax(t) != a
    # by hand: revealing x1 first gives x1 = 0 (marginal 2/3 - d), then
    # p(x2 = 1 | x1 = 0) = (1/3) / (2/3 - d) beats p(x2 = 0 | x1 = 0); the
    # other order mirrors it
    assert sequential_greedy(t, (0, 1)) == (0, 1)
    assert sequential_greedy(t, (1, 0)) == (1, 0)
    par = generate(JointTableModel(t), [], 2, 2, 1 - eps, "none")
    assert tuple(par.tokens) == a            # parallel decoding returns the bad pair
    seq = generate(JointTableModel(t), [], 2, 2, 1.01, "none")
    assert tuple(seq.tokens) != a            # sequential greedy does not
