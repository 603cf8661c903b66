"""Toy check of the parallel-equals-sequential statement (oracle).

Test infrastructure only; see ``oracle/__init__.py``.

Statement (ccyt168.com Fast-dLLM overview, section 一, item 2 "理论证明"; also
the techwalker.com article, section "解决并行解码的质量下降问题"): if n tokens
are decoded in parallel and each has confidence greater than 1 - eps, and
(n+1)*eps <= 1, then under greedy decoding the parallel result equals the
sequential result.

The toy "model" is an explicit joint probability table p(x_1..x_n) over a
small vocabulary.  Given a partially revealed sequence it returns, for each
position, the log of the exact conditional marginal given the revealed
positions.  It plugs into ``oracle.decode.generate`` (cache mode "none"), so
the same decode loop that runs the transformer is what gets checked.

Why the statement holds (the closed-form argument the tests follow): let a be
the vector of marginal argmaxes.  P(x = a) >= 1 - sum_i P(x_i != a_i) >
1 - n*eps >= eps, while any x != a differs from a somewhere, so
P(x) <= P(x_i != a_i) < eps.  Hence a is the unique joint argmax.  For a
revealed set S agreeing with a, P(x_j != a_j | x_S = a_S) <
eps / (1 - (n-1)*eps) <= 1/2, so a_j is also every conditional argmax and
sequential greedy picks a in any order.
"""
from __future__ import annotations

import itertools
from dataclasses import dataclass
from typing import Dict, List, Sequence

import numpy as np


@dataclass(frozen=True)
class ToySpec:
    mask_id: int
    vocab: int


def marginals(table: np.ndarray) -> List[np.ndarray]:
    n = table.ndim
    return [table.sum(axis=tuple(j for j in range(n) if j != i)) for i in range(n)]


def conditional(table: np.ndarray, revealed: Dict[int, int], i: int) -> np.ndarray:
    """p(x_i = . | x_j = revealed[j] for j in revealed), exactly."""
    idx = tuple(revealed.get(j, slice(None)) for j in range(table.ndim))
    sub = table[idx]
    # remaining axes are the unrevealed positions in increasing order
    free = [j for j in range(table.ndim) if j not in revealed]
    axis = free.index(i)
    p = sub.sum(axis=tuple(k for k in range(sub.ndim) if k != axis))
    tot = p.sum()
    return p / tot


def joint_argmax(table: np.ndarray) -> tuple:
    return tuple(int(v) for v in np.unravel_index(int(np.argmax(table)), table.shape))


def sequential_greedy(table: np.ndarray, order: Sequence[int]) -> tuple:
    """Reveal positions in ``order``, each time taking the argmax of the exact
    conditional given what is already revealed."""
    revealed: Dict[int, int] = {}
    for i in order:
        revealed[i] = int(np.argmax(conditional(table, revealed, i)))
    return tuple(revealed[i] for i in range(table.ndim))


def planted_table(rng: np.random.Generator, n: int, vocab: int, concentration: float,
                  mode_mass: float) -> np.ndarray:
    """Dirichlet-random joint table with extra mass ``mode_mass`` planted on a
    random configuration."""
    t = rng.dirichlet(np.full(vocab ** n, concentration)).reshape((vocab,) * n)
    a = tuple(int(v) for v in rng.integers(0, vocab, size=n))
    t = t * (1.0 - mode_mass)
    t[a] += mode_mass
    return t


class JointTableModel:
    """Callback model for ``oracle.decode.generate``: logits are the log exact
    conditional marginals of a joint table given the unmasked positions."""

    def __init__(self, table: np.ndarray):
        self.table = np.asarray(table, dtype=np.float64)
        v = self.table.shape[0]
        self.spec = ToySpec(mask_id=v, vocab=v + 1)

    def forward(self, x, rows, cache=None, return_kv=False, return_hidden=False, head_rows=None):
        x = np.asarray(x, dtype=np.int64)
        rows = np.asarray(rows, dtype=np.int64)
        if head_rows is not None:
            rows = rows[np.asarray(head_rows, dtype=np.int64)]
        mask = self.spec.mask_id
        revealed = {j: int(x[j]) for j in range(x.shape[0]) if x[j] != mask}
        z = np.full((rows.shape[0], self.spec.vocab), -np.inf)
        for r, i in enumerate(rows):
            if i in revealed:
                z[r, revealed[i]] = 0.0
                continue
            p = conditional(self.table, revealed, int(i))
            with np.errstate(divide="ignore"):
                z[r, :-1] = np.log(p)
        if return_kv:
            return z, []
        return z


def all_orders(n: int):
    return itertools.permutations(range(n))
