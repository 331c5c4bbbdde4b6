"""Selection-rule mathematics from the Fast-dLLM technical review (fp64).

TEST INFRASTRUCTURE, like the rest of ``oracle``.

Source: "Fast-dLLM: Reusing Bidirectional State and Spending Confidence on
Parallel Tokens" (technical review): section 4 eq. (4) and the product of
marginals; section 5 eqs. (5)-(8) (the (n+1)eps <= 1 agreement condition) and
the eta counterexample family; section 5.1 eq. (9) (heterogeneous budget);
section 6 eq. (13) and Algorithm 3 (factor selection).

The joint-distribution mathematics (marginals, total variation, joint and
product maximisers, the eta family) is written here in numpy: it pins the
theorem the selection rules rest on and feeds no GPU comparison.  The
selection rules themselves (eq. 9, eq. 13 / Algorithm 3) are evaluated by the
C++ oracle in ``step.cc``.
"""
from __future__ import annotations

import itertools
import math

import numpy as np

from . import step


def marginals(joint: np.ndarray):
    """Per-position marginal distributions of a joint over n positions
    (``joint`` has one axis per position)."""
    n = joint.ndim
    return [joint.sum(axis=tuple(a for a in range(n) if a != j)) for j in range(n)]


def product_of_marginals(joint: np.ndarray) -> np.ndarray:
    """q(x) = prod_j p_j(x_j), the independent approximation of eq. (5)."""
    q = np.ones(())
    for m in marginals(joint):
        q = np.multiply.outer(q, m)
    return q


def tv_distance(p: np.ndarray, q: np.ndarray) -> float:
    """Total variation: half the sum of absolute differences (section 4)."""
    return 0.5 * float(np.abs(np.asarray(p) - np.asarray(q)).sum())


def argmax_joint(p: np.ndarray):
    """Most probable complete assignment; the lowest index on a tie."""
    return tuple(int(i) for i in np.unravel_index(int(np.argmax(p)), p.shape))


def argmax_product(joint: np.ndarray):
    """Concatenation of the per-position marginal maximisers."""
    return tuple(int(np.argmax(m)) for m in marginals(joint))


def agreement_certified(joint: np.ndarray) -> bool:
    """Premise of eq. (8): every marginal maximum exceeds 1 - eps with
    (n + 1) eps <= 1.  Uses the tightest eps, 1 - min_j max p_j, and the
    theorem's strict marginal inequality is then automatic (eps is attained),
    so the certificate asks the premise for any slightly larger eps:
    (n + 1) * eps < 1."""
    n = joint.ndim
    eps = 1.0 - min(float(m.max()) for m in marginals(joint))
    return (n + 1) * eps < 1.0


def max_certified_group(eps: float) -> int:
    """Largest n with (n + 1) eps <= 1 (section 6: eps = 0.1 gives n <= 9)."""
    return int(math.floor(1.0 / eps + 1e-12)) - 1


def eta_family(n: int, eta: float) -> np.ndarray:
    """Counterexample joint over n binary positions (end of section 5): the
    all-zero string has 1/(n+1) - eta, each string with exactly one 1 has
    1/(n+1) + eta/n, every other string 0."""
    p = np.zeros((2,) * n)
    p[(0,) * n] = 1.0 / (n + 1) - eta
    for j in range(n):
        idx = [0] * n
        idx[j] = 1
        p[tuple(idx)] = 1.0 / (n + 1) + eta / n
    return p


def heterogeneous_budget_ok(eps) -> bool:
    """Eq. (9): sum_j eps_j + max_j eps_j < 1 (evaluated by the C++ oracle)."""
    return step.budget_ok(eps)


def factor_select(masked_positions, conf_of, f: float):
    """Algorithm 3 with eq. (13): sort the masked positions by decreasing
    confidence (ties: lower position first); keep the largest n with
    (n + 1) (1 - c_(n)) < f; if no n qualifies, the first position alone.
    Evaluated by the C++ oracle."""
    return step.factor_select(masked_positions, conf_of, f)


def budget_select(masked_positions, conf_of):
    """Selection by the heterogeneous error budget of eq. (9): sort the masked
    positions by decreasing confidence (ties: lower position first), with
    eps_j = 1 - c_j; keep the largest n whose first n positions satisfy
    sum eps + max eps < 1; if no n qualifies, the first position alone.
    Evaluated by the C++ oracle."""
    return step.budget_select(masked_positions, conf_of)


def all_assignments(n: int, k: int):
    """Every string of length n over an alphabet of size k."""
    return itertools.product(range(k), repeat=n)
