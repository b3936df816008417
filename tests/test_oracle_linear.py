"""CPU: pins of the oracle's dense projection, ``oracle.linear`` (C = A·Wᵀ in fp64), against facts
fixed outside it: a product worked by hand, permutation and diagonal weights, a rank-one product,
plain triple loops on tiny shapes, and a cancellation that single precision cannot resolve.

The projection stands for the 4·L·D² and 3·L·D² terms of the HSTU layer in the DLRMv3 review's
FLOP formula (section "model selection").  Each pin is a function of a candidate implementation so
that the same checks reject plausible mistakes (a missing transpose, a dropped term, a wrong sign,
single-precision accumulation), planted below as mutants.
"""
import numpy as np
import pytest

import oracle


def pin_hand_worked(lin):
    """A = [[1,2,3],[4,5,6]], W = [[1,0,-1],[2,1,0]]:
    C[0] = [1-3, 2+2] = [-2, 4];  C[1] = [4-6, 8+5] = [-2, 13]."""
    a = np.array([[1, 2, 3], [4, 5, 6]], np.float64)
    w = np.array([[1, 0, -1], [2, 1, 0]], np.float64)
    c = np.asarray(lin(a, w))
    assert c.shape == (2, 2)
    assert np.array_equal(c, np.array([[-2, 4], [-2, 13]], np.float64))


def pin_permutation(lin):
    """W = rows of the identity in the order of a 7-cycle π: C[:, n] = A[:, π(n)] exactly."""
    rng = np.random.default_rng(3)
    a = rng.standard_normal((5, 7))
    perm = np.array([1, 2, 3, 4, 5, 6, 0])
    w = np.eye(7)[perm]
    assert np.array_equal(np.asarray(lin(a, w)), a[:, perm])


def pin_diagonal(lin):
    """W = diag(s): every column of A is scaled by its own factor."""
    rng = np.random.default_rng(4)
    a = rng.standard_normal((6, 4))
    s = np.array([2.0, -0.5, 4.0, 0.25])
    assert np.array_equal(np.asarray(lin(a, np.diag(s))), a * s)


def pin_rank_one(lin):
    """K = 1: C is the outer product of A's single column and W's single column."""
    a = np.array([[1.0], [-2.0], [3.0]])
    w = np.array([[5.0], [7.0]])
    assert np.array_equal(np.asarray(lin(a, w)), np.array([[5.0, 7.0], [-10.0, -14.0], [15.0, 21.0]]))


def pin_triple_loop(lin):
    """Non-square tiny shapes against the definition C[m, n] = Σ_k A[m, k] W[n, k], written as loops."""
    rng = np.random.default_rng(5)
    M, N, K = 3, 4, 5
    a = rng.standard_normal((M, K))
    w = rng.standard_normal((N, K))
    ref = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += a[m, k] * w[n, k]
            ref[m, n] = acc
    c = np.asarray(lin(a, w))
    assert c.shape == (M, N)
    assert np.abs(c - ref).max() <= 1e-14 * np.abs(ref).max()


def pin_double_precision(lin):
    """1e8 + 1 - 1e8 = 1 in double precision; single precision loses the 1."""
    a = np.array([[1e8, 1.0, -1e8]], np.float32)
    w = np.array([[1.0, 1.0, 1.0]], np.float32)
    assert np.asarray(lin(a, w))[0, 0] == 1.0


PINS = [pin_hand_worked, pin_permutation, pin_diagonal, pin_rank_one, pin_triple_loop, pin_double_precision]

MUTANTS = {
    "no_transpose": lambda a, w: np.asarray(a, np.float64) @ np.asarray(w, np.float64),
    "transposed_result": lambda a, w: (np.asarray(a, np.float64) @ np.asarray(w, np.float64).T).T,
    "drops_last_k": lambda a, w: np.asarray(a, np.float64)[:, :-1] @ np.asarray(w, np.float64)[:, :-1].T,
    "negated": lambda a, w: -(np.asarray(a, np.float64) @ np.asarray(w, np.float64).T),
    "single_precision": lambda a, w: (np.asarray(a, np.float32) @ np.asarray(w, np.float32).T).astype(np.float64),
    "reversed_k": lambda a, w: np.asarray(a, np.float64) @ np.asarray(w, np.float64)[:, ::-1].T,
}


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_linear_pin(pin):
    pin(oracle.linear)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_linear_pins_reject_mutant(name):
    caught = []
    for pin in PINS:
        try:
            pin(MUTANTS[name])
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, "no pin rejects the linear mutant %s" % name
