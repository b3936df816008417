"""CPU: pins of the oracle's backward pass (``oracle.bwd`` / ``oracle.bwd_rows``).

The pages print no backward pass; the oracle derives it from the forward definition by the chain
rule (DLRMv3 review, section "model selection": out = Mask(SiLU(alpha Q K^T)) V / N).  It is pinned
here against facts outside it:
- central finite differences of the dense brute-force forward (tests/bruteforce.py, NumPy fp64,
  which shares nothing with the C oracle) for every input element of tiny jagged batches;
- closed forms: q = 0 gives silu'(0) = 1/2 and silu(0) = 0; a single-token user;
- the mask: a candidate key receives gradient from its own query only;
- linearity in the output gradient, and the row-selection entry equal to the full pass.
Planted mutants of the C source (a sigmoid for silu', a dropped alpha or 1/N, a swapped operand,
an unmasked pair) must each be rejected by at least one pin.
"""
import os
import subprocess

import numpy as np
import pytest

import bruteforce
import oracle

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "hstu_oracle.c")


def _batch(rng, lengths, targets, H, d, scale=0.6):
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    total = int(off[-1])
    q, k, v, do = ((rng.standard_normal((total, H, d)) * scale).astype(np.float32) for _ in range(4))
    return q, k, v, do, off, np.asarray(targets, np.int32)


def _fd_grads(q, k, v, do, off, nt, alpha, N, eps=1e-6):
    """Central differences of sum(do * attention(q, k, v)) with the dense fp64 brute force."""
    base = [np.asarray(x, np.float64) for x in (q, k, v)]
    dof = np.asarray(do, np.float64)
    grads = []
    for which in range(3):
        g = np.zeros_like(base[which])
        for idx in np.ndindex(*base[which].shape):
            args_p = [b.copy() for b in base]
            args_m = [b.copy() for b in base]
            args_p[which][idx] += eps
            args_m[which][idx] -= eps
            lp = float(np.sum(dof * bruteforce.attention(*args_p, off, nt, alpha, N)))
            lm = float(np.sum(dof * bruteforce.attention(*args_m, off, nt, alpha, N)))
            g[idx] = (lp - lm) / (2 * eps)
        grads.append(g)
    return grads


def pin_bwd_finite_differences(o):
    """Every element of dq, dk, dv of a tiny ragged batch (zero-length, single-token, history-only
    and candidate-only users) against central differences of the brute-force forward."""
    rng = np.random.default_rng(31)
    lengths, targets = [5, 0, 9, 1, 4], [2, 0, 3, 1, 0]
    q, k, v, do, off, nt = _batch(rng, lengths, targets, H=2, d=3)
    alpha, N = 0.8, 7.0
    got = o.bwd(q, k, v, do, off, nt, alpha, N)
    want = _fd_grads(q, k, v, do, off, nt, alpha, N)
    for name, g, w in zip("qkv", got, want):
        err = np.abs(g - w).max()
        assert err <= 1e-7 * max(1.0, np.abs(w).max()), (name, err)


def pin_bwd_finite_differences_large_scores(o):
    """Scores of magnitude ~5 (both SiLU tails), against central differences."""
    rng = np.random.default_rng(32)
    q, k, v, do, off, nt = _batch(rng, [6, 3], [2, 3], H=1, d=4, scale=1.5)
    alpha, N = 1.0, 3.0
    got = o.bwd(q, k, v, do, off, nt, alpha, N)
    want = _fd_grads(q, k, v, do, off, nt, alpha, N)
    for name, g, w in zip("qkv", got, want):
        err = np.abs(g - w).max()
        assert err <= 1e-6 * max(1.0, np.abs(w).max()), (name, err)


def pin_bwd_zero_queries(o):
    """q = 0: every score is 0, silu(0) = 0 and silu'(0) = 1/2, so dv = 0, dk = 0 and
    dq[i] = (alpha / 2) * sum_{j in A(i)} (do[i] . v[j] / N) * k[j]."""
    rng = np.random.default_rng(33)
    L, U, H, d = 7, 4, 1, 3
    off = np.array([0, L], np.int32)
    nt = np.array([L - U], np.int32)
    q = np.zeros((L, H, d), np.float32)
    k, v, do = (rng.standard_normal((L, H, d)).astype(np.float32) for _ in range(3))
    alpha, N = 0.9, 5.0
    dq, dk, dv = o.bwd(q, k, v, do, off, nt, alpha, N)
    assert np.all(dv == 0.0) and np.all(dk == 0.0)
    kf, vf, dof = (x[:, 0, :].astype(np.float64) for x in (k, v, do))
    for i in range(L):
        keys = list(range(i + 1)) if i < U else list(range(U)) + [i]
        want = sum((alpha / 2) * (dof[i] @ vf[j] / N) * kf[j] for j in keys)
        assert np.allclose(dq[i, 0], want, rtol=1e-13, atol=1e-15)


def pin_bwd_single_token(o):
    """A one-token user: out = silu(x) v / N with x = alpha q.k.  With q.k = 0 (orthogonal
    vectors) the gradients are dv = 0, dq = (alpha/2)(do.v/N) k, dk = (alpha/2)(do.v/N) q."""
    q = np.array([[[1.0, 2.0, 0.0]]], np.float32)
    k = np.array([[[2.0, -1.0, 3.0]]], np.float32)  # q.k = 0
    v = np.array([[[0.5, 1.0, -2.0]]], np.float32)
    do = np.array([[[2.0, 1.0, -1.0]]], np.float32)  # do.v = 1 + 1 + 2 = 4
    alpha, N = 0.5, 2.0
    dq, dk, dv = o.bwd(q, k, v, do, np.array([0, 1], np.int32), np.array([1], np.int32), alpha, N)
    g = 4.0 / N
    assert np.array_equal(dv[0, 0], np.zeros(3))
    assert np.allclose(dq[0, 0], (alpha / 2) * g * k[0, 0], rtol=1e-15)
    assert np.allclose(dk[0, 0], (alpha / 2) * g * q[0, 0], rtol=1e-15)


def pin_bwd_candidate_keys(o):
    """A candidate key j is seen by its own query only: dv[j] = silu(x_jj) do[j] / N, and changing
    the output gradient of every other row leaves dk[j] and dv[j] unchanged."""
    rng = np.random.default_rng(34)
    q, k, v, do, off, nt = _batch(rng, [9], [4], H=2, d=3)
    alpha, N = 0.7, 4.0
    dq, dk, dv = o.bwd(q, k, v, do, off, nt, alpha, N)
    U = 5
    for j in range(U, 9):
        for h in range(2):
            x = alpha * float(np.dot(q[j, h].astype(np.float64), k[j, h].astype(np.float64)))
            assert np.allclose(dv[j, h], x / (1 + np.exp(-x)) * do[j, h] / N, rtol=1e-13)
    do2 = do.copy()
    do2[:5] = rng.standard_normal(do2[:5].shape).astype(np.float32)
    do2[5] *= -3.0  # another candidate's row
    _, dk2, dv2 = o.bwd(q, k, v, do2, off, nt, alpha, N)
    for j in range(6, 9):
        assert np.array_equal(dk2[j], dk[j]) and np.array_equal(dv2[j], dv[j])


def pin_bwd_linear_in_dout(o):
    """Doubling the output gradient doubles every gradient exactly."""
    rng = np.random.default_rng(35)
    q, k, v, do, off, nt = _batch(rng, [8, 3, 11], [3, 0, 11], H=2, d=4)
    a = o.bwd(q, k, v, do, off, nt, 0.6, 9.0)
    b = o.bwd(q, k, v, 2 * do, off, nt, 0.6, 9.0)
    for x, y in zip(a, b):
        assert np.array_equal(2 * x, y)


def pin_bwd_rows_equal_full(o):
    """The row-selection entry returns the full pass's rows exactly."""
    rng = np.random.default_rng(36)
    q, k, v, do, off, nt = _batch(rng, [12, 0, 7, 2], [5, 0, 0, 2], H=3, d=5)
    full = o.bwd(q, k, v, do, off, nt, 0.4, 6.0)
    users = np.array([0, 0, 0, 2, 2, 3, 3, 0], np.int32)
    local = np.array([0, 6, 11, 0, 6, 0, 1, 7], np.int32)
    rows = o.bwd_rows(q, k, v, do, off, nt, 0.4, 6.0, users, local)
    idx = off[users] + local
    for f, r in zip(full, rows):
        assert np.array_equal(f[idx], r)


BWD_PINS = [pin_bwd_finite_differences, pin_bwd_finite_differences_large_scores, pin_bwd_zero_queries,
            pin_bwd_single_token, pin_bwd_candidate_keys, pin_bwd_linear_in_dout, pin_bwd_rows_equal_full]

MUTANTS = {
    "dsilu_is_sigmoid": ("return sg * (1.0 + x * (1.0 - sg));", "return sg;"),
    "dsilu_sign": ("return sg * (1.0 + x * (1.0 - sg));", "return sg * (1.0 - x * (1.0 - sg));"),
    "dsilu_is_sigmoid_derivative": ("return sg * (1.0 + x * (1.0 - sg));", "return sg * (1.0 - sg);"),
    "ds_missing_alpha": ("      double ds = g * dsilu(x) * alpha;\n      for (int32_t c = 0; c < d; ++c) {\n        dvj",
                         "      double ds = g * dsilu(x);\n      for (int32_t c = 0; c < d; ++c) {\n        dvj"),
    "dv_missing_normaliser": ("dvj[c] += p * (double)doi[c] / N;", "dvj[c] += p * (double)doi[c];"),
    "g_missing_normaliser": ("      g /= N;\n      double x = alpha * s;\n      double p = silu(x);\n      double ds = g * dsilu(x) * alpha;\n      for (int32_t c = 0; c < d; ++c) {\n        dvj",
                             "      double x = alpha * s;\n      double p = silu(x);\n      double ds = g * dsilu(x) * alpha;\n      for (int32_t c = 0; c < d; ++c) {\n        dvj"),
    "dk_uses_keys": ("dkj[c] += ds * (double)qi[c];", "dkj[c] += ds * (double)kj[c];"),
    "dq_uses_queries": ("dqi[c] += ds * (double)kj[c];", "dqi[c] += ds * (double)qi[c];"),
    "g_uses_keys": ("for (int32_t c = 0; c < d; ++c) g += (double)doi[c] * (double)vj[c];\n      g /= N;\n      double x",
                    "for (int32_t c = 0; c < d; ++c) g += (double)doi[c] * (double)kj[c];\n      g /= N;\n      double x"),
    "dv_uses_scores": ("dvj[c] += p * (double)doi[c] / N;", "dvj[c] += alpha * s * (double)doi[c] / N;"),
    "bwd_plain_causal": ("      if (!visible(i, j, U)) continue;\n      const float* kj = ks + (int64_t)j * stride;\n      const float* vj = vs + (int64_t)j * stride;\n      double* dkj",
                         "      if (j > i) continue;\n      const float* kj = ks + (int64_t)j * stride;\n      const float* vj = vs + (int64_t)j * stride;\n      double* dkj"),
}


@pytest.mark.parametrize("pin", BWD_PINS, ids=lambda f: f.__name__)
def test_bwd_pin(orc, pin):
    pin(orc)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_bwd_pins_reject_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, "mutation anchor not found: %s" % name
    cfile = tmp_path / "mutant.c"
    cfile.write_text(src.replace(old, new, 1))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", str(lib), str(cfile), "-lm"],
                   check=True)
    o = oracle.Oracle(str(lib))
    caught = []
    for pin in BWD_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, "no pin rejects mutant %s" % name
