"""Pins of the fp64 oracle against facts fixed outside it: brute force on tiny inputs, closed
forms, regimes where SiLU reduces to a known function, invariants of the mask, and the DLRMv3
review's FLOP formula.  Each pin is a function of an oracle instance so the same checks also run
against deliberately broken builds (tests/test_oracle_mutants.py).

Method: "DLRMv3: MLPerf Inference generative recommendation benchmark" review, section "model
selection" (attention = Mask(SiLU(Q K^T)) V; shared history encoding; K/V reuse; FLOP formula);
infolabhq.com multi-stage sequence model page (user side independent of candidates; target-
aware attention).  alpha and N are explicit scalars.
"""
import math

import numpy as np
from scipy.special import expit

import bruteforce
from hstu_pointwise_attention_jagged_b200 import workloads


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _rand_batch(rng, lengths, targets, H, d, scale=1.0):
    off = workloads.offsets_from_lengths(lengths)
    total = int(off[-1])
    q = (rng.standard_normal((total, H, d)) * scale).astype(np.float32)
    k = (rng.standard_normal((total, H, d)) * scale).astype(np.float32)
    v = rng.standard_normal((total, H, d)).astype(np.float32)
    return q, k, v, off, np.asarray(targets, np.int32)


# ----------------------------------------------------------------------------- brute force
def pin_bruteforce_tiny(o):
    """The tiny workload (fp32) against the dense brute force, to 1e-12 relative."""
    w = workloads.make("tiny")
    got = o.fwd(w.q, w.k, w.v, w.seq_offsets, w.num_targets, w.alpha, w.N)
    ref = bruteforce.attention(w.q, w.k, w.v, w.seq_offsets, w.num_targets, w.alpha, w.N)
    assert _rel(got, ref) <= 1e-12, _rel(got, ref)


def pin_bruteforce_random(o):
    """Random short users (T in {0, 1, L}, a zero-length user) against the brute force."""
    rng = np.random.default_rng(11)
    lengths = [7, 0, 1, 13, 40, 5, 29, 2]
    targets = [0, 0, 1, 13, 3, 5, 1, 0]
    q, k, v, off, nt = _rand_batch(rng, lengths, targets, H=3, d=5, scale=0.7)
    got = o.fwd(q, k, v, off, nt, 0.9, 17.0)
    ref = bruteforce.attention(q, k, v, off, nt, 0.9, 17.0)
    assert _rel(got, ref) <= 1e-12, _rel(got, ref)


# ----------------------------------------------------------------------------- closed forms
def pin_closed_form_counts(o):
    """d=1, q=k=v=1, alpha=ln 3: every visible key contributes silu(ln 3) = (3/4) ln 3, so
    out_i = (3/4) ln 3 * |A(i)| / N with |A(i)| = i+1 (history) or U+1 (candidate)."""
    L, U, N = 23, 9, 5.0
    ones = np.ones((L, 1, 1), np.float32)
    off = np.array([0, L], np.int32)
    got = o.fwd(ones, ones, ones, off, np.array([L - U], np.int32), math.log(3.0), N)[:, 0, 0]
    counts = np.array([i + 1 if i < U else U + 1 for i in range(L)], np.float64)
    ref = 0.75 * math.log(3.0) * counts / N
    assert np.allclose(got, ref, rtol=1e-14, atol=0), (got, ref)


def pin_zero_query(o):
    """q = 0 gives scores 0 and silu(0) = 0, so the output is exactly zero."""
    rng = np.random.default_rng(3)
    q, k, v, off, nt = _rand_batch(rng, [12, 9], [4, 0], H=2, d=4)
    got = o.fwd(np.zeros_like(q), k, v, off, nt, 1.3, 2.0)
    assert np.all(got == 0.0)


def pin_single_token(o):
    """L = 1: out = silu(alpha q.k) v / N.  q.k = 2 and alpha = ln(3)/2 give silu = (3/4) ln 3."""
    q = np.array([[[1.0, 1.0]]], np.float32)
    k = np.array([[[1.5, 0.5]]], np.float32)
    v = np.array([[[2.0, -4.0]]], np.float32)
    for T in (0, 1):
        got = o.fwd(q, k, v, np.array([0, 1], np.int32), np.array([T], np.int32), math.log(3.0) / 2, 4.0)
        ref = 0.75 * math.log(3.0) * np.array([2.0, -4.0]) / 4.0
        assert np.allclose(got[0, 0], ref, rtol=1e-14, atol=0), (got, ref)


def pin_linear_regime(o):
    """All scores >= 40: silu(x) = x to 1e-16, so out = (M * alpha Q K^T) V / N (plain matmuls)."""
    rng = np.random.default_rng(5)
    lengths, targets = [20, 11], [6, 3]
    off = workloads.offsets_from_lengths(lengths)
    total, H, d = int(off[-1]), 2, 8
    q = (4.0 + 0.2 * rng.standard_normal((total, H, d))).astype(np.float32)
    k = (4.0 + 0.2 * rng.standard_normal((total, H, d))).astype(np.float32)
    v = rng.standard_normal((total, H, d)).astype(np.float32)
    alpha, N = 0.5, 3.0
    got = o.fwd(q, k, v, off, np.array(targets, np.int32), alpha, N)
    ref = np.zeros_like(got)
    for b in range(len(lengths)):
        s0, s1 = off[b], off[b + 1]
        M = bruteforce.visibility(s1 - s0, lengths[b] - targets[b])
        for h in range(H):
            S = alpha * (q[s0:s1, h].astype(np.float64) @ k[s0:s1, h].astype(np.float64).T)
            assert S.min() >= 40.0
            ref[s0:s1, h] = (np.where(M, S, 0.0) @ v[s0:s1, h].astype(np.float64)) / N
    assert _rel(got, ref) <= 1e-13, _rel(got, ref)


def pin_negative_regime(o):
    """All scores <= -40: silu(x) = x e^x / (1 + e^x) is below 2e-16 in magnitude, so out ~ 0."""
    rng = np.random.default_rng(6)
    lengths, targets = [15], [5]
    off = workloads.offsets_from_lengths(lengths)
    total, H, d = 15, 1, 8
    q = (4.0 + 0.2 * rng.standard_normal((total, H, d))).astype(np.float32)
    k = -q
    v = rng.standard_normal((total, H, d)).astype(np.float32)
    got = o.fwd(q, k, v, off, np.array(targets, np.int32), 0.5, 1.0)
    assert np.abs(got).max() <= 1e-14, np.abs(got).max()


def pin_small_score_taylor(o):
    """|x| <= 1e-2: silu(x) = x/2 + x^2/4 - x^4/48 + ..., so out = (M * (S/2 + S^2/4)) V / N with
    S = alpha Q K^T to ~1e-7 relative, while the x^2/4 term itself weighs ~1e-3.  Fixes the
    sigmoid's sign and its 1/2 and 1/4 terms."""
    rng = np.random.default_rng(7)
    lengths, targets = [31, 18], [9, 18]
    q, k, v, off, nt = _rand_batch(rng, lengths, targets, H=2, d=6, scale=0.02)
    alpha, N = 0.5, 2.0
    got = o.fwd(q, k, v, off, nt, alpha, N)
    ref = np.zeros_like(got)
    for b in range(len(lengths)):
        s0, s1 = off[b], off[b + 1]
        M = bruteforce.visibility(s1 - s0, lengths[b] - targets[b])
        for h in range(2):
            S = alpha * (q[s0:s1, h].astype(np.float64) @ k[s0:s1, h].astype(np.float64).T)
            assert np.abs(S).max() <= 1e-2
            ref[s0:s1, h] = (np.where(M, S / 2 + S * S / 4, 0.0) @ v[s0:s1, h].astype(np.float64)) / N
    assert _rel(got, ref) <= 1e-6, _rel(got, ref)


def pin_causal_textbook(o):
    """No candidates (T = 0): plain causal pointwise attention (tril * silu(alpha Q K^T)) V / N."""
    rng = np.random.default_rng(8)
    q, k, v, off, nt = _rand_batch(rng, [37], [0], H=1, d=7, scale=0.6)
    alpha, N = 1.1, 9.0
    S = alpha * (q[:, 0].astype(np.float64) @ k[:, 0].astype(np.float64).T)
    ref = (np.tril(S * expit(S)) @ v[:, 0].astype(np.float64)) / N
    got = o.fwd(q, k, v, off, None, alpha, N)[:, 0]
    assert _rel(got, ref) <= 1e-12, _rel(got, ref)


# ----------------------------------------------------------------------------- invariants
def _base(seed=9):
    rng = np.random.default_rng(seed)
    lengths, targets = [45, 30, 12], [7, 30, 3]
    return _rand_batch(rng, lengths, targets, H=2, d=6, scale=0.8) + (lengths, targets)


def pin_history_ignores_candidates(o):
    """Changing the candidates' K/V leaves every history row bitwise unchanged."""
    q, k, v, off, nt, lengths, targets = _base()
    a = o.fwd(q, k, v, off, nt, 0.8, 11.0)
    k2, v2 = k.copy(), v.copy()
    for b in range(3):
        s0, U = off[b], lengths[b] - targets[b]
        k2[s0 + U:off[b + 1]] += 1.5
        v2[s0 + U:off[b + 1]] -= 2.0
    c = o.fwd(q, k2, v2, off, nt, 0.8, 11.0)
    for b in range(3):
        s0, U = off[b], lengths[b] - targets[b]
        assert np.array_equal(a[s0:s0 + U], c[s0:s0 + U])


def pin_candidates_independent(o):
    """Changing one candidate's K/V leaves every other candidate's row bitwise unchanged, and
    dropping trailing candidates leaves the remaining rows bitwise unchanged (N fixed)."""
    q, k, v, off, nt, lengths, targets = _base()
    a = o.fwd(q, k, v, off, nt, 0.8, 11.0)
    s0, U, L = off[0], lengths[0] - targets[0], lengths[0]
    j = s0 + U + 2
    k2, v2 = k.copy(), v.copy()
    k2[j] += 3.0
    v2[j] += 3.0
    c = o.fwd(q, k2, v2, off, nt, 0.8, 11.0)
    for i in range(s0 + U, s0 + L):
        if i != j:
            assert np.array_equal(a[i], c[i])
    assert not np.array_equal(a[j], c[j])
    # drop the last 4 candidates of user 0
    keep = np.ones(len(q), bool)
    keep[s0 + L - 4:s0 + L] = False
    off2 = workloads.offsets_from_lengths([L - 4, lengths[1], lengths[2]])
    nt2 = np.array([targets[0] - 4, targets[1], targets[2]], np.int32)
    d = o.fwd(q[keep], k[keep], v[keep], off2, nt2, 0.8, 11.0)
    assert np.array_equal(d, a[keep])


def pin_cached_equals_full(o):
    """Streaming: rows at positions >= cached_len are bitwise the full pass's rows."""
    q, k, v, off, nt, lengths, targets = _base()
    cl = np.array([20, 0, 9], np.int32)
    full = o.fwd(q, k, v, off, nt, 0.8, 11.0)
    sel = np.concatenate([np.arange(off[b] + cl[b], off[b + 1]) for b in range(3)])
    got = o.fwd_cached(q[sel], k, v, off, nt, cl, 0.8, 11.0)
    assert np.array_equal(got, full[sel])
    rows = o.rows(q[sel], k, v, off, nt, cl, 0.8, 11.0, [0, 2, 1], [0, 2, 29])
    assert np.array_equal(rows[0], full[off[0] + 20]) and np.array_equal(rows[1], full[off[2] + 11])
    assert np.array_equal(rows[2], full[off[1] + 29])


def pin_linearity_and_scale(o):
    """Linear in V (x2 is exact), proportional to 1/N (x2 is exact), heads independent, users
    permutable."""
    q, k, v, off, nt, lengths, targets = _base()
    a = o.fwd(q, k, v, off, nt, 0.8, 11.0)
    assert np.array_equal(o.fwd(q, k, 2 * v, off, nt, 0.8, 11.0), 2 * a)
    assert np.array_equal(o.fwd(q, k, v, off, nt, 0.8, 22.0), a / 2)
    q2 = q.copy()
    q2[:, 1] += 1.0
    c = o.fwd(q2, k, v, off, nt, 0.8, 11.0)
    assert np.array_equal(c[:, 0], a[:, 0]) and not np.array_equal(c[:, 1], a[:, 1])
    perm = [2, 0, 1]
    segs = [np.arange(off[b], off[b + 1]) for b in perm]
    idx = np.concatenate(segs)
    off_p = workloads.offsets_from_lengths([lengths[b] for b in perm])
    got = o.fwd(q[idx], k[idx], v[idx], off_p, nt[perm], 0.8, 11.0)
    assert np.array_equal(got, a[idx])


# ----------------------------------------------------------------------------- FLOP formula
def pin_flop_formula(o):
    """One layer, no candidates: the oracle performs d*L(L+1)/2 multiply-adds per matmul per head,
    i.e. 2 * (L*L*D/2) + L*D FLOPs for one matmul over all heads (D = H*d) — the review's
    attention term plus the diagonal."""
    rng = np.random.default_rng(10)
    L, H, d = 29, 3, 4
    q, k, v, off, nt = _rand_batch(rng, [L], [0], H=H, d=d)
    _, macs = o.fwd(q, k, v, off, None, 0.5, 1.0, return_macs=True)
    D = H * d
    per_matmul = macs // 2
    assert 2 * per_matmul == 2 * (L * L * D // 2) + L * D, (macs, L, D)


def pin_rab_bruteforce(o):
    """Relative-bias variant against the dense restatement, with a table shorter than the longest
    distance (so clipping is exercised) and random entries of both signs."""
    rng = np.random.default_rng(61)
    q, k, v, off, nt = _rand_batch(rng, [23, 1, 17, 0, 30], [4, 1, 0, 0, 9], 2, 8)
    rab = rng.normal(size=(2, 7)).astype(np.float32)
    users, local = [], []
    for b in range(len(off) - 1):
        for r in range(int(off[b + 1] - off[b])):
            users.append(b)
            local.append(r)
    got = o.rows_rab(q, k, v, off, nt, None, rab, 0.37, 11.0, users, local)
    ref = bruteforce.attention_rab(q, k, v, off, nt, rab, 0.37, 11.0)
    assert _rel(got, ref) <= 1e-12, _rel(got, ref)


def pin_rab_constant_closed_form(o):
    """A constant bias c adds c * (sum of the visible values) / N to every row: history rows the
    prefix sum of v up to themselves, candidates the history sum plus their own v."""
    rng = np.random.default_rng(62)
    q, k, v, off, nt = _rand_batch(rng, [19, 33], [5, 3], 3, 4)
    c = 0.625
    rab = np.full((3, 4), c, np.float32)
    users = [b for b in range(2) for _ in range(int(off[b + 1] - off[b]))]
    local = [r for b in range(2) for r in range(int(off[b + 1] - off[b]))]
    got = o.rows_rab(q, k, v, off, nt, None, rab, 0.5, 7.0, users, local)
    base = o.fwd(q, k, v, off, nt, 0.5, 7.0)
    vs = np.zeros_like(base)
    for b in range(2):
        s0, s1 = int(off[b]), int(off[b + 1])
        U = (s1 - s0) - int(nt[b])
        vv = v[s0:s1].astype(np.float64)
        pref = np.cumsum(vv, axis=0)
        for i in range(s1 - s0):
            vs[s0 + i] = pref[i] if i < U else pref[U - 1] + vv[i]
    assert _rel(got, base + c * vs / 7.0) <= 1e-12


def pin_rab_zero_is_plain(o):
    """A zero bias table reproduces the plain oracle exactly."""
    rng = np.random.default_rng(63)
    q, k, v, off, nt = _rand_batch(rng, [40, 9], [6, 2], 2, 16)
    users = [b for b in range(2) for _ in range(int(off[b + 1] - off[b]))]
    local = [r for b in range(2) for r in range(int(off[b + 1] - off[b]))]
    got = o.rows_rab(q, k, v, off, nt, None, np.zeros((2, 3), np.float32), 0.2, 5.0, users, local)
    assert np.array_equal(got, o.fwd(q, k, v, off, nt, 0.2, 5.0))


def pin_rab_cached_equals_full(o):
    """Cached rows of the bias variant equal the same positions of the full computation."""
    rng = np.random.default_rng(64)
    q, k, v, off, nt = _rand_batch(rng, [31, 12], [5, 4], 2, 8)
    rab = rng.normal(size=(2, 9)).astype(np.float32)
    cl = np.array([20, 7], np.int32)
    users = [b for b in range(2) for _ in range(int(off[b + 1] - off[b] - cl[b]))]
    local = [r for b in range(2) for r in range(int(off[b + 1] - off[b] - cl[b]))]
    sel = np.concatenate([np.arange(off[b] + cl[b], off[b + 1]) for b in range(2)])
    got = o.rows_rab(q[sel], k, v, off, nt, cl, rab, 0.3, 9.0, users, local)
    full = bruteforce.attention_rab(q, k, v, off, nt, rab, 0.3, 9.0)[sel]
    assert _rel(got, full) <= 1e-12


ALL_PINS = [pin_rab_bruteforce, pin_rab_constant_closed_form, pin_rab_zero_is_plain, pin_rab_cached_equals_full,
            pin_bruteforce_tiny, pin_bruteforce_random, pin_closed_form_counts, pin_zero_query, pin_single_token,
            pin_linear_regime, pin_negative_regime, pin_small_score_taylor, pin_causal_textbook,
            pin_history_ignores_candidates, pin_candidates_independent, pin_cached_equals_full,
            pin_linearity_and_scale, pin_flop_formula]
