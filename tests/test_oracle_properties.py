"""CPU: property-based checks of the oracle on random small jagged batches (hypothesis).

For every drawn batch (users of 0..24 tokens, any number of candidates, any history-only cached
prefix, 1..3 heads, random bias tables), the oracle's rows equal the dense restatement in
tests/bruteforce.py, plain and with the relative bias, and the cached form equals the matching rows
of the full form."""
import numpy as np
from hypothesis import given, settings, strategies as st

import bruteforce
import oracle
from hstu_pointwise_attention_jagged_b200 import workloads


@st.composite
def batches(draw):
    B = draw(st.integers(1, 4))
    L = [draw(st.integers(0, 24)) for _ in range(B)]
    T = [draw(st.integers(0, l)) for l in L]
    C = [draw(st.integers(0, l - t)) for l, t in zip(L, T)]
    H = draw(st.integers(1, 3))
    d = draw(st.sampled_from([1, 4, 8]))
    R = draw(st.integers(1, 30))
    seed = draw(st.integers(0, 2**31 - 1))
    return L, T, C, H, d, R, seed


def _inputs(L, T, H, d, R, seed):
    rng = np.random.default_rng(seed)
    off = workloads.offsets_from_lengths(L)
    total = int(off[-1])
    q = rng.standard_normal((total, H, d)).astype(np.float32)
    k = rng.standard_normal((total, H, d)).astype(np.float32)
    v = rng.standard_normal((total, H, d)).astype(np.float32)
    rab = rng.normal(size=(H, R)).astype(np.float32)
    return off, np.asarray(T, np.int32), q, k, v, rab


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@settings(max_examples=60, deadline=None)
@given(batches())
def test_oracle_matches_dense_restatement(batch):
    L, T, C, H, d, R, seed = batch
    off, nt, q, k, v, rab = _inputs(L, T, H, d, R, seed)
    alpha, N = 0.7, 3.0
    got = oracle.fwd(q, k, v, off, nt, alpha, N)
    assert _rel(got, bruteforce.attention(q, k, v, off, nt, alpha, N)) <= 1e-12
    got_rab = oracle.fwd_rab(q, k, v, off, nt, rab, alpha, N)
    assert _rel(got_rab, bruteforce.attention_rab(q, k, v, off, nt, rab, alpha, N)) <= 1e-12


@settings(max_examples=60, deadline=None)
@given(batches())
def test_cached_rows_equal_full_rows(batch):
    L, T, C, H, d, R, seed = batch
    off, nt, q, k, v, rab = _inputs(L, T, H, d, R, seed)
    cl = np.asarray(C, np.int32)
    sel = np.concatenate([np.arange(off[b] + cl[b], off[b + 1]) for b in range(len(L))]).astype(np.int64)
    full = oracle.fwd(q, k, v, off, nt, 0.5, 2.0)
    cached = oracle.fwd_cached(q[sel], k, v, off, nt, cl, 0.5, 2.0)
    assert np.array_equal(cached, full[sel])
    full_rab = oracle.fwd_rab(q, k, v, off, nt, rab, 0.5, 2.0)
    cached_rab = oracle.fwd_rab(q[sel], k, v, off, nt, rab, 0.5, 2.0, cached_len=cl)
    assert np.array_equal(cached_rab, full_rab[sel])
