"""GPU parity of the backward pass (hstu_attn_bwd, through the C ABI) against the fp64 oracle's
backward (oracle.bwd / oracle.bwd_rows, derived from the forward by the chain rule and pinned by
finite differences on the CPU).

- small ragged batches for every head size, compared element by element over all of dq, dk, dv:
  lengths around the 128-row tiles, zero-length, history-only and candidate-only users;
- the DLRMv3-shaped batch at full size, compared on sampled rows (tile edges, the history /
  candidate boundary, both ends, random rows);
- determinism, and no writes outside the users' rows.
Bar: the forward's (relative L2 <= 5e-3 over each gradient, every user within it, every row within
2e-2, max abs <= 3e-2); P and dS are rounded to bf16 before their products, like P in the forward.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_parity, dev_bf16, dev_i32, row_users, sample_rows, to_f64
from hstu_pointwise_attention_jagged_b200 import binding, workloads

pytestmark = pytest.mark.gpu


def _dout(w, seed):
    rng = np.random.default_rng(seed)
    return workloads.round_bf16(rng.standard_normal(w.q.shape, dtype=np.float32))


def _run(w, do, **kw):
    got = binding.hstu_attn_bwd(dev_bf16(w.q), dev_bf16(w.k), dev_bf16(w.v), dev_bf16(do), dev_i32(w.seq_offsets),
                                dev_i32(w.num_targets), w.alpha, w.N, max(w.max_seq_len, 1), **kw)
    torch.cuda.synchronize()
    return got


RAGGED = [
    ([1, 127, 128, 129, 0, 255, 256, 257], [0, 1, 2, 3, 0, 4, 0, 5]),
    ([300, 513, 0, 700, 64], [17, 0, 0, 129, 64]),
    ([0, 0, 5, 1000], [130, 1, 0, 300]),
]


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("case", range(len(RAGGED)))
def test_bwd_ragged(d, case):
    uih, nt = RAGGED[case]
    H = 3 if d == 32 else 2
    w = workloads.make_custom("bwd%d" % case, uih, nt, H, d, 1 / math.sqrt(d),
                              float(max(u + t for u, t in zip(uih, nt))), seed=300 + case)
    do = _dout(w, 400 + case)
    got = _run(w, do)
    want = oracle.bwd(w.q, w.k, w.v, do, w.seq_offsets, w.num_targets, w.alpha, w.N)
    assert binding.hstu_attn_get_error() == 0
    for name, g, r in zip(("dq", "dk", "dv"), got, want):
        assert_parity(to_f64(g), r, what="bwd %s ragged %d d=%d" % (name, case, d), users=row_users(w))


def test_bwd_tiny_config():
    w = workloads.make("tiny")
    w.q, w.k, w.v = (workloads.round_bf16(x) for x in (w.q, w.k, w.v))
    do = _dout(w, 7)
    got = _run(w, do)
    want = oracle.bwd(w.q, w.k, w.v, do, w.seq_offsets, w.num_targets, w.alpha, w.N)
    for name, g, r in zip(("dq", "dk", "dv"), got, want):
        assert_parity(to_f64(g), r, what="bwd %s tiny" % name, users=row_users(w))


def test_bwd_stress_large_scores():
    """Unscaled N(0,1) inputs with alpha = 1: scores deep into both SiLU tails."""
    w = workloads.make_custom("bwdstress", [190, 31, 260], [20, 5, 1], 2, 64, 1.0, 64.0, seed=9, scale=1.0)
    do = _dout(w, 8)
    got = _run(w, do)
    want = oracle.bwd(w.q, w.k, w.v, do, w.seq_offsets, w.num_targets, w.alpha, w.N)
    for name, g, r in zip(("dq", "dk", "dv"), got, want):
        assert_parity(to_f64(g), r, max_abs=1e-2 * np.abs(r).max(), what="bwd %s stress" % name, users=row_users(w))


def test_bwd_dlrmv3_sampled():
    """The DLRMv3-shaped batch at full size; sampled rows of every gradient against the oracle."""
    w = workloads.make("dlrmv3")
    do = _dout(w, 9)
    got = _run(w, do)
    assert binding.hstu_attn_get_error() == 0
    users, local = sample_rows(w, per_user_random=12)
    rows = torch.from_numpy(w.seq_offsets[users] + local).cuda()
    want = oracle.bwd_rows(w.q, w.k, w.v, do, w.seq_offsets, w.num_targets, w.alpha, w.N, users, local)
    for name, g, r in zip(("dq", "dk", "dv"), got, want):
        assert torch.isfinite(g.float()).all()
        assert_parity(to_f64(g[rows]), r, what="bwd %s dlrmv3" % name, users=users)


def test_bwd_deterministic_and_guarded():
    """Two calls give identical gradients; guard rows around every gradient stay untouched."""
    w = workloads.make_custom("bwdguard", [129, 0, 250], [3, 0, 6], 2, 128, 1 / math.sqrt(128), 256.0, seed=25)
    do = _dout(w, 10)
    a = _run(w, do)
    pad = 64
    bigs = [torch.full((w.total + 2 * pad, w.H, w.d), 7.0, dtype=torch.bfloat16, device="cuda") for _ in range(3)]
    b = _run(w, do, dq=bigs[0][pad:pad + w.total], dk=bigs[1][pad:pad + w.total], dv=bigs[2][pad:pad + w.total])
    for x, y, big in zip(a, b, bigs):
        assert torch.equal(x, y)
        assert torch.all(big[:pad] == 7.0) and torch.all(big[pad + w.total:] == 7.0)
    assert binding.hstu_attn_get_error() == 0


@pytest.mark.parametrize("d", [32, 64, 128])
def test_bwd_stored_ds_path_matches_recompute_path(d):
    """hstu_attn_bwd with its dS workspace (dq from the stored dS tiles) and with the workspace limit
    at 0 (the dQ kernel recomputes S, dP and dS): both match the oracle, dk and dv are bitwise
    equal (same kernel), and the two dq agree to fp32 accumulation order."""
    uih, nt = RAGGED[1]
    w = workloads.make_custom("bwdws%d" % d, uih, nt, 2, d, 1 / math.sqrt(d),
                              float(max(u + t for u, t in zip(uih, nt))), seed=500 + d)
    do = _dout(w, 600 + d)
    stored = _run(w, do)
    previous = binding.hstu_attn_bwd_workspace_limit(0)
    try:
        recomputed = _run(w, do)
    finally:
        binding.hstu_attn_bwd_workspace_limit(previous)
    assert binding.hstu_attn_get_error() == 0
    want = oracle.bwd(w.q, w.k, w.v, do, w.seq_offsets, w.num_targets, w.alpha, w.N)
    for path, got in (("stored dS", stored), ("recomputed dS", recomputed)):
        for name, g, r in zip(("dq", "dk", "dv"), got, want):
            assert_parity(to_f64(g), r, what="bwd %s %s d=%d" % (name, path, d), users=row_users(w))
    assert torch.equal(stored[1], recomputed[1]) and torch.equal(stored[2], recomputed[2])
    a, b = stored[0].double(), recomputed[0].double()
    assert float((a - b).norm() / b.norm()) <= 1e-2 * 2.0 ** -8  # a few bf16 ulps at most, by accumulation order
