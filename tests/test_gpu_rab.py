"""GPU: the relative-attention-bias variant (hstu_attn_fwd_rab) against the oracle's
rows_rab / fwd_rab, element by element, on ragged, cached and full-size inputs."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_parity, dev_bf16, dev_i32, query_row_index, row_users, sample_rows, to_f64
from hstu_pointwise_attention_jagged_b200 import binding, workloads

pytestmark = pytest.mark.gpu


def _table(H, R, seed, scale=0.05):
    return np.random.default_rng(seed).normal(scale=scale, size=(H, R)).astype(np.float32)


def _run(w, rab, q=None, cached_len=None):
    return binding.hstu_attn_fwd_rab(dev_bf16(w.q) if q is None else q, dev_bf16(w.k), dev_bf16(w.v),
                                     dev_i32(w.seq_offsets), dev_i32(w.num_targets), torch.from_numpy(rab).cuda(),
                                     w.alpha, w.N, w.max_seq_len,
                                     cached_len=None if cached_len is None else dev_i32(cached_len))


@pytest.mark.parametrize("d", [32, 64, 128])
def test_rab_ragged(d):
    """Users from 0 to 900 tokens; the table (300 entries) is shorter than the longest distances,
    so clipping is exercised."""
    uih, nt = [1, 127, 0, 300, 700, 129], [0, 3, 2, 17, 200, 1]
    H = 3 if d == 32 else 2
    w = workloads.make_custom("rab%d" % d, uih, nt, H, d, 1 / math.sqrt(d), 900.0, seed=200 + d)
    rab = _table(H, 300, seed=d)
    got = to_f64(_run(w, rab))
    ref = oracle.fwd_rab(w.q, w.k, w.v, w.seq_offsets, w.num_targets, rab, w.alpha, w.N)
    assert_parity(got, ref, what="rab ragged d=%d" % d, users=row_users(w))


def test_rab_zero_table_is_plain_attention():
    """An all-zero table gives exactly the plain kernel's output (the bias adds +0.0)."""
    w = workloads.make_custom("rab0", [200, 64], [30, 5], 2, 128, 1 / math.sqrt(128), 300.0, seed=211)
    got = _run(w, np.zeros((2, 50), np.float32))
    plain = binding.hstu_attn_fwd(dev_bf16(w.q), dev_bf16(w.k), dev_bf16(w.v), dev_i32(w.seq_offsets),
                                  dev_i32(w.num_targets), w.alpha, w.N, w.max_seq_len)
    assert torch.equal(got, plain)


def test_rab_cached_matches_oracle_and_full():
    """Cached form: the bias uses positions from the segment start, so it equals the full form's rows."""
    w = workloads.make_custom("rabc", [400, 260, 90], [40, 17, 3], 2, 128, 1 / math.sqrt(128), 500.0,
                              cached_len=[250, 0, 60], seed=212)
    rab = _table(2, 512, seed=7)
    sel = w.new_rows()
    got = _run(w, rab, q=dev_bf16(w.q[sel]), cached_len=w.cached_len)
    ref = oracle.fwd_rab(w.q[sel], w.k, w.v, w.seq_offsets, w.num_targets, rab, w.alpha, w.N,
                         cached_len=w.cached_len)
    assert_parity(to_f64(got), ref, what="rab cached vs oracle", users=row_users(w, cached=True))
    full = _run(w, rab)
    assert_parity(to_f64(got), to_f64(full[torch.from_numpy(sel).cuda()]), what="rab cached vs full",
                  users=row_users(w, cached=True))


def test_rab_full_size_sampled():
    """The DLRMv3-shaped batch with a 4096-entry table; sampled rows against the oracle."""
    w = workloads.make("dlrmv3")
    rab = _table(w.H, 4096, seed=5, scale=0.02)
    got_all = _run(w, rab)
    users, local = sample_rows(w)
    rows = query_row_index(w, users, local)
    got = to_f64(got_all[torch.from_numpy(rows).cuda()])
    ref = oracle.rows_rab(w.q, w.k, w.v, w.seq_offsets, w.num_targets, None, rab, w.alpha, w.N, users, local)
    assert_parity(got, ref, what="rab dlrmv3", users=users)
    assert binding.hstu_attn_get_error() == 0
