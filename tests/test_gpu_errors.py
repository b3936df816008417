"""GPU: error reporting.  Inconsistent lengths are detected on the device, reported through
hstu_attn_get_error, and the offending users are skipped while the others are computed; bad
arguments are rejected synchronously."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_parity, dev_bf16, dev_i32, row_users, to_f64
from hstu_pointwise_attention_jagged_b200 import binding, workloads

pytestmark = pytest.mark.gpu


def test_clean_call_reports_ok():
    w = workloads.make_custom("ok", [100, 50], [3, 2], 2, 64, 0.125, 103.0, seed=31)
    binding.hstu_attn_fwd(dev_bf16(w.q), dev_bf16(w.k), dev_bf16(w.v), dev_i32(w.seq_offsets),
                          dev_i32(w.num_targets), w.alpha, w.N, w.max_seq_len)
    assert binding.hstu_attn_get_error() == 0


def test_bad_targets_skip_user_and_report():
    """User 1 claims more candidates than tokens: it is skipped, users 0 and 2 are still right."""
    w = workloads.make_custom("bad", [150, 60, 90], [10, 5, 4], 2, 128, 1 / math.sqrt(128), 160.0, seed=32)
    bad_nt = w.num_targets.copy()
    bad_nt[1] = 1000
    out = torch.full((w.total, w.H, w.d), 5.0, dtype=torch.bfloat16, device="cuda")
    binding.hstu_attn_fwd(dev_bf16(w.q), dev_bf16(w.k), dev_bf16(w.v), dev_i32(w.seq_offsets), dev_i32(bad_nt),
                          w.alpha, w.N, w.max_seq_len, out=out)
    assert binding.hstu_attn_get_error() == 4  # HSTU_ERR_BAD_OFFSETS
    assert binding.hstu_attn_get_error() == 0  # cleared by the read
    ref = oracle.fwd(w.q, w.k, w.v, w.seq_offsets, w.num_targets, w.alpha, w.N)
    o = to_f64(out)
    s = w.seq_offsets
    assert np.all(o[s[1]:s[2]] == 5.0)
    keep = np.r_[s[0]:s[1], s[2]:s[3]]
    assert_parity(o[keep], ref[keep], what="valid users", users=row_users(w)[keep])


def test_user_longer_than_max_seq_len_is_skipped():
    w = workloads.make_custom("long", [300, 20], [0, 0], 1, 64, 0.125, 300.0, seed=33)
    out = torch.full((w.total, 1, 64), 5.0, dtype=torch.bfloat16, device="cuda")
    binding.hstu_attn_fwd(dev_bf16(w.q), dev_bf16(w.k), dev_bf16(w.v), dev_i32(w.seq_offsets), None,
                          w.alpha, w.N, 100, out=out)
    assert binding.hstu_attn_get_error() == 4
    assert torch.all(out[:300] == 5.0)
    ref = oracle.fwd(w.q, w.k, w.v, w.seq_offsets, None, w.alpha, w.N)
    assert_parity(to_f64(out[300:]), ref[300:], what="short user", users=row_users(w)[300:])


def test_cached_prefix_into_candidates_is_rejected():
    w = workloads.make_custom("cbad", [100, 80], [20, 10], 1, 64, 0.125, 120.0, seed=34, cached_len=[0, 0])
    cl = np.array([110, 0], np.int32)  # reaches into user 0's candidates
    q_new = dev_bf16(w.q[np.r_[110:120, 120:210]])
    out = torch.full((100, 1, 64), 5.0, dtype=torch.bfloat16, device="cuda")
    binding.hstu_attn_fwd_cached(q_new, dev_bf16(w.k), dev_bf16(w.v), dev_i32(w.seq_offsets),
                                 dev_i32(w.num_targets), dev_i32(cl), w.alpha, w.N, 120, out=out)
    assert binding.hstu_attn_get_error() == 4


def test_synchronous_argument_errors():
    q = torch.zeros((16, 2, 48), dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, 16], dtype=torch.int32, device="cuda")
    with pytest.raises(binding.HstuError) as e:
        binding.hstu_attn_fwd(q, q, q, off, None, 1.0, 1.0, 16)
    assert e.value.status == 2
    q = torch.zeros((16, 2, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.HstuError) as e:
        binding.hstu_attn_fwd(q, q, q, off, None, 1.0, 0.0, 16)
    assert e.value.status == 1
    with pytest.raises(binding.HstuError) as e:
        binding.hstu_attn_fwd(q, q, q, off, None, 1.0, 1.0, 16, out=q)
    assert e.value.status == 1


def test_bounded_wait_times_out_and_reports():
    """The bounded mbarrier wait every role of the attention kernel uses gives up on a barrier
    that nothing arrives on: the kernel returns, the device reports HSTU_ERR_TIMEOUT once, and
    the context still computes correct results afterwards (no trap, no hang)."""
    assert binding.hstu_attn_get_error() == 0
    binding.hstu_attn_selfcheck_wait_timeout(2_000_000)  # 2 ms
    assert binding.hstu_attn_get_error() == 5  # HSTU_ERR_TIMEOUT
    assert binding.hstu_attn_get_error() == 0  # cleared by the read
    w = workloads.make_custom("after_timeout", [130, 40], [6, 3], 2, 64, 0.125, 140.0, seed=33)
    out = binding.hstu_attn_fwd(dev_bf16(w.q), dev_bf16(w.k), dev_bf16(w.v), dev_i32(w.seq_offsets),
                                dev_i32(w.num_targets), w.alpha, w.N, w.max_seq_len)
    assert binding.hstu_attn_get_error() == 0
    ref = oracle.fwd(w.q, w.k, w.v, w.seq_offsets, w.num_targets, w.alpha, w.N)
    assert_parity(to_f64(out), ref, what="after a timed-out self-check", users=row_users(w))


def test_selfcheck_rejects_out_of_range_limits():
    for bad in (0, 2_000_000_000):
        with pytest.raises(binding.HstuError):
            binding.hstu_attn_selfcheck_wait_timeout(bad)


def test_corrupt_lengths_near_int_max_write_nothing_outside_out():
    """Two corrupt users whose lengths are about 2^31 rows, then a well-formed user.  The plan
    kernel takes lengths in 64 bits and caps a corrupt user's rows, so no query-row start wraps
    negative: the call reports HSTU_ERR_BAD_OFFSETS, no work item points outside `out`, and the
    guard rows on both sides of `out` keep their sentinel."""
    off = np.array([0, 2147483000, -5, 2147483000, 0, 100], np.int32)
    nt = np.zeros(5, np.int32)
    H, d, total = 2, 64, 100
    plan = binding.hstu_attn_plan(dev_i32(off), dev_i32(nt), None, H, total, total, 100)
    _, q_start, items = binding.plan_contents(plan, 5)
    assert binding.hstu_attn_get_error() == 4
    assert all(int(s) == -1 or 0 <= int(s) < total for s in q_start)
    for it in items:
        assert 0 <= int(q_start[int(it[0])]) < total
    rng = np.random.default_rng(35)
    q = dev_bf16(workloads.round_bf16(rng.standard_normal((total, H, d), dtype=np.float32) / 8))
    pad = 256
    big = torch.full((total + 2 * pad, H, d), 7.0, dtype=torch.bfloat16, device="cuda")
    binding.hstu_attn_fwd(q, q, q, dev_i32(off), dev_i32(nt), 0.125, 100.0, 100, out=big[pad:pad + total])
    torch.cuda.synchronize()
    assert binding.hstu_attn_get_error() == 4
    assert torch.all(big[:pad] == 7.0) and torch.all(big[pad + total:] == 7.0)


def test_attention_kernel_abort_path_then_recovers():
    """The attention kernel itself with every pipeline wait limited to 1 µs: the waits that are not
    met at once run out, the CTAs raise their abort flag, drain the copies and MMAs they issued,
    free TMEM and return.  The device reports HSTU_ERR_TIMEOUT once, and a normal call on the same
    context afterwards matches the oracle."""
    w = workloads.make_custom("abort", [600, 300, 40], [100, 20, 2], 2, 128, 1 / math.sqrt(128), 700.0, seed=36)
    q, k, v = dev_bf16(w.q), dev_bf16(w.k), dev_bf16(w.v)
    off, nt = dev_i32(w.seq_offsets), dev_i32(w.num_targets)
    assert binding.hstu_attn_get_error() == 0
    for _ in range(2):
        binding.hstu_attn_selfcheck_fwd_timeout(q, k, v, off, nt, w.alpha, w.N, w.max_seq_len, 1000)
        assert binding.hstu_attn_get_error() == 5  # HSTU_ERR_TIMEOUT
        assert binding.hstu_attn_get_error() == 0
    out = binding.hstu_attn_fwd(q, k, v, off, nt, w.alpha, w.N, w.max_seq_len)
    assert binding.hstu_attn_get_error() == 0
    ref = oracle.fwd(w.q, w.k, w.v, w.seq_offsets, w.num_targets, w.alpha, w.N)
    assert_parity(to_f64(out), ref, what="after an aborted attention kernel", users=row_users(w))
