"""CPU: hstu_attn_partition, the split of one jagged batch into contiguous per-GPU runs of users
(host function of the C library; no GPU needed).

- the largest per-GPU cost equals the optimum found by enumerating every contiguous split
  (integer work: compared exactly), on random small batches, with cached prefixes and empty users;
- a user's cost is its number of visible (query, key) pairs, the mask-exact attention work;
- two gloo ranks each take their run of a jagged batch, rebase its offsets and run the CPU-side
  path (the oracle) on it; the gathered rows equal the full batch's rows bit for bit, because no
  row of one user depends on another user.
"""
import itertools
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cost(L, T, c):
    """Visible pairs of one user, counted one query at a time from the mask's definition."""
    U = L - T
    return sum((i + 1) if i < U else (U + 1) for i in range(c, L))


def _best_max(costs, parts):
    """Smallest achievable largest part over every split into `parts` contiguous (possibly empty) runs."""
    B = len(costs)
    best = None
    for cuts in itertools.combinations_with_replacement(range(B + 1), parts - 1):
        bounds = (0,) + cuts + (B,)
        m = max(sum(costs[bounds[p]:bounds[p + 1]]) for p in range(parts))
        best = m if best is None else min(best, m)
    return best


def test_partition_is_optimal_on_small_batches(cuda_lib):
    from hstu_pointwise_attention_jagged_b200 import binding, workloads
    rng = np.random.default_rng(5)
    for trial in range(60):
        B = int(rng.integers(1, 8))
        parts = int(rng.integers(1, 5))
        L = rng.integers(0, 300, B)
        T = np.array([int(rng.integers(0, l + 1)) for l in L])
        c = np.array([int(rng.integers(0, l - t + 1)) if trial % 2 else 0 for l, t in zip(L, T)])
        off = workloads.offsets_from_lengths(L)
        us = binding.hstu_attn_partition(off, T, c, parts)
        assert us[0] == 0 and us[-1] == B and np.all(np.diff(us) >= 0), us
        costs = [_cost(int(l), int(t), int(cc)) for l, t, cc in zip(L, T, c)]
        got = max(sum(costs[us[p]:us[p + 1]]) for p in range(parts))
        assert got == _best_max(costs, parts), (L, T, c, parts, us)


def test_partition_uniform_batch_splits_evenly(cuda_lib):
    from hstu_pointwise_attention_jagged_b200 import binding, workloads
    for n in (1, 2, 4, 8):
        L = np.full(8 * n, 4096)
        T = np.full(8 * n, 2048)
        us = binding.hstu_attn_partition(workloads.offsets_from_lengths(L), T, None, n)
        assert us.tolist() == [8 * p for p in range(n + 1)]


def test_partition_rejects_inconsistent_lengths(cuda_lib):
    from hstu_pointwise_attention_jagged_b200 import binding
    with pytest.raises(binding.HstuError) as e:
        binding.hstu_attn_partition(np.array([0, 10, 20], np.int32), np.array([0, 11], np.int32), None, 2)
    assert e.value.status == 4
    with pytest.raises(binding.HstuError):
        binding.hstu_attn_partition(np.array([0, 10], np.int32), None, None, 0)


def test_shard_of_rebases_offsets(cuda_lib):
    from hstu_pointwise_attention_jagged_b200 import binding
    off = np.array([0, 5, 5, 12, 20], np.int32)
    u0, u1, r0, r1, o = binding.shard_of(off, np.array([0, 2, 4]), 1)
    assert (u0, u1, r0, r1) == (2, 4, 5, 20) and o.tolist() == [0, 7, 15]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime

    import torch.distributed as dist

    import oracle
    from hstu_pointwise_attention_jagged_b200 import binding, workloads
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    # the same batch on every rank (lengths and values from one seed)
    w = workloads.make_custom("shard", [40, 3, 0, 77, 12, 60, 9], [5, 3, 0, 7, 0, 20, 1], 2, 16, 0.25, 100.0, seed=3)
    us = binding.hstu_attn_partition(w.seq_offsets, w.num_targets, None, world)
    u0, u1, r0, r1, off = binding.shard_of(w.seq_offsets, us, rank)
    out = oracle.fwd(w.q[r0:r1], w.k[r0:r1], w.v[r0:r1], off, w.num_targets[u0:u1], w.alpha, w.N)
    gathered = [None] * world
    dist.all_gather_object(gathered, (rank, r0, r1, out))
    if rank == 0:
        full = oracle.fwd(w.q, w.k, w.v, w.seq_offsets, w.num_targets, w.alpha, w.N)
        rows = np.concatenate([g[3] for g in sorted(gathered, key=lambda g: g[0])])
        q.put((bool(np.array_equal(rows, full)), [g[1:3] for g in sorted(gathered, key=lambda g: g[0])]))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_one_batch(cuda_lib):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    equal, ranges = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert equal
    assert ranges[0][0] == 0 and ranges[0][1] == ranges[1][0] and ranges[1][1] == 201 + 36  # all rows
