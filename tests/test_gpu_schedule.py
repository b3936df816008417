"""GPU: the device-built work plan, bit-exact against an enumeration written from the mask's
definition (integer work: compared exactly; the order of equal keys is free, so the multiset is
compared and the order checked).  The plan takes users in waves by their first key row, each wave's K
and V about 32 MB at d = 128 (32 MiB / (512 bytes x H) rows), and orders items by wave, then by
non-increasing cost; a batch within one window is ordered by cost alone."""
import math

import numpy as np
import pytest
import torch

from gpu_util import dev_i32
from hstu_pointwise_attention_jagged_b200 import binding, workloads

pytestmark = pytest.mark.gpu


def visible_keys(i, U, L):
    """Keys query position i may see: history causal, candidates all history plus themselves."""
    if i < U:
        return range(0, i + 1)
    return list(range(0, U)) + [i]


def expected_items(seq_offsets, num_targets, cached_len, H):
    items = []
    for b in range(len(seq_offsets) - 1):
        L = int(seq_offsets[b + 1] - seq_offsets[b])
        T = int(num_targets[b]) if num_targets is not None else 0
        c = int(cached_len[b]) if cached_len is not None else 0
        U = L - T
        nq = L - c
        for blk in range(0, (nq + 127) // 128):
            r0 = blk * 128
            r1 = min(r0 + 128, nq)
            tiles = set()
            for r in range(r0, r1):
                tiles |= {j // 128 for j in visible_keys(c + r, U, L)}
            for h in range(H):
                items.append((b, blk, h, len(tiles)))
    return items


CASES = [
    ([1, 127, 128, 129, 0, 255, 256, 257, 1000], [0, 1, 2, 3, 0, 4, 0, 5, 300], None, 3),
    ([300, 513, 0, 700], [17, 0, 0, 129], [130, 0, 0, 200], 2),
    ([2048] * 8, [2048] * 8, None, 4),
    # more users than the plan kernel keeps on chip: its global-memory path
    (list(np.random.default_rng(41).integers(0, 700, 300)), list(np.random.default_rng(42).integers(0, 40, 300)),
     None, 2),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_schedule_matches_definition(case):
    uih, nt, cl, H = CASES[case]
    L = np.array(uih) + np.array(nt)
    off = workloads.offsets_from_lengths(L)
    total_kv = int(off[-1])
    cl_arr = None if cl is None else np.array(cl, np.int32)
    total_q = total_kv - (0 if cl is None else int(np.sum(cl)))
    plan = binding.hstu_attn_plan(dev_i32(off), dev_i32(nt), None if cl is None else dev_i32(cl), H, total_kv,
                                  total_q, int(L.max()))
    header, q_start, items = binding.plan_contents(plan, len(uih))
    got = [tuple(int(x) for x in r) for r in items]
    assert header[0] == 0 and header[2] == 0
    c = np.zeros(len(uih), np.int64) if cl is None else np.array(cl)
    assert q_start.tolist() == np.concatenate([[0], np.cumsum(L - c)[:-1]]).tolist()
    exp = expected_items(off, nt, cl_arr, H)
    assert sorted(got) == sorted(exp)
    max_len = int(L.max())
    nbins = min(2 * (max_len // 128 + 3) + 1, 4096)
    wave_rows = max((32 << 20) // (512 * H), 1)
    nwaves = max(min(4096 // nbins, -(-total_kv // wave_rows)), 1)
    keys = [(min(int(off[g[0]]) // wave_rows, nwaves - 1), -g[3]) for g in got]
    assert all(keys[i] <= keys[i + 1] for i in range(len(keys) - 1))
    assert binding.hstu_attn_get_error() == 0


def test_skipped_user_keeps_layout():
    """A user with inconsistent lengths is skipped (q_start = -1) but later users keep their rows."""
    off = workloads.offsets_from_lengths([100, 50, 70])
    nt = np.array([10, 60, 5], np.int32)  # user 1 claims more candidates than tokens
    plan = binding.hstu_attn_plan(dev_i32(off), dev_i32(nt), None, 2, 220, 220, 100)
    _, q_start, items = binding.plan_contents(plan, 3)
    assert q_start.tolist() == [0, -1, 150]
    assert sorted({int(r[0]) for r in items}) == [0, 2]
    assert binding.hstu_attn_get_error() == 4
