"""CPU: the seeded synthetic workloads have the documented shapes, are reproducible, and are valid
inputs (lengths, targets, cached prefixes, bf16-representable values)."""
import math

import numpy as np
import pytest

from hstu_pointwise_attention_jagged_b200 import workloads

SHAPES = {  # name: (B, H, d, N)
    "tiny": (4, 2, 32, 68.0),
    "dlrmv3": (8, 4, 128, 4096.0),
    "jagged": (64, 4, 128, 4112.0),
    "long_history": (4, 8, 64, 8704.0),
    "streaming": (16, 4, 128, 5348.0),
}


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_shapes_and_validity(name):
    w = workloads.make(name)
    B, H, d, N = SHAPES[name]
    assert (w.B, w.H, w.d, w.N) == (B, H, d, N)
    assert w.q.shape == w.k.shape == w.v.shape == (w.total, H, d)
    assert w.seq_offsets[0] == 0 and np.all(np.diff(w.seq_offsets) >= 0)
    assert np.array_equal(np.diff(w.seq_offsets), w.uih_len + w.num_targets)
    assert np.all(w.cached_len >= 0) and np.all(w.cached_len <= w.uih_len)
    assert w.max_seq_len == int(np.diff(w.seq_offsets).max())
    assert math.isclose(w.alpha, 1 / math.sqrt(d)) or name == "long_history"
    if w.bf16:
        for x in (w.q, w.k, w.v):
            assert np.array_equal(workloads.round_bf16(x), x)


def test_named_workload_structure():
    j = workloads.make("jagged")
    assert np.all(j.uih_len >= 32) and np.all(j.uih_len <= 4096) and np.all(j.num_targets == 16)
    s = workloads.make("streaming")
    assert np.all(s.cached_len == 3000) and np.all(s.uih_len == 3300) and np.all(s.num_targets == 2048)
    assert s.total_q == int(s.total - s.cached_len.sum()) == len(s.new_rows())


def test_reproducible_and_seed_dependent():
    a, b = workloads.make("tiny"), workloads.make("tiny")
    assert np.array_equal(a.q, b.q) and np.array_equal(a.seq_offsets, b.seq_offsets)
    c = workloads.make("dlrmv3", seed=1001)
    assert not np.array_equal(workloads.make("dlrmv3").q[:64], c.q[:64])


def test_round_bf16_is_round_to_nearest_even():
    # 1 + 2^-8 lies halfway between two bf16 values (1 and 1 + 2^-7): ties go to the even mantissa, 1.
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 1.0 + 2.0 ** -9], np.float32)
    assert workloads.round_bf16(x).tolist() == [1.0, 1.0 + 2.0 ** -6, -1.0, 1.0]
