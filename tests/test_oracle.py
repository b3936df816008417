"""CPU: the fp64 oracle against its pins (see tests/oracle_pins.py), the jagged-layout golden
example from the TorchRec tutorial page, and the product's FLOP counter against the oracle."""
import json
import os

import numpy as np
import pytest

import oracle_pins
import bruteforce
from hstu_pointwise_attention_jagged_b200 import metrics, workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_oracle_pin(orc, pin):
    pin(orc)


def test_golden_jagged_layout(orc):
    """voagi.com TorchRec tutorial, section 2.1: 10 lengths (one zero) over 14 values."""
    g = json.load(open(os.path.join(GOLDEN, "jagged_lengths_page_example.json")))
    lengths, values = g["lengths"], g["values"]
    off = workloads.offsets_from_lengths(lengths)
    assert off.tolist() == [0, 1, 2, 3, 4, 5, 7, 10, 12, 14, 14]
    assert int(off[-1]) == len(values)
    segs = [values[off[b]:off[b + 1]] for b in range(len(lengths))]
    assert [len(s) for s in segs] == lengths and segs[-1] == []
    # The same lengths as a jagged attention batch (last token of each non-empty user a candidate).
    rng = np.random.default_rng(12)
    H, d = 2, 3
    q, k, v = (rng.standard_normal((14, H, d)).astype(np.float32) for _ in range(3))
    nt = np.array([min(1, n) for n in lengths], np.int32)
    got = orc.fwd(q, k, v, off, nt, 0.7, 3.0)
    ref = bruteforce.attention(q, k, v, off, nt, 0.7, 3.0)
    assert np.abs(got - ref).max() <= 1e-12
    # single-token users: out = silu(alpha q.k) v / N for their only (candidate) token
    s = 0.7 * float(np.dot(q[0, 0].astype(np.float64), k[0, 0].astype(np.float64)))
    assert np.allclose(got[0, 0], s / (1 + np.exp(-s)) * v[0, 0] / 3.0, rtol=1e-12)


def test_oracle_rejects_inconsistent_offsets(orc):
    q = np.zeros((4, 1, 2), np.float32)
    with pytest.raises(ValueError):
        orc.fwd(q, q, q, np.array([0, 3, 2, 4], np.int32), None, 1.0, 1.0)  # decreasing
    with pytest.raises(ValueError):
        orc.fwd(q, q, q, np.array([0, 4], np.int32), np.array([5], np.int32), 1.0, 1.0)  # T > L
    with pytest.raises(ValueError):
        orc.fwd_cached(q[:1], q, q, np.array([0, 4], np.int32), np.array([2], np.int32),
                       np.array([3], np.int32), 1.0, 1.0)  # cached prefix reaches a candidate


def test_oracle_thread_count_independent(orc, monkeypatch):
    """The oracle's result does not depend on how many threads computed it."""
    import oracle
    w = workloads.make("tiny")
    a = orc.fwd(w.q, w.k, w.v, w.seq_offsets, w.num_targets, w.alpha, w.N)
    r = oracle.rows(w.q, w.k, w.v, w.seq_offsets, w.num_targets, None, w.alpha, w.N,
                    np.repeat(np.arange(w.B), 3), np.tile([0, 5, 10], w.B))
    for n, (b, i) in enumerate(zip(np.repeat(np.arange(w.B), 3), np.tile([0, 5, 10], w.B))):
        assert np.array_equal(r[n], a[w.seq_offsets[b] + i])


@pytest.mark.parametrize("name", ["tiny"])
def test_metrics_flops_match_oracle_macs(orc, name):
    w = workloads.make(name)
    _, macs = orc.fwd(w.q, w.k, w.v, w.seq_offsets, w.num_targets, w.alpha, w.N, return_macs=True)
    assert metrics.algorithmic_flops(w.seq_offsets, w.num_targets, w.H, w.d) == 2 * macs


def test_metrics_flops_cached_match_oracle_macs(orc):
    rng = np.random.default_rng(13)
    lengths, targets, cl = [40, 17, 9, 0], [6, 17, 2, 0], [10, 0, 7, 0]
    off = workloads.offsets_from_lengths(lengths)
    H, d = 2, 4
    q, k, v = (rng.standard_normal((int(off[-1]), H, d)).astype(np.float32) for _ in range(3))
    sel = np.concatenate([np.arange(off[b] + cl[b], off[b + 1]) for b in range(4)])
    _, macs = orc.fwd_cached(q[sel], k, v, off, targets, cl, 1.0, 1.0, return_macs=True)
    assert metrics.algorithmic_flops(off, targets, H, d, cl) == 2 * macs


def test_metrics_named_workloads():
    """Algorithmic GFLOP of the named workloads (closed-form arithmetic, no oracle run)."""
    w = workloads.make("dlrmv3")
    f = metrics.algorithmic_flops(w.seq_offsets, w.num_targets, w.H, w.d)
    # 8 users x 4 heads x 4 x 128 x (2048*2049/2 + 2048*2049)
    assert f == 8 * 4 * 4 * 128 * (2048 * 2049 // 2 + 2048 * 2049)
    assert abs(f / 1e9 - 103.1) < 0.1
    assert metrics.page_attention_flops(2048, 512) == 2048 * 2048 * 512
