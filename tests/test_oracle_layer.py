"""CPU: pins of the oracle's HSTU layer (``oracle.layer`` / ``oracle.layers``) and of its bf16
storage rounding (``oracle.round_bf16``).

The layer (DLRMv3 review, section "model selection": per-layer flops 4 L D^2 + L^2 D / 2 + 3 L D^2;
infolabhq.com multi-stage page, "Target-Aware Multi-Head Attention": stacked blocks) is composed
of oracle.linear and oracle.fwd.  It is pinned against a dense NumPy restatement built from
independent pieces (plain matrix products and the dense brute-force attention of
tests/bruteforce.py) on tiny one- and two-layer cases; plausible mistakes (the Q and K blocks
swapped, the U*A term dropped, the gate taken from the V block) must each be rejected.
The rounding is pinned by worked ties and by torch's own float32 -> bfloat16 conversion.
"""
import numpy as np
import pytest
import torch

import bruteforce
import oracle


def test_round_bf16_worked_values():
    """bf16 keeps 7 fraction bits: 1 + 2^-8 is a tie and goes to the even 1.0; 1 + 3 * 2^-8 is a
    tie and goes to the even 1 + 2^-6; 1 + 2^-9 rounds down; signs and zeros are kept."""
    x = np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -1 - 2 ** -8, 1 + 2 ** -9, 1 + 3 * 2 ** -9, 0.0, -0.0], np.float32)
    want = [1.0, 1 + 2 ** -6, -1.0, 1.0, 1 + 2 ** -7, 0.0, -0.0]
    got = oracle.round_bf16(x)
    assert got.tolist() == want
    assert np.signbit(got[-1])


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(200000).astype(np.float32) * np.float32(50.0),
                        rng.standard_normal(1000).astype(np.float32) * np.float32(1e-38)])
    want = torch.from_numpy(x).to(torch.bfloat16).float().numpy()
    assert np.array_equal(oracle.round_bf16(x).astype(np.float32), want)


def _dense_layer(x, w1, w2, off, nt, H, d, alpha, N):
    """The layer restated with plain matrix products and the dense brute-force attention."""
    r = oracle.round_bf16
    total, D = x.shape
    uvqk = r(np.asarray(x, np.float64) @ np.asarray(w1, np.float64).T)
    u, v, q, k = uvqk[:, :D], uvqk[:, D:2 * D], uvqk[:, 2 * D:3 * D], uvqk[:, 3 * D:]
    a = r(bruteforce.attention(q.reshape(total, H, d), k.reshape(total, H, d), v.reshape(total, H, d), off, nt,
                               alpha, N).reshape(total, D))
    cat = np.concatenate([u, a, r(u * a)], axis=1)
    return cat @ np.asarray(w2, np.float64).T


def _case(seed, lengths, targets, H, d):
    rng = np.random.default_rng(seed)
    D = H * d
    off = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    total = int(off[-1])
    x = oracle.round_bf16(rng.standard_normal((total, D)))
    w1 = oracle.round_bf16(rng.standard_normal((4 * D, D)) / np.sqrt(D))
    w2 = oracle.round_bf16(rng.standard_normal((D, 3 * D)) / np.sqrt(3 * D))
    return x, w1, w2, off, np.asarray(targets, np.int32)


def pin_layer_dense(layer_fn):
    x, w1, w2, off, nt = _case(3, [9, 0, 5, 17], [3, 0, 5, 0], 2, 4)
    got = layer_fn(x, w1, w2, off, nt, 2, 4, 0.5, 20.0)
    want = _dense_layer(x, w1, w2, off, nt, 2, 4, 0.5, 20.0)
    assert got.shape == want.shape
    assert np.abs(got - want).max() <= 1e-12 * max(1.0, np.abs(want).max())


def pin_layer_single_token_user(layer_fn):
    """One user of one token: A = silu(alpha q.k) v / N per head, so Y follows in closed form."""
    x, w1, w2, off, nt = _case(4, [1], [1], 1, 4)
    r = oracle.round_bf16
    uvqk = r(x @ w1.T)
    u, v, q, k = (uvqk[:, 4 * i:4 * (i + 1)] for i in range(4))
    s = 0.5 * float(q[0] @ k[0])
    a = r(s / (1 + np.exp(-s)) * v / 7.0)
    want = np.concatenate([u, a, r(u * a)], axis=1) @ w2.T
    got = layer_fn(x, w1, w2, off, nt, 1, 4, 0.5, 7.0)
    assert np.allclose(got, want, rtol=1e-13, atol=1e-15)


LAYER_PINS = [pin_layer_dense, pin_layer_single_token_user]


def _swap_qk(x, w1, w2, off, nt, H, d, alpha, N):
    D = H * d
    w = np.concatenate([w1[:2 * D], w1[3 * D:], w1[2 * D:3 * D]])
    return oracle.layer(x, w, w2, off, nt, H, d, alpha, N)


def _no_gate_product(x, w1, w2, off, nt, H, d, alpha, N):
    D = H * d
    w = w2.copy()
    w[:, 2 * D:] = 0
    return oracle.layer(x, w1, w, off, nt, H, d, alpha, N)


def _gate_from_v(x, w1, w2, off, nt, H, d, alpha, N):
    D = H * d
    w = np.concatenate([w1[D:2 * D], w1[D:2 * D], w1[2 * D:]])
    return oracle.layer(x, w, w2, off, nt, H, d, alpha, N)


def _unrounded_attention(x, w1, w2, off, nt, H, d, alpha, N):
    r = oracle.round_bf16
    total, D = x.shape
    uvqk = r(oracle.linear(x, w1))
    u, v, q, k = (uvqk[:, i * D:(i + 1) * D] for i in range(4))
    a = oracle.fwd(q.reshape(total, H, d), k.reshape(total, H, d), v.reshape(total, H, d), off, nt, alpha,
                   N).reshape(total, D)
    return oracle.linear(np.concatenate([u, a, u * a], axis=1), w2)


MUTANTS = {"qk_swapped": _swap_qk, "no_gate_product": _no_gate_product, "gate_from_v": _gate_from_v,
           "unrounded_attention": _unrounded_attention}


@pytest.mark.parametrize("pin", LAYER_PINS, ids=lambda f: f.__name__)
def test_layer_pin(pin):
    pin(oracle.layer)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_layer_pins_reject_mutant(name):
    caught = []
    for pin in LAYER_PINS:
        try:
            pin(MUTANTS[name])
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, "no pin rejects the layer mutant %s" % name


def test_layers_is_the_composition():
    """Two stacked layers equal the dense restatement applied twice with a bf16 hidden activation."""
    x, w1, w2, off, nt = _case(5, [6, 11], [2, 0], 2, 4)
    _, w1b, w2b, _, _ = _case(6, [6, 11], [2, 0], 2, 4)
    got = oracle.layers(x, [w1, w1b], [w2, w2b], off, nt, 2, 4, 0.6, 12.0)
    h = oracle.round_bf16(_dense_layer(x, w1, w2, off, nt, 2, 4, 0.6, 12.0))
    want = _dense_layer(h, w1b, w2b, off, nt, 2, 4, 0.6, 12.0)
    assert np.abs(got - want).max() <= 1e-12 * max(1.0, np.abs(want).max())
