"""GPU: the HSTU layer (hstu_layer_fwd, hstu_layers_fwd: projection GEMM, attention reading Q, K, V in
place with the [U | A | U*A] epilogue, projection GEMM) against the oracle's layer (oracle.layer,
composed of the pinned oracle.linear and oracle.fwd with bf16 storage of the stored tensors).

- one layer on a ragged batch and on the DLRMv3-shaped batch (D = 512), every output compared;
- a stack of three layers: the one-call stack equals three single-layer calls on one plan bit for
  bit, each layer matches the oracle layer applied to that layer's GPU input (the parity bar), and
  the stack matches the oracle stack within 1e-2 (three layers of bf16 storage: each adds about
  3e-3 of independent relative error).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_parity, dev_i32, row_users, to_f64
from hstu_pointwise_attention_jagged_b200 import binding, workloads

pytestmark = pytest.mark.gpu


def _bf16_dev(a):
    a32 = oracle.round_bf16(a).astype(np.float32)
    return torch.from_numpy(workloads.bf16_bits(a32).view(np.int16)).view(torch.bfloat16).cuda()


def _weights(rng, H, d, layers):
    D = H * d
    w1 = [oracle.round_bf16(rng.standard_normal((4 * D, D)) / np.sqrt(D)) for _ in range(layers)]
    w2 = [oracle.round_bf16(rng.standard_normal((D, 3 * D)) / np.sqrt(3 * D)) for _ in range(layers)]
    return w1, w2


def _users(w):
    return row_users(w)


@pytest.mark.parametrize("shape", [("ragged", [300, 1, 0, 700, 129], [20, 0, 3, 129, 1], 2, 64),
                                   ("ragged128", [257, 40], [5, 300], 4, 128)])
def test_one_layer_ragged(shape):
    name, uih, nt, H, d = shape
    w = workloads.make_custom(name, uih, nt, H, d, 1 / math.sqrt(d), float(max(u + t for u, t in zip(uih, nt))),
                              seed=500)
    rng = np.random.default_rng(501)
    D = H * d
    x = oracle.round_bf16(rng.standard_normal((w.total, D)))
    w1, w2 = _weights(rng, H, d, 1)
    off, ntd = dev_i32(w.seq_offsets), dev_i32(w.num_targets)
    plan = binding.hstu_attn_plan(off, ntd, None, H, w.total, w.total, w.max_seq_len)
    y = binding.hstu_layer_fwd(_bf16_dev(x), _bf16_dev(w1[0]), _bf16_dev(w2[0]), off, ntd, H, d, w.alpha, w.N, plan)
    torch.cuda.synchronize()
    assert binding.hstu_attn_get_error() == 0
    want = oracle.layer(x, w1[0], w2[0], w.seq_offsets, w.num_targets, H, d, w.alpha, w.N)
    assert_parity(to_f64(y), want, what="layer %s" % name, users=_users(w))


def test_one_layer_dlrmv3_shapes():
    """The DLRMv3-shaped batch (32768 tokens, D = H d = 512): every output row against the oracle."""
    w = workloads.make("dlrmv3")
    H, d = w.H, w.d
    rng = np.random.default_rng(502)
    x = oracle.round_bf16(rng.standard_normal((w.total, H * d)))
    w1, w2 = _weights(rng, H, d, 1)
    y = binding.hstu_layers_fwd(_bf16_dev(x), [_bf16_dev(w1[0])], [_bf16_dev(w2[0])], dev_i32(w.seq_offsets),
                                dev_i32(w.num_targets), H, d, w.alpha, w.N, w.max_seq_len)
    torch.cuda.synchronize()
    assert binding.hstu_attn_get_error() == 0
    want = oracle.layer(x, w1[0], w2[0], w.seq_offsets, w.num_targets, H, d, w.alpha, w.N)
    assert_parity(to_f64(y), want, what="layer dlrmv3", users=_users(w))


def test_three_layer_stack():
    w = workloads.make_custom("stack", [400, 130, 60], [40, 3, 60], 2, 64, 0.125, 500.0, seed=503)
    H, d = w.H, w.d
    rng = np.random.default_rng(504)
    x = oracle.round_bf16(rng.standard_normal((w.total, H * d)))
    w1, w2 = _weights(rng, H, d, 3)
    w1d, w2d = [_bf16_dev(a) for a in w1], [_bf16_dev(a) for a in w2]
    off, ntd = dev_i32(w.seq_offsets), dev_i32(w.num_targets)
    stack = binding.hstu_layers_fwd(_bf16_dev(x), w1d, w2d, off, ntd, H, d, w.alpha, w.N, w.max_seq_len)
    plan = binding.hstu_attn_plan(off, ntd, None, H, w.total, w.total, w.max_seq_len)
    h = _bf16_dev(x)
    for l in range(3):
        h_in = h
        h = binding.hstu_layer_fwd(h_in, w1d[l], w2d[l], off, ntd, H, d, w.alpha, w.N, plan)
        torch.cuda.synchronize()
        want = oracle.layer(to_f64(h_in), w1[l], w2[l], w.seq_offsets, w.num_targets, H, d, w.alpha, w.N)
        assert_parity(to_f64(h), want, what="stack layer %d" % l, users=_users(w))
    assert binding.hstu_attn_get_error() == 0
    assert torch.equal(stack, h)
    want = oracle.layers(x, w1, w2, w.seq_offsets, w.num_targets, H, d, w.alpha, w.N)
    assert_parity(to_f64(stack), want, rel=1e-2, what="stack of 3 vs oracle stack", users=_users(w))
