"""GPU: the projection GEMM (hstu_attn_gemm_bf16) against the fp64 oracle, element by element, on
shapes with ragged M, N and K tails and on the DLRMv3 layer's projection shapes (sampled rows)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_parity, to_f64
from hstu_pointwise_attention_jagged_b200 import binding, workloads

pytestmark = pytest.mark.gpu


def _mats(M, N, K, seed):
    rng = np.random.default_rng(seed)
    a = workloads.round_bf16(rng.standard_normal((M, K), dtype=np.float32))
    w = workloads.round_bf16((rng.standard_normal((N, K), dtype=np.float32) / np.sqrt(K)).astype(np.float32))
    return a, w


def _dev(x):
    return torch.from_numpy(workloads.bf16_bits(x).view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("shape", [(1, 8, 8), (300, 264, 200), (129, 520, 72), (1000, 2048, 512), (777, 512, 1536)])
def test_gemm_tails(shape):
    M, N, K = shape
    a, w = _mats(M, N, K, seed=M + N + K)
    got = to_f64(binding.hstu_attn_gemm_bf16(_dev(a), _dev(w)))
    assert_parity(got, oracle.linear(a, w), what="gemm %s" % (shape,))
    assert binding.hstu_attn_get_error() == 0


@pytest.mark.parametrize("shape", [(32768, 2048, 512), (32768, 512, 1536)])
def test_gemm_layer_projection_shapes(shape):
    """The DLRMv3 layer's projections (L = 32768 tokens, D = H·d = 512): [L, D]·[D, 4D] and
    [L, 3D]·[3D, D]; 512 sampled rows, including the first and last tiles, against the oracle."""
    M, N, K = shape
    a, w = _mats(M, N, K, seed=5)
    c = binding.hstu_attn_gemm_bf16(_dev(a), _dev(w))
    rows = np.unique(np.concatenate([np.arange(0, 130), np.arange(M - 130, M),
                                     np.random.default_rng(6).integers(0, M, 252)]))
    got = to_f64(c[torch.from_numpy(rows).cuda()])
    assert_parity(got, oracle.linear(a[rows], w), what="gemm %s" % (shape,))
    assert torch.isfinite(c.float()).all()


@pytest.mark.parametrize("M", [200, 300])
def test_gemm_writes_nothing_outside_c(M):
    """Guard rows around C stay untouched (row- and column-predicated stores); M = 200 runs the one-SM
    kernel, M = 300 the two-SM kernel with a ragged last tile."""
    N, K = 264, 128
    a, w = _mats(M, N, K, seed=9)
    buf = torch.full((M + 2, N), 7.0, dtype=torch.bfloat16, device="cuda")
    binding.hstu_attn_gemm_bf16(_dev(a), _dev(w), out=buf[1:M + 1])
    assert torch.all(buf[0] == 7.0) and torch.all(buf[M + 1] == 7.0)
