"""GPU: sharding one jagged batch by user (hstu_attn_partition).  The runs of users are computed one
after another on one GPU, each with its own rebased seq_offsets as a separate call, and their
outputs, concatenated, equal the single call over the whole batch bit for bit: no row of one user
depends on another user, N is the same scalar in every call, and each row is computed by the same
kernel code whatever batch it sits in."""
import math

import numpy as np
import pytest
import torch

from gpu_util import dev_bf16, dev_i32
from hstu_pointwise_attention_jagged_b200 import binding, workloads

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("parts", [2, 3, 8])
def test_shards_concatenate_to_the_single_call(parts):
    w = workloads.make("jagged")
    q, k, v = dev_bf16(w.q), dev_bf16(w.k), dev_bf16(w.v)
    full = binding.hstu_attn_fwd(q, k, v, dev_i32(w.seq_offsets), dev_i32(w.num_targets), w.alpha, w.N,
                                 w.max_seq_len)
    us = binding.hstu_attn_partition(w.seq_offsets, w.num_targets, None, parts)
    pieces = []
    for p in range(parts):
        u0, u1, r0, r1, off = binding.shard_of(w.seq_offsets, us, p)
        if u1 == u0:
            continue
        pieces.append(binding.hstu_attn_fwd(q[r0:r1].contiguous(), k[r0:r1].contiguous(), v[r0:r1].contiguous(),
                                            dev_i32(off), dev_i32(w.num_targets[u0:u1]), w.alpha, w.N,
                                            w.max_seq_len))
    torch.cuda.synchronize()
    assert binding.hstu_attn_get_error() == 0
    assert torch.equal(torch.cat(pieces), full)
