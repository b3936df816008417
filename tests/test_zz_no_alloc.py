"""GPU: hstu_attn_fwd_noalloc, the entry point for callers that cannot allocate device memory
during a call (for example a serving process whose own caching allocator has reserved the GPU's
memory, or a latency-critical loop where an allocator call could block).  Its plan lives in a
fixed 1 MiB device array inside the library instead of a pool buffer.

Checked through the C ABI: two calls on different batches are queued back to back on one stream,
each with its own output and no synchronisation between them, so the second call's plan kernel
rewrites the shared array right after the first call's attention kernel has read it.  Each output
must equal the allocating entry point's bit for bit (same kernels, same plan contents) and match
the fp64 oracle within the parity bars; a batch whose plan would not fit is refused before
anything runs.  This file is collected last so that a failure here never hides the other tests'
results; it passes both alone in a fresh process and after the rest of the suite.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_parity, dev_bf16, dev_i32, row_users, to_f64
from hstu_pointwise_attention_jagged_b200 import binding, workloads

pytestmark = pytest.mark.gpu


def _call_noalloc(lib, w, q, k, v, off, nt, cl, out):
    vp = ctypes.c_void_p
    total_q = q.shape[0]
    stream = vp(torch.cuda.current_stream().cuda_stream)
    return lib.hstu_attn_fwd_noalloc(vp(q.data_ptr()), vp(k.data_ptr()), vp(v.data_ptr()), vp(off.data_ptr()),
                                     vp(nt.data_ptr()), None if cl is None else vp(cl.data_ptr()), w.B, w.H, w.d,
                                     w.total, total_q, w.max_seq_len, w.alpha, w.N, vp(out.data_ptr()), stream)


def test_noalloc_matches_allocating_entry_point_twice_in_a_row():
    lib = binding.load_library()
    batches = [
        workloads.make_custom("na1", [700, 130, 0, 2000], [64, 2, 5, 300], 4, 128, 1 / math.sqrt(128), 2300.0,
                              seed=41),
        workloads.make_custom("na2", [90, 1500], [10, 7], 2, 64, 0.125, 1507.0, seed=42, cached_len=[30, 900]),
    ]
    calls = []
    for w in batches:
        k, v = dev_bf16(w.k), dev_bf16(w.v)
        off, nt = dev_i32(w.seq_offsets), dev_i32(w.num_targets)
        cached = bool(w.cached_len.any())
        q = dev_bf16(w.q[w.new_rows()])
        cl = dev_i32(w.cached_len) if cached else None
        ref = binding.hstu_attn_fwd_cached(q, k, v, off, nt, cl, w.alpha, w.N, w.max_seq_len)
        calls.append((w, q, k, v, off, nt, cl, ref, torch.full_like(q, float("nan"))))
    torch.cuda.synchronize()
    assert binding.hstu_attn_get_error() == 0
    # Both calls queued on one stream with no synchronisation between them.
    for w, q, k, v, off, nt, cl, ref, out in calls:
        assert _call_noalloc(lib, w, q, k, v, off, nt, cl, out) == 0
    torch.cuda.synchronize()
    assert binding.hstu_attn_get_error() == 0
    for w, q, k, v, off, nt, cl, ref, out in calls:
        assert torch.equal(out, ref), w.name
        cached = cl is not None
        if cached:
            want = oracle.fwd_cached(w.q[w.new_rows()], w.k, w.v, w.seq_offsets, w.num_targets, w.cached_len,
                                     w.alpha, w.N)
        else:
            want = oracle.fwd(w.q, w.k, w.v, w.seq_offsets, w.num_targets, w.alpha, w.N)
        assert_parity(to_f64(out), want, what="noalloc %s" % w.name, users=row_users(w, cached=cached))


def test_noalloc_refuses_batches_over_the_limit():
    lib = binding.load_library()
    vp = ctypes.c_void_p
    # H = 64 heads over 2M query rows needs a plan far beyond the fixed 1 MiB array.
    B, H, d, total = 4, 64, 64, 1 << 21
    assert lib.hstu_attn_plan_bytes(B, H, total) > (1 << 20)
    st = lib.hstu_attn_fwd_noalloc(vp(1 << 12), vp(1 << 12), vp(1 << 12), vp(1 << 12), None, None, B, H, d, total,
                                   total, total, 1.0, 1.0, vp(1 << 40), None)
    assert st == 2  # HSTU_ERR_UNSUPPORTED, returned before any GPU work
