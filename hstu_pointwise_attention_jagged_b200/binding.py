"""ctypes binding of libhstu_attn.so (C ABI: include/hstu_attn.h).

Argument marshalling only: every function checks the torch tensors it is given, passes their
device pointers, sizes and the current CUDA stream to the C entry point of the same name, and
raises :class:`HstuError` on a non-zero status.  All arithmetic happens in the library's CUDA
kernels; there is no other code path.  If the library has not been built the first call raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libhstu_attn.so")
_lib = None

STATUS = {
    0: "HSTU_OK",
    1: "HSTU_ERR_INVALID_ARGUMENT",
    2: "HSTU_ERR_UNSUPPORTED",
    3: "HSTU_ERR_CUDA",
    4: "HSTU_ERR_BAD_OFFSETS",
    5: "HSTU_ERR_TIMEOUT",
}

# Every symbol include/hstu_attn.h declares.
EXPORTS = (
    "hstu_attn_fwd",
    "hstu_attn_fwd_cached",
    "hstu_attn_fwd_rab",
    "hstu_attn_plan_bytes",
    "hstu_attn_plan",
    "hstu_attn_fwd_planned",
    "hstu_attn_fwd_noalloc",
    "hstu_attn_get_error",
    "hstu_attn_status_string",
    "hstu_attn_selfcheck_wait_timeout",
    "hstu_attn_gemm_bf16",
    "hstu_attn_bwd",
    "hstu_attn_bwd_workspace_limit",
    "hstu_attn_partition",
    "hstu_layer_workspace_bytes",
    "hstu_layer_fwd",
    "hstu_layers_fwd",
    "hstu_attn_selfcheck_fwd_timeout",
)


class HstuError(RuntimeError):
    """A libhstu_attn call returned a status other than HSTU_OK."""

    def __init__(self, status, where):
        self.status = int(status)
        super().__init__("%s: %s" % (where, STATUS.get(self.status, "status %d" % self.status)))


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Loads libhstu_attn.so once; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError("libhstu_attn.so is not built (run __graft_entry__.build() or "
                           "python -m hstu_pointwise_attention_jagged_b200.build)")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, i32, f32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float
    lib.hstu_attn_fwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, vp, vp]
    lib.hstu_attn_fwd_cached.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, f32,
                                         vp, vp]
    i64 = ctypes.c_int64
    lib.hstu_attn_fwd_rab.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, f32, f32,
                                      vp, vp]
    lib.hstu_attn_plan_bytes.argtypes = [i32, i32, i32]
    lib.hstu_attn_plan_bytes.restype = i64
    lib.hstu_attn_plan.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, vp, i64, vp]
    lib.hstu_attn_fwd_planned.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, vp, vp, vp]
    lib.hstu_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, f32, f32,
                                          vp, vp]
    lib.hstu_attn_fwd_noalloc.restype = ctypes.c_int
    lib.hstu_attn_get_error.argtypes = [vp]
    lib.hstu_attn_status_string.argtypes = [ctypes.c_int]
    lib.hstu_attn_selfcheck_wait_timeout.argtypes = [ctypes.c_uint64, vp]
    lib.hstu_attn_gemm_bf16.argtypes = [vp, vp, vp, i32, i32, i32, vp]
    lib.hstu_attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, vp, vp, vp, vp]
    lib.hstu_attn_bwd_workspace_limit.argtypes = [ctypes.c_uint64]
    lib.hstu_attn_bwd_workspace_limit.restype = ctypes.c_uint64
    lib.hstu_attn_partition.argtypes = [vp, vp, vp, i32, i32, vp]
    lib.hstu_attn_selfcheck_fwd_timeout.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, f32, f32, vp,
                                                    ctypes.c_uint64, vp]
    lib.hstu_layer_workspace_bytes.argtypes = [i32, i32, i32, i32]
    lib.hstu_layer_workspace_bytes.restype = i64
    lib.hstu_layer_fwd.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, f32, vp, vp, i64, vp, vp]
    lib.hstu_layers_fwd.argtypes = [i32, vp, ctypes.POINTER(vp), ctypes.POINTER(vp), vp, vp, i32, i32, i32, i32, i32,
                                    f32, f32, vp, i64, vp, vp]
    lib.hstu_attn_status_string.restype = ctypes.c_char_p
    for name in ("hstu_attn_fwd", "hstu_attn_fwd_cached", "hstu_attn_fwd_rab", "hstu_attn_plan", "hstu_attn_fwd_planned",
                 "hstu_attn_get_error", "hstu_attn_selfcheck_wait_timeout", "hstu_attn_gemm_bf16", "hstu_attn_bwd",
                 "hstu_attn_partition", "hstu_layer_fwd", "hstu_layers_fwd",
                 "hstu_attn_selfcheck_fwd_timeout"):
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def _stream_ptr(stream, device):
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _check_tokens(name, t, H=None, d=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != torch.bfloat16 or t.dim() != 3 or not t.is_contiguous():
        raise TypeError("%s must be a contiguous bf16 tensor [rows, H, d]" % name)
    if H is not None and (t.shape[1] != H or t.shape[2] != d):
        raise ValueError("%s has shape %s, expected [*, %d, %d]" % (name, tuple(t.shape), H, d))


def _check_index(name, t, n, device, optional=True):
    if t is None:
        if optional:
            return
        raise TypeError("%s is required" % name)
    if not isinstance(t, torch.Tensor) or t.device != device or t.dtype != torch.int32 or \
            t.dim() != 1 or not t.is_contiguous() or t.numel() != n:
        raise TypeError("%s must be a contiguous int32 tensor of %d elements on %s" % (name, n, device))


def _raise_if(status, where):
    if status != 0:
        raise HstuError(status, where)


def hstu_attn_fwd(q, k, v, seq_offsets, num_targets, alpha, N, max_seq_len, out=None, stream=None):
    """Full forward pass; returns ``out`` (bf16 [total, H, d]). See include/hstu_attn.h."""
    lib = load_library()
    _check_tokens("q", q)
    total, H, d = q.shape
    _check_tokens("k", k, H, d)
    _check_tokens("v", v, H, d)
    if k.shape[0] != total or v.shape[0] != total:
        raise ValueError("q, k and v must have the same number of rows")
    B = seq_offsets.numel() - 1
    _check_index("seq_offsets", seq_offsets, B + 1, q.device, optional=False)
    _check_index("num_targets", num_targets, B, q.device)
    if out is None:
        out = torch.empty_like(q)
    _check_tokens("out", out, H, d)
    with torch.cuda.device(q.device):
        st = lib.hstu_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), _ptr(num_targets), B, H, d,
                               total, int(max_seq_len), float(alpha), float(N), _ptr(out),
                               _stream_ptr(stream, q.device))
    _raise_if(st, "hstu_attn_fwd")
    return out


def hstu_attn_fwd_cached(q, k, v, seq_offsets, num_targets, cached_len, alpha, N, max_seq_len, out=None,
                         stream=None):
    """Streaming forward: new-token queries against cached prefix + new K/V; returns ``out``."""
    lib = load_library()
    _check_tokens("q", q)
    total_q, H, d = q.shape
    _check_tokens("k", k, H, d)
    _check_tokens("v", v, H, d)
    total_kv = k.shape[0]
    if v.shape[0] != total_kv:
        raise ValueError("k and v must have the same number of rows")
    B = seq_offsets.numel() - 1
    _check_index("seq_offsets", seq_offsets, B + 1, q.device, optional=False)
    _check_index("num_targets", num_targets, B, q.device)
    _check_index("cached_len", cached_len, B, q.device)
    if out is None:
        out = torch.empty_like(q)
    _check_tokens("out", out, H, d)
    with torch.cuda.device(q.device):
        st = lib.hstu_attn_fwd_cached(_ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), _ptr(num_targets),
                                      _ptr(cached_len), B, H, d, total_kv, total_q, int(max_seq_len),
                                      float(alpha), float(N), _ptr(out), _stream_ptr(stream, q.device))
    _raise_if(st, "hstu_attn_fwd_cached")
    return out


def hstu_attn_fwd_rab(q, k, v, seq_offsets, num_targets, rab, alpha, N, max_seq_len, cached_len=None, out=None,
                      stream=None):
    """Relative-attention-bias variant: each visible pair gets silu(alpha*s) + rab[h, min(i-j, R-1)].
    ``rab`` is a float32 [H, R] tensor on the same device; with ``cached_len`` the queries are the
    new tokens only, as in :func:`hstu_attn_fwd_cached`.  Returns ``out``."""
    lib = load_library()
    _check_tokens("q", q)
    total_q, H, d = q.shape
    _check_tokens("k", k, H, d)
    _check_tokens("v", v, H, d)
    total_kv = k.shape[0]
    if v.shape[0] != total_kv:
        raise ValueError("k and v must have the same number of rows")
    if rab.dtype != torch.float32 or rab.dim() != 2 or rab.shape[0] != H or not rab.is_contiguous() \
            or rab.device != q.device:
        raise TypeError("rab must be a contiguous float32 [H, R] tensor on %s" % q.device)
    B = seq_offsets.numel() - 1
    _check_index("seq_offsets", seq_offsets, B + 1, q.device, optional=False)
    _check_index("num_targets", num_targets, B, q.device)
    _check_index("cached_len", cached_len, B, q.device)
    if out is None:
        out = torch.empty_like(q)
    _check_tokens("out", out, H, d)
    with torch.cuda.device(q.device):
        st = lib.hstu_attn_fwd_rab(_ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), _ptr(num_targets),
                                   _ptr(cached_len), _ptr(rab), int(rab.shape[1]), B, H, d, total_kv, total_q,
                                   int(max_seq_len), float(alpha), float(N), _ptr(out),
                                   _stream_ptr(stream, q.device))
    _raise_if(st, "hstu_attn_fwd_rab")
    return out


def hstu_attn_plan_bytes(B, H, total_q):
    """Bytes of a plan buffer for these sizes (see include/hstu_attn.h for its layout)."""
    return int(load_library().hstu_attn_plan_bytes(int(B), int(H), int(total_q)))


def hstu_attn_plan(seq_offsets, num_targets, cached_len, H, total_kv, total_q, max_seq_len, plan=None,
                   stream=None):
    """Builds the work plan on the device; returns the plan (uint8 CUDA tensor)."""
    lib = load_library()
    B = seq_offsets.numel() - 1
    dev = seq_offsets.device
    _check_index("seq_offsets", seq_offsets, B + 1, dev, optional=False)
    _check_index("num_targets", num_targets, B, dev)
    _check_index("cached_len", cached_len, B, dev)
    nbytes = hstu_attn_plan_bytes(B, H, total_q)
    if plan is None:
        plan = torch.empty((max(nbytes, 16),), dtype=torch.uint8, device=dev)
    if plan.dtype != torch.uint8 or not plan.is_contiguous() or plan.device != dev:
        raise TypeError("plan must be a contiguous uint8 tensor on %s" % dev)
    with torch.cuda.device(dev):
        st = lib.hstu_attn_plan(_ptr(seq_offsets), _ptr(num_targets), _ptr(cached_len), B, int(H), int(total_kv),
                                int(total_q), int(max_seq_len), _ptr(plan), plan.numel(), _stream_ptr(stream, dev))
    _raise_if(st, "hstu_attn_plan")
    return plan


def hstu_attn_fwd_planned(q, k, v, seq_offsets, num_targets, cached_len, alpha, N, plan, out=None, stream=None):
    """Attention over a plan from hstu_attn_plan (same offsets); returns ``out``."""
    lib = load_library()
    _check_tokens("q", q)
    total_q, H, d = q.shape
    _check_tokens("k", k, H, d)
    _check_tokens("v", v, H, d)
    total_kv = k.shape[0]
    B = seq_offsets.numel() - 1
    _check_index("seq_offsets", seq_offsets, B + 1, q.device, optional=False)
    _check_index("num_targets", num_targets, B, q.device)
    _check_index("cached_len", cached_len, B, q.device)
    if out is None:
        out = torch.empty_like(q)
    _check_tokens("out", out, H, d)
    with torch.cuda.device(q.device):
        st = lib.hstu_attn_fwd_planned(_ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), _ptr(num_targets),
                                       _ptr(cached_len), B, H, d, total_kv, total_q, float(alpha), float(N),
                                       _ptr(plan), _ptr(out), _stream_ptr(stream, q.device))
    _raise_if(st, "hstu_attn_fwd_planned")
    return out


def hstu_attn_fwd_noalloc(q, k, v, seq_offsets, num_targets, cached_len, alpha, N, max_seq_len, out=None,
                          stream=None):
    """hstu_attn_fwd_cached whose plan lives in the library's fixed device array, for callers that
    must not allocate device memory during a call (see include/hstu_attn.h for the size limit and
    the rule that calls must not overlap on the GPU).  Pass cached_len=None for a full pass."""
    lib = load_library()
    _check_tokens("q", q)
    total_q, H, d = q.shape
    _check_tokens("k", k, H, d)
    _check_tokens("v", v, H, d)
    total_kv = k.shape[0]
    B = seq_offsets.numel() - 1
    _check_index("seq_offsets", seq_offsets, B + 1, q.device, optional=False)
    _check_index("num_targets", num_targets, B, q.device)
    _check_index("cached_len", cached_len, B, q.device)
    if out is None:
        out = torch.empty_like(q)
    _check_tokens("out", out, H, d)
    with torch.cuda.device(q.device):
        st = lib.hstu_attn_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), _ptr(num_targets),
                                       _ptr(cached_len), B, H, d, total_kv, total_q, int(max_seq_len),
                                       float(alpha), float(N), _ptr(out), _stream_ptr(stream, q.device))
    _raise_if(st, "hstu_attn_fwd_noalloc")
    return out


def plan_contents(plan, B):
    """Reads a plan's header, query-row starts and valid items back to the host (inspection)."""
    raw = plan.cpu().numpy().view("<i4")
    header = raw[:4].copy()
    qs_words = ((B * 4 + 15) // 16) * 4
    ps_words = (((B + 1) * 4 + 15) // 16) * 4
    q_start = raw[4:4 + B].copy()
    items = raw[4 + qs_words + ps_words:].reshape(-1, 4)[:int(header[1])].copy()
    return header, q_start, items


def hstu_attn_get_error(device=None, stream=None):
    """Synchronises the stream and returns (and clears) the device error status (0 = clean)."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        return int(lib.hstu_attn_get_error(_stream_ptr(stream, dev)))


def hstu_attn_status_string(status):
    return load_library().hstu_attn_status_string(int(status)).decode()


def hstu_attn_selfcheck_wait_timeout(limit_ns, device=None, stream=None):
    """Launches the failure-path self-check: a bounded wait that must time out after limit_ns."""
    lib = load_library()
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        _raise_if(lib.hstu_attn_selfcheck_wait_timeout(int(limit_ns), _stream_ptr(stream, dev)),
                  "hstu_attn_selfcheck_wait_timeout")


def hstu_attn_gemm_bf16(a, w, out=None, stream=None):
    """C = A · Wᵀ (bf16 [M, K] · bf16 [N, K]ᵀ -> bf16 [M, N]) on the tensor cores; returns ``out``."""
    lib = load_library()
    for name, t in (("a", a), ("w", w)):
        if t.dtype != torch.bfloat16 or t.dim() != 2 or not t.is_contiguous() or not t.is_cuda:
            raise TypeError("%s must be a contiguous bf16 CUDA matrix" % name)
    M, K = a.shape
    N = w.shape[0]
    if w.shape[1] != K or w.device != a.device:
        raise ValueError("w must be [N, K] on the same device as a")
    if out is None:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=a.device)
    if out.dtype != torch.bfloat16 or tuple(out.shape) != (M, N) or not out.is_contiguous():
        raise TypeError("out must be a contiguous bf16 [M, N] tensor")
    with torch.cuda.device(a.device):
        st = lib.hstu_attn_gemm_bf16(_ptr(a), _ptr(w), _ptr(out), M, N, K, _stream_ptr(stream, a.device))
    _raise_if(st, "hstu_attn_gemm_bf16")
    return out


def hstu_attn_bwd(q, k, v, dout, seq_offsets, num_targets, alpha, N, max_seq_len, dq=None, dk=None, dv=None,
                  stream=None):
    """Backward pass of hstu_attn_fwd; returns (dq, dk, dv), bf16 [total, H, d]. See include/hstu_attn.h."""
    lib = load_library()
    _check_tokens("q", q)
    total, H, d = q.shape
    for name, t in (("k", k), ("v", v), ("dout", dout)):
        _check_tokens(name, t, H, d)
        if t.shape[0] != total:
            raise ValueError("q, k, v and dout must have the same number of rows")
    B = seq_offsets.numel() - 1
    _check_index("seq_offsets", seq_offsets, B + 1, q.device, optional=False)
    _check_index("num_targets", num_targets, B, q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _check_tokens(name, t, H, d)
    with torch.cuda.device(q.device):
        st = lib.hstu_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(seq_offsets), _ptr(num_targets), B, H,
                               d, total, int(max_seq_len), float(alpha), float(N), _ptr(dq), _ptr(dk), _ptr(dv),
                               _stream_ptr(stream, q.device))
    _raise_if(st, "hstu_attn_bwd")
    return dq, dk, dv


def hstu_attn_bwd_workspace_limit(max_bytes):
    """Largest dS workspace (bytes) hstu_attn_bwd may take per call (0: recompute dS for dq); returns
    the previous limit. See include/hstu_attn.h."""
    return int(load_library().hstu_attn_bwd_workspace_limit(int(max_bytes)))


def hstu_attn_partition(seq_offsets, num_targets, cached_len, parts):
    """Contiguous user runs, one per GPU, minimising the largest visible-pair cost (host arrays in,
    numpy int32 [parts+1] out: GPU p takes users [out[p], out[p+1])). See include/hstu_attn.h."""
    import numpy as np
    lib = load_library()
    off = np.ascontiguousarray(seq_offsets, np.int32)
    B = len(off) - 1
    nt = None if num_targets is None else np.ascontiguousarray(num_targets, np.int32)
    cl = None if cached_len is None else np.ascontiguousarray(cached_len, np.int32)
    out = np.zeros(int(parts) + 1, np.int32)

    def p(a):
        return None if a is None else ctypes.c_void_p(a.ctypes.data)

    st = lib.hstu_attn_partition(p(off), p(nt), p(cl), B, int(parts), p(out))
    _raise_if(st, "hstu_attn_partition")
    return out


def shard_of(seq_offsets, user_start, part):
    """Rows and rebased offsets of one GPU's run of users: (first user, last user + 1, first token
    row, last token row + 1, seq_offsets of the run starting at 0)."""
    import numpy as np
    off = np.asarray(seq_offsets, np.int64)
    u0, u1 = int(user_start[part]), int(user_start[part + 1])
    r0, r1 = int(off[u0]), int(off[u1])
    return u0, u1, r0, r1, (off[u0:u1 + 1] - r0).astype(np.int32)


def hstu_layer_workspace_bytes(H, d, total, num_layers=1):
    return int(load_library().hstu_layer_workspace_bytes(int(H), int(d), int(total), int(num_layers)))


def _check_act(name, t, D):
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.bfloat16 or t.dim() != 2 or \
            t.shape[1] != D or not t.is_contiguous():
        raise TypeError("%s must be a contiguous bf16 CUDA tensor [rows, %d]" % (name, D))


def hstu_layer_fwd(x, w_uvqk, w_out, seq_offsets, num_targets, H, d, alpha, N, plan, workspace=None, y=None,
                   stream=None):
    """One HSTU layer (projection, attention, projection) over a plan from hstu_attn_plan; returns y
    (bf16 [total, H*d]). See include/hstu_attn.h."""
    lib = load_library()
    D = H * d
    _check_act("x", x, D)
    total = x.shape[0]
    _check_act("w_uvqk", w_uvqk, D)
    _check_act("w_out", w_out, 3 * D)
    if w_uvqk.shape[0] != 4 * D or w_out.shape[0] != D:
        raise ValueError("w_uvqk must be [4D, D] and w_out [D, 3D]")
    B = seq_offsets.numel() - 1
    _check_index("seq_offsets", seq_offsets, B + 1, x.device, optional=False)
    _check_index("num_targets", num_targets, B, x.device)
    nbytes = hstu_layer_workspace_bytes(H, d, total, 1)
    if workspace is None:
        workspace = torch.empty((nbytes,), dtype=torch.uint8, device=x.device)
    y = torch.empty_like(x) if y is None else y
    _check_act("y", y, D)
    with torch.cuda.device(x.device):
        st = lib.hstu_layer_fwd(_ptr(x), _ptr(w_uvqk), _ptr(w_out), _ptr(seq_offsets), _ptr(num_targets), B, H, d,
                                total, float(alpha), float(N), _ptr(plan), _ptr(workspace), workspace.numel(),
                                _ptr(y), _stream_ptr(stream, x.device))
    _raise_if(st, "hstu_layer_fwd")
    return y


def hstu_layers_fwd(x, w_uvqk_list, w_out_list, seq_offsets, num_targets, H, d, alpha, N, max_seq_len,
                    workspace=None, y=None, stream=None):
    """A stack of HSTU layers over one work plan; returns the last layer's output. See
    include/hstu_attn.h."""
    lib = load_library()
    D = H * d
    L = len(w_uvqk_list)
    if L < 1 or len(w_out_list) != L:
        raise ValueError("need one w_uvqk and one w_out per layer")
    _check_act("x", x, D)
    for w1, w2 in zip(w_uvqk_list, w_out_list):
        _check_act("w_uvqk", w1, D)
        _check_act("w_out", w2, 3 * D)
    total = x.shape[0]
    B = seq_offsets.numel() - 1
    _check_index("seq_offsets", seq_offsets, B + 1, x.device, optional=False)
    _check_index("num_targets", num_targets, B, x.device)
    nbytes = hstu_layer_workspace_bytes(H, d, total, L)
    if workspace is None:
        workspace = torch.empty((nbytes,), dtype=torch.uint8, device=x.device)
    y = torch.empty_like(x) if y is None else y
    _check_act("y", y, D)
    w1p = (ctypes.c_void_p * L)(*[w.data_ptr() for w in w_uvqk_list])
    w2p = (ctypes.c_void_p * L)(*[w.data_ptr() for w in w_out_list])
    with torch.cuda.device(x.device):
        st = lib.hstu_layers_fwd(L, _ptr(x), w1p, w2p, _ptr(seq_offsets), _ptr(num_targets), B, H, d, total,
                                 int(max_seq_len), float(alpha), float(N), _ptr(workspace), workspace.numel(), _ptr(y),
                                 _stream_ptr(stream, x.device))
    _raise_if(st, "hstu_layers_fwd")
    return y


def hstu_attn_selfcheck_fwd_timeout(q, k, v, seq_offsets, num_targets, alpha, N, max_seq_len, limit_ns, out=None,
                                    stream=None):
    """hstu_attn_fwd with every attention-kernel wait limited to limit_ns (test hook of the abort path)."""
    lib = load_library()
    _check_tokens("q", q)
    total, H, d = q.shape
    B = seq_offsets.numel() - 1
    out = torch.empty_like(q) if out is None else out
    with torch.cuda.device(q.device):
        st = lib.hstu_attn_selfcheck_fwd_timeout(_ptr(q), _ptr(k), _ptr(v), _ptr(seq_offsets), _ptr(num_targets), B,
                                                 H, d, total, int(max_seq_len), float(alpha), float(N), _ptr(out),
                                                 int(limit_ns), _stream_ptr(stream, q.device))
    _raise_if(st, "hstu_attn_selfcheck_fwd_timeout")
    return out
