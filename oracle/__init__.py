"""fp64 CPU oracle for jagged target-aware HSTU pointwise (SiLU) attention.

TEST INFRASTRUCTURE ONLY.  The oracle is a plain, slow, obviously-correct restatement of what
the CUDA library computes; it exists to check that library and shares no code with it.  Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference leg may
import it.  The library never falls back to it.

Computation (pages: the DLRMv3 MLPerf review, section "model selection" — attention is
Mask(SiLU(Q K^T)) V without relative bias, the history encoding is shared by all candidates
and its K/V reused across timestamps; the infolabhq.com multi-stage page — the user side never
depends on a candidate, and target-aware attention weighs history against each candidate):

    out[i,h,:] = (1/N) * sum_{j in A(i)} silu(alpha * q[i,h,:].k[j,h,:]) * v[j,h,:]
    A(i) = {j <= i} for a history token (i < U); {j < U} + {i} for a candidate (i >= U)

The backward pass (``bwd``, ``bwd_rows``) is derived from that definition by the chain rule; the
pages print none.  The C source (``hstu_oracle.c``) holds the arithmetic; this module only marshals
numpy arrays.
"""
import ctypes
import os

import numpy as np

from . import build as _build

class Oracle:
    """ctypes view of one build of the C oracle (the default build, or a test's mutant build)."""

    def __init__(self, path):
        lib = ctypes.CDLL(path)
        f32p = ctypes.POINTER(ctypes.c_float)
        i32p = ctypes.POINTER(ctypes.c_int32)
        f64p = ctypes.POINTER(ctypes.c_double)
        i64p = ctypes.POINTER(ctypes.c_int64)
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.hstu_oracle_fwd.argtypes = [f32p, f32p, f32p, i32p, i32p, i32, i32, i32, i64, f64,
                                        f64, f64p, i64p]
        lib.hstu_oracle_fwd_cached.argtypes = [f32p, f32p, f32p, i32p, i32p, i32p, i32, i32, i32,
                                               i64, i64, f64, f64, f64p, i64p]
        lib.hstu_oracle_rows.argtypes = [f32p, f32p, f32p, i32p, i32p, i32p, i32, i32, i32, i64,
                                         i64, f64, f64, i32p, i32p, i64, f64p, i64p]
        lib.hstu_oracle_rows_rab.argtypes = [f32p, f32p, f32p, i32p, i32p, i32p, f32p, i32, i32, i32,
                                             i32, i64, i64, f64, f64, i32p, i32p, i64, f64p]
        lib.hstu_oracle_bwd.argtypes = [f32p, f32p, f32p, f32p, i32p, i32p, i32, i32, i32, i64, f64, f64,
                                        f64p, f64p, f64p]
        lib.hstu_oracle_bwd_rows.argtypes = [f32p, f32p, f32p, f32p, i32p, i32p, i32, i32, i32, i64, f64, f64,
                                             i32p, i32p, i64, f64p, f64p, f64p]
        for fn in (lib.hstu_oracle_fwd, lib.hstu_oracle_fwd_cached, lib.hstu_oracle_rows,
                   lib.hstu_oracle_rows_rab, lib.hstu_oracle_num_threads, lib.hstu_oracle_bwd,
                   lib.hstu_oracle_bwd_rows):
            fn.restype = ctypes.c_int
        self.lib = lib

    def num_threads(self) -> int:
        """Threads the oracle's OpenMP loops use (OMP_NUM_THREADS or all cores)."""
        return int(self.lib.hstu_oracle_num_threads())

    def fwd(self, q, k, v, seq_offsets, num_targets, alpha, N, return_macs=False):
        """Full forward: q, k, v [total, H, d]; returns float64 [total, H, d]."""
        q, k, v = _f32(q), _f32(k), _f32(v)
        off = _i32(seq_offsets)
        nt = None if num_targets is None else _i32(num_targets)
        total, H, d = q.shape
        out = np.zeros((total, H, d), dtype=np.float64)
        macs = ctypes.c_int64(0)
        rc = self.lib.hstu_oracle_fwd(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                      _ptr(v, ctypes.c_float), _ptr(off, ctypes.c_int32),
                                      _ptr(nt, ctypes.c_int32), len(off) - 1, H, d, total,
                                      float(alpha), float(N), _ptr(out, ctypes.c_double),
                                      ctypes.byref(macs))
        if rc != 0:
            raise ValueError("oracle: inconsistent seq_offsets / num_targets")
        return (out, macs.value) if return_macs else out

    def fwd_cached(self, q_new, k, v, seq_offsets, num_targets, cached_len, alpha, N,
                   return_macs=False):
        """Streaming forward: q_new [total_q, H, d] new rows; k, v [total_kv, H, d] full segments."""
        q_new, k, v = _f32(q_new), _f32(k), _f32(v)
        off = _i32(seq_offsets)
        nt = None if num_targets is None else _i32(num_targets)
        cl = None if cached_len is None else _i32(cached_len)
        total_q, H, d = q_new.shape
        out = np.zeros((total_q, H, d), dtype=np.float64)
        macs = ctypes.c_int64(0)
        rc = self.lib.hstu_oracle_fwd_cached(_ptr(q_new, ctypes.c_float), _ptr(k, ctypes.c_float),
                                             _ptr(v, ctypes.c_float), _ptr(off, ctypes.c_int32),
                                             _ptr(nt, ctypes.c_int32), _ptr(cl, ctypes.c_int32),
                                             len(off) - 1, H, d, k.shape[0], total_q, float(alpha),
                                             float(N), _ptr(out, ctypes.c_double), ctypes.byref(macs))
        if rc != 0:
            raise ValueError("oracle: inconsistent seq_offsets / num_targets / cached_len")
        return (out, macs.value) if return_macs else out

    def rows(self, q, k, v, seq_offsets, num_targets, cached_len, alpha, N, row_user, row_local,
             return_macs=False):
        """Selected output rows [n, H, d] for (user, local query row) pairs; cached_len may be None."""
        q, k, v = _f32(q), _f32(k), _f32(v)
        off = _i32(seq_offsets)
        nt = None if num_targets is None else _i32(num_targets)
        cl = None if cached_len is None else _i32(cached_len)
        ru, rl = _i32(row_user), _i32(row_local)
        total_q, H, d = q.shape
        out = np.zeros((len(ru), H, d), dtype=np.float64)
        macs = ctypes.c_int64(0)
        rc = self.lib.hstu_oracle_rows(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                       _ptr(v, ctypes.c_float), _ptr(off, ctypes.c_int32),
                                       _ptr(nt, ctypes.c_int32), _ptr(cl, ctypes.c_int32),
                                       len(off) - 1, H, d, k.shape[0], total_q, float(alpha),
                                       float(N), _ptr(ru, ctypes.c_int32), _ptr(rl, ctypes.c_int32),
                                       len(ru), _ptr(out, ctypes.c_double), ctypes.byref(macs))
        if rc != 0:
            raise ValueError("oracle: inconsistent offsets or row selection")
        return (out, macs.value) if return_macs else out


    def rows_rab(self, q, k, v, seq_offsets, num_targets, cached_len, rab, alpha, N, row_user, row_local):
        """Selected rows of the relative-attention-bias variant; rab is the [H, R] bias table."""
        q, k, v, rab = _f32(q), _f32(k), _f32(v), _f32(rab)
        off = _i32(seq_offsets)
        nt = None if num_targets is None else _i32(num_targets)
        cl = None if cached_len is None else _i32(cached_len)
        ru, rl = _i32(row_user), _i32(row_local)
        total_q, H, d = q.shape
        if rab.ndim != 2 or rab.shape[0] != H or rab.shape[1] < 1:
            raise ValueError("oracle: rab must be [H, R] with R >= 1")
        out = np.zeros((len(ru), H, d), dtype=np.float64)
        rc = self.lib.hstu_oracle_rows_rab(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                           _ptr(v, ctypes.c_float), _ptr(off, ctypes.c_int32),
                                           _ptr(nt, ctypes.c_int32), _ptr(cl, ctypes.c_int32),
                                           _ptr(rab, ctypes.c_float), rab.shape[1], len(off) - 1, H, d,
                                           k.shape[0], total_q, float(alpha), float(N),
                                           _ptr(ru, ctypes.c_int32), _ptr(rl, ctypes.c_int32), len(ru),
                                           _ptr(out, ctypes.c_double))
        if rc != 0:
            raise ValueError("oracle: inconsistent offsets, row selection or bias table")
        return out

    def fwd_rab(self, q, k, v, seq_offsets, num_targets, rab, alpha, N, cached_len=None):
        """Every query row of the relative-attention-bias variant ([total_q, H, d]; with cached_len
        the query rows are the new tokens, packed per user as in the library)."""
        off = np.asarray(seq_offsets, np.int64)
        L = np.diff(off)
        c = np.zeros_like(L) if cached_len is None else np.asarray(cached_len, np.int64)
        users = np.concatenate([np.full(max(int(L[b] - c[b]), 0), b) for b in range(len(L))] + [np.zeros(0)])
        local = np.concatenate([np.arange(max(int(L[b] - c[b]), 0)) for b in range(len(L))] + [np.zeros(0)])
        return self.rows_rab(q, k, v, seq_offsets, num_targets, cached_len, rab, alpha, N, users, local)


    def bwd(self, q, k, v, dout, seq_offsets, num_targets, alpha, N):
        """Backward pass of the full forward: returns (dq, dk, dv), float64 [total, H, d] each, for
        the loss gradient dout [total, H, d] with respect to out."""
        q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
        off = _i32(seq_offsets)
        nt = None if num_targets is None else _i32(num_targets)
        total, H, d = q.shape
        dq, dk, dv = (np.zeros((total, H, d), dtype=np.float64) for _ in range(3))
        rc = self.lib.hstu_oracle_bwd(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float), _ptr(v, ctypes.c_float),
                                      _ptr(dout, ctypes.c_float), _ptr(off, ctypes.c_int32),
                                      _ptr(nt, ctypes.c_int32), len(off) - 1, H, d, total, float(alpha),
                                      float(N), _ptr(dq, ctypes.c_double), _ptr(dk, ctypes.c_double),
                                      _ptr(dv, ctypes.c_double))
        if rc != 0:
            raise ValueError("oracle: inconsistent seq_offsets / num_targets")
        return dq, dk, dv

    def bwd_rows(self, q, k, v, dout, seq_offsets, num_targets, alpha, N, row_user, row_local):
        """Selected rows of the backward pass: for each (user, position) pair, dq of that query row
        and dk, dv of that key row ([n, H, d] float64 each), equal to the full pass's rows."""
        q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
        off = _i32(seq_offsets)
        nt = None if num_targets is None else _i32(num_targets)
        ru, rl = _i32(row_user), _i32(row_local)
        total, H, d = q.shape
        dq, dk, dv = (np.zeros((len(ru), H, d), dtype=np.float64) for _ in range(3))
        rc = self.lib.hstu_oracle_bwd_rows(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float),
                                           _ptr(v, ctypes.c_float), _ptr(dout, ctypes.c_float),
                                           _ptr(off, ctypes.c_int32), _ptr(nt, ctypes.c_int32), len(off) - 1, H, d,
                                           total, float(alpha), float(N), _ptr(ru, ctypes.c_int32),
                                           _ptr(rl, ctypes.c_int32), len(ru), _ptr(dq, ctypes.c_double),
                                           _ptr(dk, ctypes.c_double), _ptr(dv, ctypes.c_double))
        if rc != 0:
            raise ValueError("oracle: inconsistent offsets or row selection")
        return dq, dk, dv


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _ptr(a, ctype):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctype))


_default = None


def default() -> Oracle:
    """The oracle built from oracle/hstu_oracle.c (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def num_threads() -> int:
    return default().num_threads()


def fwd(*args, **kwargs):
    return default().fwd(*args, **kwargs)


def fwd_cached(*args, **kwargs):
    return default().fwd_cached(*args, **kwargs)


def rows(*args, **kwargs):
    return default().rows(*args, **kwargs)


def rows_rab(*args, **kwargs):
    return default().rows_rab(*args, **kwargs)


def fwd_rab(*args, **kwargs):
    return default().fwd_rab(*args, **kwargs)


def bwd(*args, **kwargs):
    return default().bwd(*args, **kwargs)


def bwd_rows(*args, **kwargs):
    return default().bwd_rows(*args, **kwargs)


def linear(a, w):
    """C = A · Wᵀ in fp64 (A [M, K], W [N, K]): the dense projections of the HSTU layer whose flops
    the DLRMv3 review counts as 4·L·D² and 3·L·D² per layer.  A matrix product is the definition."""
    return np.asarray(a, np.float64) @ np.asarray(w, np.float64).T


def round_bf16(a):
    """Rounds to the nearest bf16 value, ties to even (the storage format of every tensor the library
    passes between steps), returned as float64.  Written from the format: keep the top 16 bits of the
    float32 pattern, rounding the dropped 16 bits to nearest with ties to the even kept pattern."""
    f = np.ascontiguousarray(np.asarray(a, np.float64).astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    keep = u >> np.uint64(16)
    rest = u & np.uint64(0xFFFF)
    up = (rest > 0x8000) | ((rest == 0x8000) & ((keep & np.uint64(1)) == 1))
    keep = keep + up.astype(np.uint64)
    return (keep << np.uint64(16)).astype(np.uint32).view(np.float32).astype(np.float64)


def layer(x, w_uvqk, w_out, seq_offsets, num_targets, H, d, alpha, N):
    """One HSTU layer as the library composes it, from oracle.linear and oracle.fwd only (fp64, with
    every tensor the library stores between its steps rounded to bf16):

        UVQK = X W_uvqk^T   -> blocks U, V, Q, K of D = H d columns
        A    = attention(Q, K, V)
        Y    = [U | A | U*A] W_out^T

    The DLRMv3 review (section "model selection", FLOP-formula paragraph) gives the layer's flops as
    4 L D^2 + L^2 D / 2 + 3 L D^2; the blocks above are the plainest reading with those terms.
    Returns Y [total, D] in fp64 (not rounded)."""
    x = np.asarray(x, np.float64)
    total, D = x.shape
    uvqk = round_bf16(linear(x, w_uvqk))
    u, v, q, k = (uvqk[:, i * D:(i + 1) * D] for i in range(4))
    a = fwd(q.reshape(total, H, d), k.reshape(total, H, d), v.reshape(total, H, d), seq_offsets, num_targets,
            alpha, N).reshape(total, D)
    a = round_bf16(a)
    cat = np.concatenate([u, a, round_bf16(u * a)], axis=1)
    return linear(cat, w_out)


def layers(x, w_uvqk_list, w_out_list, seq_offsets, num_targets, H, d, alpha, N):
    """A stack of layers; the hidden activations between layers are stored as bf16."""
    y = np.asarray(x, np.float64)
    for i, (w1, w2) in enumerate(zip(w_uvqk_list, w_out_list)):
        if i > 0:
            y = round_bf16(y)
        y = layer(y, w1, w2, seq_offsets, num_targets, H, d, alpha, N)
    return y
