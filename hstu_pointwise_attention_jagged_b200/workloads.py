"""Seeded synthetic inputs for jagged target-aware HSTU attention.

Input generation only: lengths, offsets and random Q/K/V.  This module holds none of the
attention arithmetic, so both the CUDA path and the fp64 oracle can consume its output.

The DLRMv3 dataset the review describes (its section "dataset selection": thousands of history
events per request, a ~1B-item vocabulary, a streaming time order) is not available here; these
synthetic batches stand in for it with the shapes of the five named workloads below.

Recipe: ``numpy.random.default_rng(seed)`` draws, in this order, the per-user history lengths
(where random), then Q, K and V as float32 ``standard_normal * scale`` over the whole jagged
[total, H, d] tensor (scale = 1/sqrt(d) unless stated).  bf16 workloads are rounded to bf16
(round to nearest even) and kept as float32 arrays holding exactly those bf16 values.
"""
import math
from dataclasses import dataclass, field

import numpy as np


@dataclass
class Workload:
    name: str
    B: int
    H: int
    d: int
    alpha: float
    N: float
    uih_len: np.ndarray        # [B] history tokens per user (cached prefix included)
    num_targets: np.ndarray    # [B] candidates per user (last T_b rows of each segment)
    cached_len: np.ndarray     # [B] cached history prefix (0 unless streaming)
    seq_offsets: np.ndarray    # [B+1] int32, exclusive prefix sum of segment lengths
    q: np.ndarray              # [total, H, d] float32 (queries for every position)
    k: np.ndarray
    v: np.ndarray
    bf16: bool = True
    meta: dict = field(default_factory=dict)

    @property
    def total(self) -> int:
        return int(self.seq_offsets[-1])

    @property
    def seq_len(self) -> np.ndarray:
        return np.diff(self.seq_offsets).astype(np.int64)

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_len.max()) if self.B else 0

    def new_rows(self) -> np.ndarray:
        """Indices of the rows at positions >= cached_len[b] (the streaming call's query rows)."""
        idx = [np.arange(self.seq_offsets[b] + self.cached_len[b], self.seq_offsets[b + 1]) for b in range(self.B)]
        return np.concatenate(idx).astype(np.int64) if idx else np.zeros(0, np.int64)

    @property
    def total_q(self) -> int:
        return int(self.total - self.cached_len.sum())


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Rounds float32 values to the nearest bf16 (ties to even); returns float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + r) & np.uint32(0xFFFF0000)).view(np.float32)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """The bf16 bit patterns (uint16) of float32 values that are already bf16-representable."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def offsets_from_lengths(lengths) -> np.ndarray:
    """Exclusive prefix sum: the row where each jagged segment starts, plus the total."""
    lengths = np.asarray(lengths, dtype=np.int64)
    off = np.zeros(len(lengths) + 1, dtype=np.int64)
    np.cumsum(lengths, out=off[1:])
    return off.astype(np.int32)


def _draw(rng, total, H, d, scale, bf16):
    out = []
    for _ in range(3):
        x = rng.standard_normal((total, H, d), dtype=np.float32)
        x *= np.float32(scale)
        out.append(round_bf16(x) if bf16 else x)
    return out


def make_custom(name, uih_len, num_targets, H, d, alpha, N, seed, cached_len=None, scale=None, bf16=True):
    """A workload from explicit per-user lengths; Q/K/V drawn after any length draws."""
    rng = np.random.default_rng(seed)
    return _finish(rng, name, np.asarray(uih_len, np.int64), np.asarray(num_targets, np.int64), H, d, alpha, N,
                   cached_len, scale, bf16)


def _finish(rng, name, uih, nt, H, d, alpha, N, cached_len, scale, bf16, meta=None, values=True):
    B = len(uih)
    cl = np.zeros(B, np.int64) if cached_len is None else np.asarray(cached_len, np.int64)
    off = offsets_from_lengths(uih + nt)
    total = int(off[-1])
    if values:
        q, k, v = _draw(rng, total, H, d, (1.0 / math.sqrt(d)) if scale is None else scale, bf16)
    else:
        q = k = v = np.zeros((0, H, d), np.float32)
    return Workload(name=name, B=B, H=H, d=d, alpha=float(alpha), N=float(N), uih_len=uih.astype(np.int32),
                    num_targets=nt.astype(np.int32), cached_len=cl.astype(np.int32), seq_offsets=off,
                    q=q, k=k, v=v, bf16=bf16, meta=meta or {})


# The five named workloads: (description, builder).
def _tiny(seed=0, values=True):
    rng = np.random.default_rng(seed)
    uih = rng.integers(16, 64, size=4, endpoint=True).astype(np.int64)
    return _finish(rng, "tiny", uih, np.full(4, 4, np.int64), 2, 32, 1 / math.sqrt(32), 68, None, None, False,
                   values=values)


def _dlrmv3(seed=1, values=True):
    rng = np.random.default_rng(seed)
    return _finish(rng, "dlrmv3", np.full(8, 2048, np.int64), np.full(8, 2048, np.int64), 4, 128,
                   1 / math.sqrt(128), 4096, None, None, True, values=values)


def _jagged(seed=2, values=True):
    rng = np.random.default_rng(seed)
    u = rng.lognormal(mean=math.log(1024.0), sigma=1.0, size=64)
    uih = np.clip(np.rint(u), 32, 4096).astype(np.int64)
    return _finish(rng, "jagged", uih, np.full(64, 16, np.int64), 4, 128, 1 / math.sqrt(128), 4112, None, None,
                   True, values=values)


def _long(seed=3, values=True):
    rng = np.random.default_rng(seed)
    return _finish(rng, "long_history", np.full(4, 8192, np.int64), np.full(4, 512, np.int64), 8, 64,
                   1 / 8.0, 8704, None, None, True, values=values)


def _streaming(seed=4, values=True):
    rng = np.random.default_rng(seed)
    return _finish(rng, "streaming", np.full(16, 3300, np.int64), np.full(16, 2048, np.int64), 4, 128,
                   1 / math.sqrt(128), 5348, np.full(16, 3000, np.int64), None, True, values=values)


CONFIGS = {
    "tiny": ("4 users, history ~ U{16..64}, 4 candidates each, H=2, d=32, fp32 N(0,1)/sqrt(32), "
             "alpha=1/sqrt(32), N=68, seed 0", _tiny),
    "dlrmv3": ("8 users x (2048 history + 2048 candidates), H=4, d=128, bf16 N(0,1)/sqrt(128), "
               "alpha=1/sqrt(128), N=4096, seed 1", _dlrmv3),
    "jagged": ("64 users, history = clip(rint(lognormal(ln 1024, 1.0)), 32, 4096), 16 candidates each, H=4, "
               "d=128, bf16, N=4112, seed 2", _jagged),
    "long_history": ("4 users x (8192 history + 512 candidates), H=8, d=64, bf16, alpha=1/8, N=8704, seed 3",
                     _long),
    "streaming": ("16 users x (3000 cached + 300 new history + 2048 candidates), H=4, d=128, bf16, N=5348, "
                  "seed 4", _streaming),
}


def make(name: str, seed=None) -> Workload:
    desc, fn = CONFIGS[name]
    w = fn() if seed is None else fn(seed)
    w.meta["description"] = desc
    return w


def structure(name: str, seed=None):
    """The per-user lengths of a named workload without drawing its Q/K/V: (uih_len, num_targets,
    cached_len, H, d, alpha, N), the same lengths that ``make(name, seed)`` draws."""
    _, fn = CONFIGS[name]
    w = fn(values=False) if seed is None else fn(seed, values=False)
    return w.uih_len, w.num_targets, w.cached_len, w.H, w.d, w.alpha, w.N
