"""Work counts of jagged target-aware HSTU attention, for throughput reporting.

Algorithmic FLOPs count only visible (query, key) pairs — the mask-exact work of both matmuls
(scores Q K^T and the weighted sum P V), 2 FLOPs per multiply-add:

    flops = 4 * d * H * sum_b sum_{i queried} |A(i)|,
    |A(i)| = i + 1 for a history token (i < U_b), U_b + 1 for a candidate.

The DLRMv3 review (section "model selection", FLOP-formula paragraph) counts a layer as
2 * layers * (L*L*D/2 + 4*L*D^2 + 3*L*D^2) with L the history length and D the embedding
width; ``page_attention_flops`` returns its attention term 2 * (L*L*D/2) for one layer.
"""
import numpy as np


def visible_pairs(L, U, c=0):
    """Sum over queried positions i in [c, L) of |A(i)| for one user (history U, cached prefix c)."""
    L, U, c = int(L), int(U), int(c)
    hist = (U * (U + 1) - c * (c + 1)) // 2 if c < U else 0
    return hist + (L - max(U, c)) * (U + 1)


def algorithmic_flops(seq_offsets, num_targets, H, d, cached_len=None):
    seq_offsets = np.asarray(seq_offsets, np.int64)
    L = np.diff(seq_offsets)
    T = np.zeros_like(L) if num_targets is None else np.asarray(num_targets, np.int64)
    c = np.zeros_like(L) if cached_len is None else np.asarray(cached_len, np.int64)
    pairs = sum(visible_pairs(L[b], L[b] - T[b], c[b]) for b in range(len(L)))
    return 4 * int(d) * int(H) * int(pairs)


def page_attention_flops(uih_len, emb_dim, layers=1):
    """Attention term of the review's per-layer FLOP formula: 2 * layers * (L * L * D / 2)."""
    return 2 * int(layers) * (int(uih_len) * int(uih_len) * int(emb_dim) // 2)


def tile_flops(seq_offsets, num_targets, H, d, cached_len=None):
    """FLOPs of the 128x128 score tiles the kernel computes (masked tiles skipped), for context."""
    seq_offsets = np.asarray(seq_offsets, np.int64)
    L = np.diff(seq_offsets)
    T = np.zeros_like(L) if num_targets is None else np.asarray(num_targets, np.int64)
    c = np.zeros_like(L) if cached_len is None else np.asarray(cached_len, np.int64)
    tiles = 0
    for b in range(len(L)):
        U = int(L[b] - T[b])
        nq = int(L[b] - c[b])
        for r0 in range(0, nq, 128):
            p0, p1 = int(c[b]) + r0, int(c[b]) + min(r0 + 128, nq)
            keys = set(range(0, p1)) if p1 <= U else set(range(0, U)) | set(range(max(p0, U), p1))
            tiles += len({j // 128 for j in keys})
    return tiles * 2 * 2 * 128 * 128 * int(d) * int(H)
