"""Dense brute-force restatement used to pin the oracle on tiny inputs (numpy/scipy, fp64).

It builds each user's L x L visibility matrix as a block matrix from the wording of the method
(history block causal, candidates see the whole history block, candidates see only themselves
among candidates, history never sees candidates) and evaluates
``(M * silu(alpha * Q K^T)) V / N`` with dense matrix products and scipy's logistic function.
It shares nothing with oracle/hstu_oracle.c.
"""
import numpy as np
from scipy.special import expit


def visibility(L, U):
    T = L - U
    hist_hist = np.tril(np.ones((U, U), dtype=bool))     # history -> earlier history and itself
    hist_cand = np.zeros((U, T), dtype=bool)             # history never sees candidates
    cand_hist = np.ones((T, U), dtype=bool)              # every candidate sees all history
    cand_cand = np.eye(T, dtype=bool)                    # ... and only itself among candidates
    return np.block([[hist_hist, hist_cand], [cand_hist, cand_cand]])


def attention(q, k, v, seq_offsets, num_targets, alpha, N):
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    out = np.zeros_like(q)
    H = q.shape[1]
    for b in range(len(seq_offsets) - 1):
        s0, s1 = int(seq_offsets[b]), int(seq_offsets[b + 1])
        L = s1 - s0
        if L == 0:
            continue
        T = 0 if num_targets is None else int(num_targets[b])
        M = visibility(L, L - T)
        for h in range(H):
            S = alpha * (q[s0:s1, h, :] @ k[s0:s1, h, :].T)
            P = np.where(M, S * expit(S), 0.0)
            out[s0:s1, h, :] = (P @ v[s0:s1, h, :]) / N
    return out


def attention_rab(q, k, v, seq_offsets, num_targets, rab, alpha, N):
    """The relative-attention-bias variant, densely: each visible pair gets
    silu(alpha * s) + rab[h, min(i - j, R - 1)], masked pairs nothing."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    rab = np.asarray(rab, np.float64)
    R = rab.shape[1]
    out = np.zeros_like(q)
    H = q.shape[1]
    for b in range(len(seq_offsets) - 1):
        s0, s1 = int(seq_offsets[b]), int(seq_offsets[b + 1])
        L = s1 - s0
        if L == 0:
            continue
        T = 0 if num_targets is None else int(num_targets[b])
        M = visibility(L, L - T)
        rel = np.arange(L)[:, None] - np.arange(L)[None, :]
        idx = np.clip(rel, 0, R - 1)
        for h in range(H):
            S = alpha * (q[s0:s1, h, :] @ k[s0:s1, h, :].T)
            P = np.where(M, S * expit(S) + rab[h][idx], 0.0)
            out[s0:s1, h, :] = (P @ v[s0:s1, h, :]) / N
    return out
