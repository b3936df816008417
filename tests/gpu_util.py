"""Helpers shared by the GPU tests: moving workloads to the device, running the library through
its binding, and the tolerances the parity tests apply."""
import numpy as np
import torch

from hstu_pointwise_attention_jagged_b200 import binding, workloads

# Parity bar for bf16 inputs drawn N(0,1)/sqrt(d): relative L2 error over all compared outputs
# and the largest absolute error (the global bars), the same relative bar for every user on its
# own, and a ceiling on any single output row's relative L2 error, so that one wrong row cannot
# hide among thousands of correct ones.  A row of a correct result carries at most two bf16
# roundings (P and the output, 2^-9 each), so its relative error stays near 3e-3.
REL_L2 = 5e-3
MAX_ABS = 3e-2
ROW_REL_L2 = 2e-2

# (what, global rel_l2, max_abs, worst user and its rel_l2, worst row and its rel_l2) of every
# assert_parity call in this session; printed in the terminal summary.
PARITY_LOG = []


def dev_bf16(x):
    """float32 array of bf16-representable values -> bf16 CUDA tensor with exactly those values."""
    bits = workloads.bf16_bits(x)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


def dev_i32(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.int32)).cuda()


def to_f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def rel_l2(a, b):
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def assert_parity(got, ref, rel=REL_L2, max_abs=MAX_ABS, what="", users=None, row_rel=ROW_REL_L2):
    """got, ref: [rows, ...].  users: the user of each compared row (None: the rows form one user).
    Checks the global relative L2 and max-abs bars, the relative L2 of every user against the
    same bar, and every row's relative L2 against `row_rel`."""
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), "%s: non-finite output" % what
    r = rel_l2(got, ref)
    m = float(np.abs(got - ref).max()) if got.size else 0.0
    n = got.shape[0]
    err_rows = np.linalg.norm((got - ref).reshape(n, -1), axis=1)
    ref_rows = np.linalg.norm(ref.reshape(n, -1), axis=1)
    row_rel_l2 = err_rows / np.maximum(ref_rows, 1e-300)
    worst_row = int(np.argmax(row_rel_l2)) if n else -1
    users = np.zeros(n, np.int64) if users is None else np.asarray(users)
    worst_user, worst_user_rel = -1, 0.0
    for b in np.unique(users):
        sel = users == b
        den = float(np.linalg.norm(ref_rows[sel]))
        ur = float(np.linalg.norm(err_rows[sel])) / max(den, 1e-300)
        if den > 0 and ur >= worst_user_rel:
            worst_user, worst_user_rel = int(b), ur
    rec = {"what": what, "rel_l2": r, "max_abs": m, "worst_user": worst_user, "worst_user_rel_l2": worst_user_rel,
           "worst_row": worst_row, "worst_row_rel_l2": float(row_rel_l2[worst_row]) if n else 0.0, "rows": n}
    PARITY_LOG.append(rec)
    assert r <= rel and m <= max_abs, "%s: rel_l2=%.3e (bar %.1e) max_abs=%.3e (bar %.1e)" % (what, r, rel, m,
                                                                                             max_abs)
    assert worst_user_rel <= rel, "%s: user %d rel_l2=%.3e (bar %.1e)" % (what, worst_user, worst_user_rel, rel)
    assert rec["worst_row_rel_l2"] <= row_rel, "%s: row %d rel_l2=%.3e (bar %.1e)" % (
        what, worst_row, rec["worst_row_rel_l2"], row_rel)
    return r, m


def row_users(w, cached=False):
    """User of every query row of a workload (every token, or the new tokens with a cached prefix)."""
    nq = np.diff(w.seq_offsets) - (w.cached_len if cached else 0)
    return np.repeat(np.arange(w.B), np.maximum(nq, 0))


def run_fwd(w, q=None, k=None, v=None, out=None, num_targets="w"):
    q = dev_bf16(w.q) if q is None else q
    k = dev_bf16(w.k) if k is None else k
    v = dev_bf16(w.v) if v is None else v
    nt = dev_i32(w.num_targets) if isinstance(num_targets, str) else num_targets
    out = binding.hstu_attn_fwd(q, k, v, dev_i32(w.seq_offsets), nt, w.alpha, w.N, max(w.max_seq_len, 1), out=out)
    torch.cuda.synchronize()
    return out


def run_cached(w, q_new=None, k=None, v=None, out=None):
    sel = w.new_rows()
    q_new = dev_bf16(w.q[sel]) if q_new is None else q_new
    k = dev_bf16(w.k) if k is None else k
    v = dev_bf16(w.v) if v is None else v
    out = binding.hstu_attn_fwd_cached(q_new, k, v, dev_i32(w.seq_offsets), dev_i32(w.num_targets),
                                       dev_i32(w.cached_len), w.alpha, w.N, max(w.max_seq_len, 1), out=out)
    torch.cuda.synchronize()
    return out


def sample_rows(w, per_user_random=24, seed=0, cached=False):
    """(user, local query row) pairs: tile edges, the history/candidate boundary, both ends of each
    user, plus random rows."""
    rng = np.random.default_rng(seed)
    users, local = [], []
    for b in range(w.B):
        L = int(w.seq_offsets[b + 1] - w.seq_offsets[b])
        c = int(w.cached_len[b]) if cached else 0
        U = L - int(w.num_targets[b])
        nq = L - c
        if nq <= 0:
            continue
        pos = {0, 1, 126, 127, 128, 129, 255, 256, 257, U - 1, U, U + 1, L - 2, L - 1}
        cand = sorted(p - c for p in pos if c <= p < L)
        cand += list(rng.integers(0, nq, size=min(per_user_random, nq)))
        for r in sorted(set(int(x) for x in cand)):
            users.append(b)
            local.append(r)
    return np.array(users, np.int32), np.array(local, np.int32)


def query_row_index(w, users, local, cached=False):
    """Row of the query/output tensor holding (user, local row)."""
    if cached:
        qstart = np.concatenate([[0], np.cumsum(np.diff(w.seq_offsets) - w.cached_len)])
        return qstart[users] + local
    return w.seq_offsets[users] + local
