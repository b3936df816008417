"""CPU: the multi-process plumbing of bench.py with two gloo ranks — the max/sum over ranks that
the timing uses, the per-rank batch seeds (each GPU gets its own batch of the same shape, no
data exchange), and the reference arm running on rank 0 only."""
import io
import json
import multiprocessing as mp
import os
import socket
import sys
from contextlib import redirect_stdout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    r = bench.Ranks(backend="gloo")
    m = r.max(float(rank + 1))
    s = r.sum(10.0 * (rank + 1))
    r.barrier()
    q.put((rank, m, s, bench.rank_seed(1, rank)))
    r.close()


def test_two_gloo_ranks_reduce_and_seed():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == [2.0, 2.0]        # max over ranks
    assert [r[2] for r in res] == [30.0, 30.0]      # sum over ranks
    assert res[0][3] != res[1][3]                   # distinct batches per rank


def test_rank_batches_same_shape_different_values():
    sys.path.insert(0, ROOT)
    import bench
    from hstu_pointwise_attention_jagged_b200 import workloads
    a = workloads.make("tiny", seed=bench.rank_seed(0, 0))
    b = workloads.make("tiny", seed=bench.rank_seed(0, 1))
    assert a.H == b.H and a.d == b.d and a.B == b.B
    assert not (a.q.shape == b.q.shape and (a.q == b.q).all())


def test_reference_arm_rank0_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3"]) == 0
    assert buf.getvalue() == ""
    monkeypatch.setenv("RANK", "0")
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.main(["--impl", "reference", "--gpus", "2", "--steps", "3", "--warmup", "3",
                           "--ref-rows", "64"]) == 0
    line = json.loads(buf.getvalue())
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["unit"] == "TFLOP/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_rank_workload_splits_one_batch():
    """With two ranks the bench splits one batch of two replicas of the jagged workload into two
    contiguous runs of users whose visible-pair costs differ by less than one user's cost."""
    sys.path.insert(0, ROOT)
    import bench
    from hstu_pointwise_attention_jagged_b200 import metrics
    w0, n0 = bench.rank_workload("jagged", 2, 0)
    w1, n1 = bench.rank_workload("jagged", 2, 1)
    assert n0 == n1 == 128
    assert w0.meta["users"][0] == 0 and w0.meta["users"][1] == w1.meta["users"][0] and w1.meta["users"][1] == 128
    assert w0.B + w1.B == 128
    c = [metrics.algorithmic_flops(w.seq_offsets, w.num_targets, w.H, w.d) for w in (w0, w1)]
    largest = max(metrics.algorithmic_flops(w.seq_offsets[b:b + 2] - w.seq_offsets[b], w.num_targets[b:b + 1], w.H,
                                            w.d) for w in (w0, w1) for b in range(w.B))
    assert abs(c[0] - c[1]) <= largest
    one, n = bench.rank_workload("dlrmv3", 1, 0)
    assert n == 8 and one.B == 8
