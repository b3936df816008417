"""Benchmark of jagged target-aware HSTU pointwise (SiLU) attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one forward pass of the attention (work plan + attention kernel) over one batch of
the DLRMv3-shaped workload: 8 users x (2048 history + 2048 candidate tokens), H=4 heads of
d=128, bf16 N(0,1)/sqrt(d) inputs, alpha=1/sqrt(128), N=4096 (synthetic: the DLRMv3 dataset is
not available).  Inputs are resident in HBM; L2 is flushed (256 MiB write) before every timed
step.  Multi-GPU: one process per GPU; the global batch is N replicas of the workload's users,
split by hstu_attn_partition into contiguous runs of equal visible-pair cost, one per GPU (users
are independent, so there is no collective on the data path; per-GPU work is fixed: weak
scaling); the only collectives are the barrier and the max/sum over ranks of the timings.

Prints one JSON line on rank 0.  `value` is whole-job algorithmic TFLOP/s (visible query/key
pairs only, both matmuls); `e2e` is the same metric through the one-shot public entry point
with host buffers and the host<->device copies inside the timed region; `roofline` reports the
attention kernel against the measured dense-bf16 tensor peak; `cpu_baseline` times the fp64
oracle on the host cores on a bounded sample of the same workload.

`--impl reference`: this method has no published implementation; the reference arm is the fp64
oracle on the host cores (rank 0 only), each step a bounded sample of the same workload.
"""
import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "jagged SiLU-attention TFLOP/s & target tokens/s, % of B200 BF16 TC peak"
WORKLOAD = "dlrmv3"  # the benchmark batch; --workload times one of the parity workloads instead
WORKLOAD_SEEDS = {"dlrmv3": 1, "jagged": 2, "long_history": 3, "streaming": 4}
FALLBACK_PEAK_TFLOPS = 1590.0
DATASHEET_PEAK_TFLOPS = 2250.0  # NVIDIA's dense bf16 figure for one B200, for context beside the measured peak
L2_FLUSH_BYTES = 256 << 20
RAB_LEN = 4096  # relative-bias table entries per head for --variant rab


# ------------------------------------------------------------------------------------ ranks
class Ranks:
    """RANK / WORLD_SIZE from the launcher; a process group only when there is more than one."""

    def __init__(self, backend="nccl"):
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x: float, device=None) -> float:
        if self.pg is None:
            return float(x)
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def sum(self, x: float, device=None) -> float:
        if self.pg is None:
            return float(x)
        import torch
        t = torch.tensor([float(x)], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of the r-th replica's lengths and of rank r's values."""
    return base_seed + 1000 * rank


def rank_workload(name, world, rank):
    """This rank's share of one global batch.  With one GPU it is the named workload itself.  With
    N GPUs the global batch is N replicas of the workload's users (replica r's lengths drawn with
    rank_seed(seed, r)); hstu_attn_partition splits it into contiguous runs of users of nearly equal
    visible-pair cost, and this rank draws Q/K/V for its run.  Returns (workload, users in the
    global batch)."""
    from hstu_pointwise_attention_jagged_b200 import binding, workloads
    base = WORKLOAD_SEEDS[name]
    if world == 1:
        w = workloads.make(name, seed=base)
        return w, w.B
    parts = [workloads.structure(name, seed=rank_seed(base, r)) for r in range(world)]
    uih, nt, cl = (np.concatenate([p[i] for p in parts]) for i in range(3))
    H, d, alpha, N = parts[0][3:]
    off = workloads.offsets_from_lengths(uih + nt)
    us = binding.hstu_attn_partition(off, nt, cl, world)
    u0, u1 = int(us[rank]), int(us[rank + 1])
    w = workloads.make_custom(name, uih[u0:u1], nt[u0:u1], H, d, alpha, N, seed=rank_seed(base, rank),
                              cached_len=cl[u0:u1])
    w.meta["description"] = workloads.CONFIGS[name][0]
    w.meta["users"] = (u0, u1)
    return w, len(uih)


# ------------------------------------------------------------------------------------ clocks
_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x1: "gpu_idle"}


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read only) while the timed loop runs."""

    def __init__(self, device_index, interval_s=0.02):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = int(pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM))
            self.ok = True
        except Exception:
            self.ok = False
        self.interval = interval_s

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(int(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)))
                bits = int(nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
                for b, name in _REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.interval)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._t is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------------------------------ helpers
def measured_peak():
    """Dense bf16 tensor peak in TFLOP/s: the measured burst figure if present, else the fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["bf16_tflops"]), "measured burst (MEASURED_PEAKS.json bf16_tflops)"
    except Exception:
        return FALLBACK_PEAK_TFLOPS, "fallback 1.59 PFLOP/s"


KERNEL_SOURCES = ("hstu_fwd_sm100.cuh", "schedule.cuh", "sm100_ptx.cuh", "hstu_attn.cu")


def kernel_source_digest():
    """sha256 over the attention kernel's sources, to tell whether recorded ncu counters are current."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "hstu_pointwise_attention_jagged_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def profiled_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, or None once the kernel changed."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("source_sha256") != kernel_source_digest():
        return None
    return int(rec["dram_bytes_per_launch"])


def workload_config(w, n_gpus, global_users=None):
    if w.name == WORKLOAD:
        name = "%s: %d users x (%d history + %d candidates), H=%d, d=%d, alpha=1/sqrt(%d), N=%d" % (
            w.name, w.B, int(w.uih_len[0]), int(w.num_targets[0]), w.H, w.d, w.d, int(w.N))
    else:
        name = "%s: %s" % (w.name, w.meta.get("description", ""))
    return {
        "workload": name,
        "users_per_gpu": w.B,
        "global_batch": int(global_users if global_users is not None else w.B * n_gpus),
        "seq_len": int(w.seq_len.max()),
        "heads": w.H,
        "head_dim": w.d,
        "parallelism": ("dp1" if n_gpus == 1 else
                        "dp%d (one batch of %d x the workload's users split into contiguous runs of equal "
                        "visible-pair cost by hstu_attn_partition; no collective)" % (n_gpus, n_gpus)),
        "l2": "flushed before every timed step (256 MiB write)",
    }


def oracle_sample_rows(w, n_rows, seed):
    """A sample of query rows of the workload: users uniformly among those with query rows, rows
    uniformly within each (with a cached prefix, among the new tokens only)."""
    rng = np.random.default_rng(seed)
    nq = w.seq_len - w.cached_len
    live = np.flatnonzero(nq > 0)
    users = live[rng.integers(0, len(live), size=n_rows)]
    local = (rng.random(n_rows) * nq[users]).astype(np.int64)
    return users.astype(np.int32), local.astype(np.int32)


def time_oracle(w, n_rows, seed):
    """Runs the oracle on a row sample; returns (seconds, algorithmic flops of the sample)."""
    import oracle
    users, local = oracle_sample_rows(w, n_rows, seed)
    cached = bool(w.cached_len.any())
    q = w.q[w.new_rows()] if cached else w.q
    t0 = time.perf_counter()
    _, macs = oracle.rows(q, w.k, w.v, w.seq_offsets, w.num_targets, w.cached_len if cached else None, w.alpha,
                          w.N, users, local, return_macs=True)
    dt = time.perf_counter() - t0
    return dt, 2 * macs


# ------------------------------------------------------------------------------------ arms
def run_ours(args, ranks):
    import torch
    from hstu_pointwise_attention_jagged_b200 import binding, metrics, workloads

    dev = torch.device("cuda", ranks.local_rank)
    torch.cuda.set_device(dev)
    binding.load_library()
    w, global_users = rank_workload(args.workload, ranks.world, ranks.rank)
    cached = bool(w.cached_len.any())
    flops = metrics.algorithmic_flops(w.seq_offsets, w.num_targets, w.H, w.d, w.cached_len if cached else None)
    targets = int(w.num_targets.sum())

    def to_bf16(x):
        return torch.from_numpy(workloads.bf16_bits(x).view(np.int16)).view(torch.bfloat16)

    # With a cached prefix (the streaming workload) the queries are the new tokens only.
    q_rows = w.q[w.new_rows()] if cached else w.q
    q_h, k_h, v_h = (to_bf16(x).pin_memory() for x in (q_rows, w.k, w.v))
    off_h = torch.from_numpy(w.seq_offsets.astype(np.int32)).pin_memory()
    nt_h = torch.from_numpy(w.num_targets.astype(np.int32)).pin_memory()
    q, k, v = (x.to(dev) for x in (q_h, k_h, v_h))
    off, nt = off_h.to(dev), nt_h.to(dev)
    cl = torch.from_numpy(w.cached_len.astype(np.int32)).to(dev) if cached else None
    total_q = int(q_h.shape[0])
    out = torch.empty_like(q)
    plan = torch.empty((binding.hstu_attn_plan_bytes(w.B, w.H, total_q),), dtype=torch.uint8, device=dev)
    flush = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    msl = w.max_seq_len

    # The relative-attention-bias variant runs through its one-call entry point (plan included).
    rab = None
    if args.variant == "rab":
        rab = torch.from_numpy(np.random.default_rng(rank_seed(5, ranks.rank)).normal(
            scale=0.02, size=(w.H, RAB_LEN)).astype(np.float32)).to(dev)

    def attn():
        if rab is None:
            binding.hstu_attn_fwd_planned(q, k, v, off, nt, cl, w.alpha, w.N, plan, out=out, stream=stream)
        else:
            binding.hstu_attn_fwd_rab(q, k, v, off, nt, rab, w.alpha, w.N, msl, cached_len=cl, out=out, stream=stream)

    def step():
        if rab is None:
            binding.hstu_attn_plan(off, nt, cl, w.H, w.total, total_q, msl, plan=plan, stream=stream)
        attn()

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    status = binding.hstu_attn_get_error()
    if status != 0:
        raise RuntimeError("warm-up reported %s" % binding.hstu_attn_status_string(status))

    K = args.steps
    # One timed loop of K iterations, L2 flushed before every timed launch.  Each iteration times
    # the whole hot path (plan + attention, no event between them, so the attention kernel's
    # programmatic early launch overlaps the plan kernel as it does for a user), then the
    # attention kernel alone on the same plan, for its roofline.  Interleaving the two makes both
    # figures see the same clocks and the same state of the GPU.
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    eva = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    ranks.barrier()
    torch.cuda.synchronize()
    with sampler:
        for i in range(K):
            flush.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
            flush.zero_()
            eva[i][0].record(stream)
            attn()
            eva[i][1].record(stream)
        torch.cuda.synchronize()
        ranks.barrier()
    step_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(K)]
    attn_ms = [eva[i][0].elapsed_time(eva[i][1]) for i in range(K)]
    status = binding.hstu_attn_get_error()
    if status != 0:
        raise RuntimeError("timed steps reported %s" % binding.hstu_attn_status_string(status))
    total_ms = ranks.max(sum(step_ms), dev)
    attn_total_ms = ranks.max(sum(attn_ms), dev)
    ms_per_step = total_ms / K
    job_flops = ranks.sum(flops, dev)
    job_targets = ranks.sum(targets, dev)
    value = job_flops / (ms_per_step * 1e-3) / 1e12
    attn_avg_ms = attn_total_ms / K
    achieved = flops / (attn_avg_ms * 1e-3) / 1e12
    peak, peak_src = measured_peak()

    # End to end: the one-shot public call with host buffers, every step's copies inside the timed
    # region.  Like a serving loop, steps alternate between two streams with their own device buffers,
    # so step i+1's upload overlaps step i's kernels and step i-1's download (PCIe carries the two
    # directions at once); a stream's next step reuses its buffers only after its previous one.
    E = max(4, min(args.steps, 50))
    h2d = sum(x.numel() * x.element_size() for x in (q_h, k_h, v_h, off_h, nt_h))
    streams = [stream, torch.cuda.Stream(dev)]
    dbufs = [(q, k, v, off, nt, out)] + [tuple(torch.empty_like(x) for x in (q, k, v, off, nt, out))]
    outs_h = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    d2h = outs_h[0].numel() * outs_h[0].element_size()

    def e2e_step(i):
        j = i % 2
        qd, kd, vd, od, nd, outd = dbufs[j]
        with torch.cuda.stream(streams[j]):
            qd.copy_(q_h, non_blocking=True)
            kd.copy_(k_h, non_blocking=True)
            vd.copy_(v_h, non_blocking=True)
            od.copy_(off_h, non_blocking=True)
            nd.copy_(nt_h, non_blocking=True)
            if rab is not None:
                binding.hstu_attn_fwd_rab(qd, kd, vd, od, nd, rab, w.alpha, w.N, msl, cached_len=cl, out=outd,
                                          stream=streams[j])
            elif cached:
                binding.hstu_attn_fwd_cached(qd, kd, vd, od, nd, cl, w.alpha, w.N, msl, out=outd, stream=streams[j])
            else:
                binding.hstu_attn_fwd(qd, kd, vd, od, nd, w.alpha, w.N, msl, out=outd, stream=streams[j])
            outs_h[j].copy_(outd, non_blocking=True)

    for i in range(4):
        e2e_step(i)
    torch.cuda.synchronize()
    ranks.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    done1 = torch.cuda.Event()
    e0.record(streams[0])
    streams[1].wait_event(e0)
    for i in range(E):
        e2e_step(i)
    done1.record(streams[1])
    streams[0].wait_event(done1)
    e1.record(streams[0])
    torch.cuda.synchronize()
    ranks.barrier()
    status = binding.hstu_attn_get_error()
    if status != 0:
        raise RuntimeError("end-to-end steps reported %s" % binding.hstu_attn_status_string(status))
    e2e_ms = ranks.max(e0.elapsed_time(e1), dev) / E
    e2e_value = job_flops / (e2e_ms * 1e-3) / 1e12

    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": ranks.world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1)/sqrt(d) bf16; DLRMv3 dataset unavailable)",
        "config": dict(workload_config(w, ranks.world, global_users), **({} if rab is None else {
            "variant": "relative attention bias: silu(alpha*s) + rab[h, min(i-j, %d)]" % (RAB_LEN - 1)})),
        "target_tokens_per_s": round(job_targets / (ms_per_step * 1e-3), 1),
        "pct_of_peak": round(100.0 * value / ranks.world / peak, 2),
        "algorithmic_gflop_per_step": round(job_flops / 1e9, 3),
        "e2e": {"value": round(e2e_value, 3), "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                "api": "%s (plan + attention) with pinned host buffers" % (
                    "hstu_attn_fwd_rab" if rab is not None else "hstu_attn_fwd_cached" if cached else "hstu_attn_fwd"),
                "pipelining": "2 streams, double-buffered device tensors: uploads, kernels and downloads of "
                              "neighbouring steps overlap; %d steps" % E},
        "gpu_launches": (3 * K if rab is None else 4 * K) + 2 * E,
        "roofline": {"bound": "tensor",
                     "kernel": ("hstu_fwd_kernel<%d, 0>" % w.d) if rab is None else (
                         "hstu_fwd_kernel<%d, rab> (+ plan kernel)" % w.d),
                     "achieved": round(achieved, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "datasheet_peak": DATASHEET_PEAK_TFLOPS,
                     "frac_of_datasheet": round(achieved / DATASHEET_PEAK_TFLOPS, 4),
                     "traffic": args.traffic if args.traffic is not None else (
                         profiled_traffic() if rab is None and args.workload == WORKLOAD else None),
                     "peak_source": peak_src,
                     "attn_ms_per_launch": round(attn_avg_ms, 5),
                     "timing": ("attention kernel alone, %d launches on one plan, L2 flushed before each" % K
                                if rab is None else
                                "hstu_attn_fwd_rab calls (plan + attention), %d, L2 flushed before each" % K),
                     "flops_per_launch": int(flops)},
        "clocks": sampler.summary(),
    }
    if ranks.rank == 0 and ranks.world == 1 and not args.no_cpu_baseline:
        import oracle
        cores = oracle.num_threads()
        t0 = time.perf_counter()
        if rab is not None:
            oracle.fwd_rab(q_rows, w.k, w.v, w.seq_offsets, w.num_targets, rab.cpu().numpy(), w.alpha, w.N,
                           cached_len=w.cached_len if cached else None)
            macs = flops // 2
        elif cached:
            _, macs = oracle.fwd_cached(q_rows, w.k, w.v, w.seq_offsets, w.num_targets, w.cached_len, w.alpha, w.N,
                                        return_macs=True)
        else:
            _, macs = oracle.fwd(w.q, w.k, w.v, w.seq_offsets, w.num_targets, w.alpha, w.N, return_macs=True)
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": 2 * macs / dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": "one full step: every row and head of the same batch (fp64 C oracle, "
                                          "OpenMP), %.1f s" % dt}
    return line


def run_proj(args, ranks):
    """The HSTU layer's two dense projections around the attention of the DLRMv3-shaped batch
    (L = 32768 token rows, D = H*d = 512): [L, D] x [D, 4D] and [L, 3D] x [3D, D], the 4*L*D^2 and
    3*L*D^2 terms of the review's per-layer FLOP formula, through hstu_attn_gemm_bf16.  cuBLAS
    (torch.matmul) is timed on the same shapes for context only."""
    import torch
    from hstu_pointwise_attention_jagged_b200 import binding, workloads

    dev = torch.device("cuda", ranks.local_rank)
    torch.cuda.set_device(dev)
    binding.load_library()
    w = workloads.make(WORKLOAD, seed=rank_seed(1, ranks.rank))
    L, D = w.total, w.H * w.d
    shapes = [(L, 4 * D, D), (L, D, 3 * D)]
    rng = np.random.default_rng(rank_seed(11, ranks.rank))

    def bf16(x):
        return torch.from_numpy(workloads.bf16_bits(workloads.round_bf16(x.astype(np.float32))).view(np.int16)).view(
            torch.bfloat16)

    host = [(bf16(rng.standard_normal((M, K))).pin_memory(), bf16(rng.standard_normal((N, K)) / np.sqrt(K)).pin_memory())
            for M, N, K in shapes]
    devm = [(a.to(dev), b.to(dev)) for a, b in host]
    outs = [torch.empty((M, N), dtype=torch.bfloat16, device=dev) for M, N, K in shapes]
    flops = sum(2 * M * N * K for M, N, K in shapes)
    flush = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        for (a, b), o in zip(devm, outs):
            binding.hstu_attn_gemm_bf16(a, b, out=o, stream=stream)

    def step_cublas():
        for (a, b), o in zip(devm, outs):
            torch.matmul(a, b.t(), out=o)

    def timed(fn, K):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
        for i in range(K):
            flush.zero_()
            ev[i][0].record(stream)
            fn()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(K))

    for _ in range(args.warmup):
        flush.zero_()
        step()
        step_cublas()
    torch.cuda.synchronize()
    if binding.hstu_attn_get_error() != 0:
        raise RuntimeError("warm-up reported an error")
    K = args.steps
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    ranks.barrier()
    torch.cuda.synchronize()
    with sampler:
        total_ms = ranks.max(timed(step, K), dev)
        cublas_ms = ranks.max(timed(step_cublas, K), dev)
        ranks.barrier()
    if binding.hstu_attn_get_error() != 0:
        raise RuntimeError("timed steps reported an error")
    ms = total_ms / K
    job_flops = ranks.sum(flops, dev)
    value = job_flops / (ms * 1e-3) / 1e12
    achieved = flops / (ms * 1e-3) / 1e12
    peak, peak_src = measured_peak()

    # End to end: inputs from pinned host memory, outputs back, every step.
    outs_h = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs]
    E = max(4, min(args.steps, 50))
    h2d = sum(a.numel() * 2 + b.numel() * 2 for a, b in host)
    d2h = sum(o.numel() * 2 for o in outs)

    def e2e_step():
        for (ah, bh), (a, b), o, oh in zip(host, devm, outs, outs_h):
            a.copy_(ah, non_blocking=True)
            b.copy_(bh, non_blocking=True)
            binding.hstu_attn_gemm_bf16(a, b, out=o, stream=stream)
            oh.copy_(o, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ranks.max(e0.elapsed_time(e1), dev) / E

    line = {
        "metric": "HSTU layer projection GEMMs TFLOP/s (input [L,D]x[D,4D] and output [L,3D]x[3D,D])",
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": ranks.world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1) activations, N(0,1/K) weights, bf16)",
        "config": {"workload": "dlrmv3 layer projections: L=%d, D=%d; shapes (M,N,K) %s" % (L, D, shapes),
                   "parallelism": "dp%d (token rows sharded, no collective)" % ranks.world,
                   "l2": "flushed before every timed step (256 MiB write)"},
        "e2e": {"value": round(job_flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": 2 * K + 2 * E,
        "roofline": {"bound": "tensor", "kernel": "gemm_bf16_kernel", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": None, "peak_source": peak_src,
                     "flops_per_step": int(flops)},
        "cublas_same_shapes": {"value": round(flops / (cublas_ms / K * 1e-3) / 1e12, 2), "unit": "TFLOP/s"},
        "clocks": sampler.summary(),
    }
    if ranks.rank == 0 and ranks.world == 1 and not args.no_cpu_baseline:
        import oracle
        rows = 2048
        t0 = time.perf_counter()
        for (ah, bh), (M, N, Kd) in zip(host, shapes):
            oracle.linear(ah[:rows].float().numpy(), bh.float().numpy())
        dt = time.perf_counter() - t0
        sample_flops = sum(2 * rows * N * Kd for M, N, Kd in shapes)
        line["cpu_baseline"] = {"value": sample_flops / dt / 1e12, "unit": "TFLOP/s", "cores": os.cpu_count(),
                                "kind": "oracle", "sample": "the first %d rows of both projections (fp64 numpy "
                                                            "matmul), %.2f s" % (rows, dt)}
    return line


def run_bwd(args, ranks):
    """Backward pass (hstu_attn_bwd: plan, dK/dV kernel, dQ kernel) over this rank's share of the
    workload, with a seeded N(0,1) output gradient.  Algorithmic flops are the five mask-exact
    matmuls of the chain rule (S, dP, dV, dK, dQ: 10 d flops per visible pair and head); the two
    the dQ kernel recomputes are not counted."""
    import torch
    from hstu_pointwise_attention_jagged_b200 import binding, metrics, workloads

    dev = torch.device("cuda", ranks.local_rank)
    torch.cuda.set_device(dev)
    binding.load_library()
    w, global_users = rank_workload(args.workload, ranks.world, ranks.rank)
    if w.cached_len.any():
        raise SystemExit("--variant bwd: the backward pass takes full sequences (no cached prefix)")
    flops = metrics.algorithmic_flops(w.seq_offsets, w.num_targets, w.H, w.d) * 10 // 4

    def to_bf16(x):
        return torch.from_numpy(workloads.bf16_bits(x).view(np.int16)).view(torch.bfloat16)

    do = workloads.round_bf16(np.random.default_rng(rank_seed(6, ranks.rank)).standard_normal(
        w.q.shape, dtype=np.float32))
    host = [to_bf16(x).pin_memory() for x in (w.q, w.k, w.v, do)]
    q, k, v, dout = (x.to(dev) for x in host)
    off = torch.from_numpy(w.seq_offsets.astype(np.int32)).to(dev)
    nt = torch.from_numpy(w.num_targets.astype(np.int32)).to(dev)
    grads = [torch.empty_like(q) for _ in range(3)]
    flush = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        binding.hstu_attn_bwd(q, k, v, dout, off, nt, w.alpha, w.N, w.max_seq_len, dq=grads[0], dk=grads[1],
                              dv=grads[2], stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if binding.hstu_attn_get_error() != 0:
        raise RuntimeError("warm-up reported an error")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    ranks.barrier()
    torch.cuda.synchronize()
    with sampler:
        for i in range(K):
            flush.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        ranks.barrier()
    if binding.hstu_attn_get_error() != 0:
        raise RuntimeError("timed steps reported an error")
    ms = ranks.max(sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(K)), dev) / K
    job_flops = ranks.sum(flops, dev)
    value = job_flops / (ms * 1e-3) / 1e12
    achieved = flops / (ms * 1e-3) / 1e12
    peak, peak_src = measured_peak()

    # End to end: q, k, v, dout and the offsets from pinned host memory, the three gradients back.
    off_h = torch.from_numpy(w.seq_offsets.astype(np.int32)).pin_memory()
    nt_h = torch.from_numpy(w.num_targets.astype(np.int32)).pin_memory()
    grads_h = [torch.empty(q.shape, dtype=q.dtype).pin_memory() for _ in range(3)]
    h2d = sum(x.numel() * x.element_size() for x in host + [off_h, nt_h])
    d2h = sum(g.numel() * g.element_size() for g in grads_h)
    E = max(4, min(args.steps, 50))

    def e2e_step():
        for dst, src in zip((q, k, v, dout, off, nt), host + [off_h, nt_h]):
            dst.copy_(src, non_blocking=True)
        step()
        for gh, g in zip(grads_h, grads):
            gh.copy_(g, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ranks.max(e0.elapsed_time(e1), dev) / E
    line = {
        "metric": "jagged SiLU-attention backward TFLOP/s (dQ, dK, dV)",
        "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": ranks.world, "steps": K, "warmup": args.warmup,
        "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded N(0,1)/sqrt(d) bf16 inputs, N(0,1) output gradient)",
        "config": dict(workload_config(w, ranks.world, global_users), variant="backward pass"),
        "e2e": {"value": round(job_flops / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": 3 * (K + E),
        "roofline": {"bound": "tensor", "kernel": "hstu_bwd_kernel<%d, dK/dV> + <%d, dQ> (+ plan)" % (w.d, w.d),
                     "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": None, "peak_source": peak_src,
                     "flops_per_step": int(flops)},
        "clocks": sampler.summary(),
    }
    return line


LAYERS = 3  # stacked HSTU layers for --variant layer


def run_layer(args, ranks):
    """A stack of HSTU layers (projection GEMM, attention with the [U | A | U*A] epilogue, projection
    GEMM; one work plan for all layers) through hstu_layers_fwd, on this rank's share of the
    workload with D = H d.  `value` counts the review's per-layer FLOP formula,
    2 * layers * sum_users (L*L*D/2 + 4*L*D^2 + 3*L*D^2) with L each user's length (DLRMv3 review,
    section "model selection"); the mask-exact count (projections plus visible pairs) is reported
    beside it."""
    import torch
    from hstu_pointwise_attention_jagged_b200 import binding, metrics, workloads

    dev = torch.device("cuda", ranks.local_rank)
    torch.cuda.set_device(dev)
    binding.load_library()
    w, global_users = rank_workload(args.workload, ranks.world, ranks.rank)
    if w.cached_len.any():
        raise SystemExit("--variant layer: layers take full sequences (no cached prefix)")
    H, d, D, L = w.H, w.d, w.H * w.d, w.total
    lens = w.seq_len
    page_flops = int(2 * LAYERS * sum(int(l) * int(l) * D // 2 + 7 * int(l) * D * D for l in lens))
    exact_flops = LAYERS * (2 * L * D * 7 * D + metrics.algorithmic_flops(w.seq_offsets, w.num_targets, H, d))
    rng = np.random.default_rng(rank_seed(12, ranks.rank))

    def bf16(a):
        return torch.from_numpy(workloads.bf16_bits(workloads.round_bf16(a.astype(np.float32))).view(np.int16)).view(
            torch.bfloat16)

    x_h = bf16(rng.standard_normal((L, D))).pin_memory()
    w1 = [bf16(rng.standard_normal((4 * D, D)) / np.sqrt(D)).to(dev) for _ in range(LAYERS)]
    w2 = [bf16(rng.standard_normal((D, 3 * D)) / np.sqrt(3 * D)).to(dev) for _ in range(LAYERS)]
    x = x_h.to(dev)
    off_h = torch.from_numpy(w.seq_offsets.astype(np.int32)).pin_memory()
    nt_h = torch.from_numpy(w.num_targets.astype(np.int32)).pin_memory()
    off, nt = off_h.to(dev), nt_h.to(dev)
    ws = torch.empty((binding.hstu_layer_workspace_bytes(H, d, L, LAYERS),), dtype=torch.uint8, device=dev)
    y = torch.empty_like(x)
    flush = torch.empty((L2_FLUSH_BYTES // 4,), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        binding.hstu_layers_fwd(x, w1, w2, off, nt, H, d, w.alpha, w.N, w.max_seq_len, workspace=ws, y=y,
                                stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if binding.hstu_attn_get_error() != 0:
        raise RuntimeError("warm-up reported an error")
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    ranks.barrier()
    torch.cuda.synchronize()
    with sampler:
        for i in range(K):
            flush.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        ranks.barrier()
    if binding.hstu_attn_get_error() != 0:
        raise RuntimeError("timed steps reported an error")
    ms = ranks.max(sum(ev[i][0].elapsed_time(ev[i][1]) for i in range(K)), dev) / K
    job_page = ranks.sum(page_flops, dev)
    job_exact = ranks.sum(exact_flops, dev)
    peak, peak_src = measured_peak()

    # End to end: the input activations and offsets from pinned host memory, the output back.
    y_h = torch.empty(y.shape, dtype=y.dtype).pin_memory()
    E = max(4, min(args.steps, 50))

    def e2e_step():
        x.copy_(x_h, non_blocking=True)
        off.copy_(off_h, non_blocking=True)
        nt.copy_(nt_h, non_blocking=True)
        step()
        y_h.copy_(y, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = ranks.max(e0.elapsed_time(e1), dev) / E
    h2d = sum(t.numel() * t.element_size() for t in (x_h, off_h, nt_h))
    return {
        "metric": "HSTU layer stack TFLOP/s by the review's formula 2*layers*(L^2 D/2 + 7 L D^2)",
        "value": round(job_page / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": ranks.world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations, N(0,1/fan_in) weights, bf16)",
        "config": dict(workload_config(w, ranks.world, global_users), layers=LAYERS, model_dim=D,
                       variant="HSTU layer stack: [U|V|Q|K] = X W1^T, attention, Y = [U|A|U*A] W2^T"),
        "exact_tflops": round(job_exact / (ms * 1e-3) / 1e12, 2),
        "page_gflop_per_step": round(job_page / 1e9, 3), "exact_gflop_per_step": round(job_exact / 1e9, 3),
        "e2e": {"value": round(job_page / (e2e_ms * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(y_h.numel() * y_h.element_size())},
        "gpu_launches": (1 + 3 * LAYERS) * (K + E),
        "roofline": {"bound": "tensor", "kernel": "layer stack (gemm_bf16_kernel x2 + hstu_fwd_kernel per layer)",
                     "achieved": round(exact_flops / (ms * 1e-3) / 1e12, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(exact_flops / (ms * 1e-3) / 1e12 / peak, 4), "traffic": None,
                     "peak_source": peak_src, "flops_per_step": int(exact_flops)},
        "clocks": sampler.summary(),
    }


def run_reference(args, world):
    """The fp64 oracle on the host cores, rank 0 only: each step a bounded row sample, sized so that
    warm-up plus K steps stay near a minute of CPU work."""
    import oracle
    from hstu_pointwise_attention_jagged_b200 import workloads
    w = workloads.make(args.workload, seed=rank_seed(WORKLOAD_SEEDS[args.workload], 0))
    cores = oracle.num_threads()
    rows = args.ref_rows or int(min(8000, max(16, 240000 // (args.steps + args.warmup))))
    for i in range(args.warmup):
        time_oracle(w, rows, seed=900 + i)
    secs, fl = 0.0, 0
    for i in range(args.steps):
        dt, f = time_oracle(w, rows, seed=1000 + i)
        secs += dt
        fl += f
    value = fl / secs / 1e12
    ms_step = secs / args.steps * 1e3
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1)/sqrt(d) bf16 values; DLRMv3 dataset unavailable)",
        "config": workload_config(w, world),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": "each step: %d random query rows x %d heads of the batch" % (rows, w.H)},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--ref-rows", type=int, default=0, help="rows per step of the reference arm (0: sized from K)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=sorted(WORKLOAD_SEEDS), default=WORKLOAD,
                    help="batch to time (default: the DLRMv3-shaped benchmark batch)")
    ap.add_argument("--variant", choices=["plain", "rab", "proj", "bwd", "layer"], default="plain",
                    help="layer: a stack of %d HSTU layers; bwd: the backward pass; rab: the relative-attention-bias variant (a %d-entry table per "
                         "head); proj: the layer's "
                         "projection GEMMs" % (LAYERS, RAB_LEN))
    ap.add_argument("--traffic", type=float, default=None,
                    help="DRAM bytes per attention launch from an ncu capture of this kernel, if current")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != args.gpus:
        ap.error("--gpus %d but WORLD_SIZE=%d (launch N>1 with torch.distributed.run)" % (args.gpus, world))
    if args.impl == "reference":
        # Rank 0 alone runs the CPU oracle; other ranks exit without work (no process group).
        if int(os.environ.get("RANK", "0")) == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return 0
    ranks = Ranks(backend="nccl")
    try:
        run = {"proj": run_proj, "bwd": run_bwd, "layer": run_layer}.get(args.variant, run_ours)
        line = run(args, ranks)
    finally:
        ranks.close()
    if ranks.rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
