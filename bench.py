"""Benchmark of one SparsePR attention call (all seven steps) on B200 GPUs.

`python bench.py --gpus N --steps K --warmup W` times K calls of
sparsepr_attention on the HunyuanVideo-shaped 720p workload (B=1, 24 heads,
d=128, N=118800, rho_exec=22%) per GPU and prints one JSON line. Each rank
processes its own call on its own seeded inputs (weak scaling, no data-path
collective); the time is the max over ranks of CUDA-event time.

`--impl reference` times the CPU oracle instead (the reference arm of this
build): a bounded sample of the same workload, scaled to the same metric.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "SparsePR attn ms/call & dense-equiv TFLOPS at N=118800, 24 heads, rho=22%"
UNIT = "TFLOPS (dense-equivalent)"
DEFAULT_WORKLOAD = "hunyuan720p_n118800"


# ----------------------------------------------------------------------------- distributed helpers

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def dist_init(backend: str, timeout_s: int = 300):
    import datetime

    import torch.distributed as dist

    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world


def reduce_max(value: float, device) -> float:
    """Max of a scalar over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def attn_traffic_bytes(useful_flops: float):
    """DRAM bytes (read + write) of one block-sparse attention launch, scaled from the committed
    small-case ncu capture (profiles/attn_tc_kernel_sweep_n32760_rho22.md: its traffic per launch
    and its launch's useful FLOPs) by the ratio of useful FLOPs (the attention's DRAM traffic is
    its K/V tile reads, which grow with the routed pairs). None once the kernel source differs
    from the one the counters were taken on."""
    import hashlib
    import re

    root = os.path.dirname(os.path.abspath(__file__))
    try:
        text = open(os.path.join(root, "profiles", "attn_tc_kernel_sweep_n32760_rho22.md")).read()
        src = open(os.path.join(root, "free_block_sparse_sparsepr_b200", "csrc", "attention_tc.cu"), "rb").read()
    except OSError:
        return None
    m_t = re.search(r"traffic_bytes_per_launch:\s*([0-9]+)", text)
    m_f = re.search(r"useful_flops_per_launch:\s*([0-9.eE+]+)", text)
    m_h = re.search(r"source_sha256_16:\s*([0-9a-f]{16})", text)
    if not (m_t and m_f and m_h) or hashlib.sha256(src).hexdigest()[:16] != m_h.group(1):
        return None
    return int(int(m_t.group(1)) * useful_flops / float(m_f.group(1)))


def whole_job_value(flops_per_rank: float, world: int, ms_max: float) -> float:
    """Dense-equivalent TFLOPS of the whole job: all ranks' work over the slowest rank's time."""
    return flops_per_rank * world / (ms_max * 1e-3) / 1e12


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self) -> dict:
        if not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax.append(float(p[2]))
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        under = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(under), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- peaks

def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"bf16_tflops": d["bf16_tflops"], "bf16_tflops_sustained": d["bf16_tflops_sustained"],
                "hbm_gbs": d["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0, "source": "fallback"}


# ----------------------------------------------------------------------------- oracle (CPU) sample

CPU_SAMPLE_GROUPS = 8          # query groups of the fixed attention sample
CPU_WHOLE_HEAD_N = 16384       # up to this length the sample attends every query group (no scaling)
_SAMPLE_INPUTS = {}


def sample_groups(Gq: int, n: int = CPU_SAMPLE_GROUPS) -> np.ndarray:
    """The fixed, stratified query-group sample: groups floor((2i + 1) Gq / 2n), i < n (group ids
    follow the k-means seeds, which are spread evenly over the token order)."""
    n = min(n, Gq)
    return np.array([((2 * i + 1) * Gq) // (2 * n) for i in range(n)], dtype=np.int64)


def oracle_sample(w):
    """Time the CPU oracle on one fixed sample of workload w and scale it to one whole call.

    The sample is KV head 0 with all its query heads: its whole partition and route (all N rows),
    exact sparse attention for the rows of CPU_SAMPLE_GROUPS fixed query groups (sample_groups;
    every query group, so no scaling, when N <= CPU_WHOLE_HEAD_N),
    the sparse output at the M probe rows, the probe fit (dense probe rows, ridge, subspace) and
    the correction of an N x d output. Only the sampled attention is scaled, by routed pairs (the
    head's routed pairs over the sampled groups' routed pairs: the attention work is proportional
    to pairs, not rows); every other stage is timed whole. One call = B*Hkv such KV heads.
    Returns (seconds per call, per-stage seconds of the sample, sample description).
    """
    import oracle
    from synthetic import bf16_bits_to_f64, video_qkv

    one = w.replace(B=1, Hq=w.g, Hkv=1)
    if one not in _SAMPLE_INPUTS:
        _SAMPLE_INPUTS.clear()
        _SAMPLE_INPUTS[one] = tuple(bf16_bits_to_f64(x) for x in video_qkv(one))
    Q, K, V = _SAMPLE_INPUTS[one]
    Qg, Kh, Vh = Q[0], K[0, 0], V[0, 0]
    st = dict.fromkeys(("partition", "route", "attention_sample", "probe_rows_sparse", "fit", "correction"), 0.0)
    t0 = time.perf_counter()
    part = oracle.partition_head(Qg, Kh, one)
    t1 = time.perf_counter()
    rt = oracle.route_head(Qg, part, one)
    t2 = time.perf_counter()
    st["partition"], st["route"] = t1 - t0, t2 - t1
    groups = np.arange(w.Gq) if w.N <= CPU_WHOLE_HEAD_N else sample_groups(w.Gq)
    rows = np.nonzero(np.isin(part.qgroup, groups))[0]
    qsize, ksize = np.diff(part.qoff), np.diff(part.koff)
    sampled_pairs = int((qsize[groups] * (rt.sel[groups] * ksize[None, :]).sum(axis=1)).sum())
    for j in range(w.g):
        ta = time.perf_counter()
        o_rows, _ = oracle.sparse_attention(Qg[j], Kh, Vh, part.qgroup, part.kgroup, rt.sel, rows=rows)
        tb = time.perf_counter()
        o_probe, _ = oracle.sparse_attention(Qg[j], Kh, Vh, part.qgroup, part.kgroup, rt.sel, rows=part.probe)
        tc = time.perf_counter()
        fit = oracle.fit_head(Qg[j], Kh, Vh, o_probe[part.probe], part, one)
        td = time.perf_counter()
        o_full = np.resize(o_rows[rows], (w.N, w.d))       # an N x d output: the correction's cost
        oracle.correction(o_full, fit.U, fit.A, fit.obar, fit.Rbar)
        te = time.perf_counter()
        st["attention_sample"] += tb - ta
        st["probe_rows_sparse"] += tc - tb
        st["fit"] += td - tc
        st["correction"] += te - td
    scale = rt.pairs / max(sampled_pairs, 1)
    per_head = (st["partition"] + st["route"] + st["attention_sample"] * scale + st["probe_rows_sparse"]
                + st["fit"] + st["correction"])
    per_call = per_head * w.Hkv * w.B
    which = ("every query group" if len(groups) == w.Gq else
             f"query groups {groups.tolist()} of {w.Gq} ({len(rows)} rows, {sampled_pairs} of {rt.pairs} routed pairs), "
             "scaled by routed pairs")
    desc = (f"KV head 0 of {w.name} with its {w.g} query head(s): whole partition, route, probe rows, fit and "
            f"correction; exact sparse attention for {which}; x {w.B * w.Hkv} KV heads")
    stages = dict(st, attention_scale=scale, sampled_pairs=sampled_pairs, routed_pairs=int(rt.pairs))
    return per_call, stages, desc


def cpu_cores_used() -> int:
    """Threads the oracle's BLAS actually uses (its matrix products dominate), else the core count."""
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


# ----------------------------------------------------------------------------- arms

def run_reference(args):
    """The oracle on the host cores: the reference arm (rank 0 only under torchrun)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from synthetic import get_workload

    w = get_workload(args.workload)
    # warm-up: the same code paths on the smallest configuration (imports, BLAS thread pools)
    for _ in range(args.warmup):
        oracle_sample(get_workload("tiny_n1024"))
    vals, stages = [], []
    sample_desc = ""
    for _ in range(args.steps):
        per_call, st, sample_desc = oracle_sample(w)
        vals.append(per_call)
        stages.append(st)
    per_call = statistics.mean(vals)
    value = w.dense_equiv_flops() / per_call / 1e12
    cores = cpu_cores_used()
    stage_s = {k: statistics.mean(x[k] for x in stages) for k in stages[0]}
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": per_call * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, world=1),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "cpu_count": os.cpu_count(),
                         "kind": "oracle", "sample": sample_desc, "sample_stage_seconds": stage_s,
                         "ms_per_call_scaled": per_call * 1e3},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, world: int) -> dict:
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "grid_thw": [w.T, w.Hg, w.Wg],
            "d": w.d, "Gk": w.Gk, "Gq": w.Gq, "block": w.block, "rho_exec_target": w.rho, "rK": w.rK,
            "rQ": w.rQ, "M": w.M, "r": w.r, "lambda": w.lam, "kmeans_iters": w.kmeans_iters,
            "parallelism": f"independent calls on {world} GPU(s), one per rank (no collective)",
            "l2": "inputs larger than L2 (Q, K, V are 730 MB each; no flush needed)"}


def run_ours(args):
    import torch

    import free_block_sparse_sparsepr_b200 as spr
    from synthetic import get_workload, video_qkv

    rank, world = dist_init("nccl" if torch.cuda.is_available() else "gloo")
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = get_workload(args.workload)

    # seeded inputs of this rank's call, resident in HBM
    Qb, Kb, Vb = video_qkv(w, layer=rank)
    host = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) for x in (Qb, Kb, Vb)]
    q, k, v = (t.to(dev) for t in host)
    O = torch.empty_like(q)
    h = spr.SparsePR.from_workload(w)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        h.attention(q, k, v, O)
    torch.cuda.synchronize()
    launches = h.last_launch_count()
    st = h.stats()

    # timed region: K calls, per-stage events of every call on the launching stream
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]
    for row in evs:            # torch creates the CUDA event on its first record
        for e in row:
            e.record(stream)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for i in range(args.steps):
            h.set_stage_events(evs[i])
            h.attention(q, k, v, O)
        end.record(stream)
        torch.cuda.synchronize()
    barrier()
    h.set_stage_events(None)
    ms = start.elapsed_time(end) / args.steps
    ms_max = reduce_max(ms, dev)
    stage_names = ["partition", "route", "permute", "attention", "probe_fit", "writeback"]
    stage_ms = {n: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps))
                for j, n in enumerate(stage_names)}
    st = h.stats()
    flops = w.dense_equiv_flops()
    value = whole_job_value(flops, world, ms_max)

    # roofline of the dominant kernel: block-sparse attention on the routed cells
    peaks = measured_peaks()
    routed_pairs = st["route_density"] * float(w.N) ** 2 * w.B * w.Hq
    attn_flops = 4.0 * w.d * routed_pairs
    achieved = attn_flops / (stage_ms["attention"] * 1e-3) / 1e12
    peak = peaks["bf16_tflops_sustained"]
    roofline = {"bound": "tensor", "kernel": "block-sparse attention (routed cells)", "achieved": achieved,
                "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": attn_traffic_bytes(attn_flops),
                "traffic_source": "small-case ncu capture scaled by useful FLOPs",
                "peak_kind": f"bf16 sustained ({peaks['source']})",
                "useful_flops_per_launch": attn_flops}

    # end to end through the public API with HOST buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        pin = [t.pin_memory() for t in host]
        Oh = torch.empty_like(pin[0]).pin_memory()
        h.attention_host(*pin, Oh)
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        nsteps = max(1, args.steps)
        barrier()
        torch.cuda.synchronize()
        e_start.record(stream)
        for _ in range(nsteps):
            h.attention_host(*pin, Oh)
        e_end.record(stream)
        torch.cuda.synchronize()
        barrier()
        e_ms = reduce_max(e_start.elapsed_time(e_end) / nsteps, dev)
        h2d = sum(t.numel() * t.element_size() for t in pin)
        e2e = {"value": whole_job_value(flops, world, e_ms), "unit": UNIT, "ms_per_step": e_ms, "steps": nsteps,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": Oh.numel() * Oh.element_size()}

    # dense baseline of the same library on the same shapes
    dense = None
    if not args.no_dense:
        Od = torch.empty_like(q)
        for _ in range(max(1, args.warmup)):
            h.dense_attn(q, k, v, Od)
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        dsteps = max(1, args.steps)
        barrier()
        torch.cuda.synchronize()
        d0.record(stream)
        for _ in range(dsteps):
            h.dense_attn(q, k, v, Od)
        d1.record(stream)
        torch.cuda.synchronize()
        barrier()
        dms = reduce_max(d0.elapsed_time(d1) / dsteps, dev)
        dense = {"ms_per_call": dms, "steps": dsteps, "tflops": flops / (dms * 1e-3) / 1e12,
                 "speedup_vs_dense": dms / ms_max,
                 "frac_of_peak": flops / (dms * 1e-3) / 1e12 / peaks["bf16_tflops_sustained"]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        per_call, stages, desc = oracle_sample(w)
        cpu = {"value": flops / per_call / 1e12, "unit": UNIT, "cores": cpu_cores_used(), "cpu_count": os.cpu_count(),
               "kind": "oracle", "sample": desc, "sample_stage_seconds": stages, "ms_per_call_scaled": per_call * 1e3}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, world),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches * args.steps,
            "clocks": clk.summary(),
            "stage_ms": stage_ms,
            "realised": {"route_density": st["route_density"], "rho_exec": st["rho_exec"]},
            "dense_baseline": dense,
            "impl": "ours",
        }
        print(json.dumps(line), flush=True)
    h.close()
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


def run_stack(args):
    """A stack of `--layers` calls (one per denoising-step layer: fresh seeded inputs, locality
    drawn per layer), two handles on two streams so that consecutive layers overlap, captured
    once in a CUDA graph and replayed. Times the stack eagerly on one stream, eagerly on two
    streams and as the graph (each after warm-up, CUDA events, max over ranks)."""
    import torch
    import torch.distributed as dist

    import free_block_sparse_sparsepr_b200 as spr
    from synthetic import get_workload, video_qkv_device
    from synthetic.workloads import stack_layer_locality

    rank, world = dist_init("nccl" if torch.cuda.is_available() else "gloo")
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = get_workload(args.workload)
    L = args.layers
    ins = [video_qkv_device(w, layer=1000 * rank + l, locality=stack_layer_locality(l, w.seed), device=str(dev))
           for l in range(L)]
    outs = [torch.empty_like(q) for q, _, _ in ins]
    hs = [spr.SparsePR.from_workload(w) for _ in range(2)]
    streams = [torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)]

    def stack(two: bool):
        cur = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(cur)
        for s in streams:
            s.wait_event(fork)
        for l, (q, k, v) in enumerate(ins):
            i = l % 2 if two else 0
            with torch.cuda.stream(streams[i]):
                hs[i].attention(q, k, v, outs[l])
        for s in streams:
            join = torch.cuda.Event()
            join.record(s)
            cur.wait_event(join)

    def timed(fn, reps):
        cur = torch.cuda.current_stream()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        a.record(cur)
        for _ in range(reps):
            fn()
        b.record(cur)
        torch.cuda.synchronize()
        barrier()
        return reduce_max(a.elapsed_time(b) / reps, dev)

    for _ in range(max(1, args.warmup)):
        stack(True)
    torch.cuda.synchronize()
    eager1 = timed(lambda: stack(False), 1)
    eager2 = timed(lambda: stack(True), 1)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        stack(True)
    for _ in range(args.warmup):
        graph.replay()
    with ClockSampler(local) as clk:
        ms = timed(graph.replay, args.steps)
    flops = w.dense_equiv_flops() * L
    if rank == 0:
        print(json.dumps({
            "metric": f"SparsePR {L}-layer stack (CUDA graph, two streams): dense-equiv TFLOPS",
            "value": whole_job_value(flops, world, ms), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "ms_per_call": ms / L, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (drawn on the GPU)",
            "config": dict(workload_config(w, world), layers=L,
                           locality="U[0.4, 1.2] per layer, fresh seeded inputs per layer"),
            "eager_one_stream_ms_per_call": eager1 / L, "eager_two_streams_ms_per_call": eager2 / L,
            "graph_two_streams_ms_per_call": ms / L, "gpu_launches": hs[0].last_launch_count() * L,
            "clocks": clk.summary(),
        }), flush=True)
    del graph
    for hh in hs:
        hh.close()
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


def run_sharded(args):
    """One call split by KV heads over the ranks (strong scaling): every rank draws the same
    seeded inputs, runs its shard of heads, and the output is all-gathered over NCCL. Times the
    sharded call alone and the call followed by the gather (CUDA events, max over ranks); value
    is the whole call's dense-equivalent FLOPs over the slower of the two rank times."""
    import torch
    import torch.distributed as dist

    from free_block_sparse_sparsepr_b200.sharding import ShardedSparsePR, head_range
    from synthetic import get_workload, video_qkv_device

    rank, world = dist_init("nccl" if torch.cuda.is_available() else "gloo")
    _, _, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = get_workload(args.workload)
    Q, K, V = video_qkv_device(w, layer=0, locality=w.locality, device=str(dev))
    sh = ShardedSparsePR(w.B, w.Hq, w.Hkv, w.N, w.d, Gk=w.Gk, Gq=w.Gq, block=w.block, rK=w.rK, rQ=w.rQ, M=w.M,
                         r=w.r, kmeans_iters=w.kmeans_iters, lam=w.lam, rho_exec=w.rho, seed=w.seed)

    def timed(fn, reps):
        cur = torch.cuda.current_stream()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        a.record(cur)
        for _ in range(reps):
            fn()
        b.record(cur)
        torch.cuda.synchronize()
        barrier()
        return reduce_max(a.elapsed_time(b) / reps, dev)

    for _ in range(max(3, args.warmup)):
        sh.attention(Q, K, V, gather=world > 1)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms = timed(lambda: sh.attention(Q, K, V), args.steps)
    ms_gather = timed(lambda: sh.attention(Q, K, V, gather=True), args.steps) if world > 1 else ms
    launches = sh.handle.last_launch_count() if sh.handle is not None else 0
    if rank == 0:
        print(json.dumps({
            "metric": METRIC + " (one call sharded by KV heads)",
            "value": w.dense_equiv_flops() / (ms * 1e-3) / 1e12, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "ms_per_step_with_gather": ms_gather,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (drawn on the GPU)",
            "config": dict(workload_config(w, world), parallelism=f"heads{world}",
                           heads_per_rank=[hi - lo for lo, hi in (head_range(w.B * w.Hkv, world, r)
                                                                  for r in range(world))]),
            "gpu_launches": launches, "clocks": clk.summary(),
        }), flush=True)
    sh.close()
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
    return 0


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--layers", type=int, default=1,
                    help="> 1: time a stack of this many calls as one CUDA graph (two streams)")
    ap.add_argument("--shard-heads", action="store_true",
                    help="split one call's KV heads over the ranks and all-gather O (strong scaling)")
    return ap.parse_args(argv)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.layers > 1:
        return run_stack(args)
    if args.shard_heads:
        return run_sharded(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
