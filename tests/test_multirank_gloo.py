"""The multi-rank path of bench.py on CPU: two gloo ranks (no GPU) run the host logic that a
torchrun launch of bench.py exercises — rendezvous, the max-over-ranks reduction of the timed
region, the barrier, the whole-job value (all ranks' work over the slowest rank's time), the
per-rank seeding of the inputs, and the reference arm's rule that rank 0 alone runs and prints."""
import contextlib
import io
import json
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench
    from synthetic import get_workload, video_qkv

    try:
        r, w = bench.dist_init("gloo", timeout_s=60)
        ms = bench.reduce_max(10.0 + 5.0 * rank, "cpu")
        bench.barrier()
        value = bench.whole_job_value(2e12, w, ms)
        wl = get_workload("tiny_n1024")
        Qb, _, _ = video_qkv(wl, layer=r)
        buf = io.StringIO()
        args = bench.parse_args(["--impl", "reference", "--workload", "tiny_n1024", "--steps", "1", "--warmup", "0",
                                 "--gpus", str(world)])
        with contextlib.redirect_stdout(buf):
            rc = bench.run_reference(args)
        bench.barrier()
        out.put((rank, r, w, ms, value, int(Qb[0, 0, :64].astype(np.int64).sum()), rc, buf.getvalue()))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, rr0, w0, ms0, v0, s0, rc0, o0), (r1, rr1, w1, ms1, v1, s1, rc1, o1) = res
    assert (rr0, rr1, w0, w1) == (0, 1, 2, 2)
    assert ms0 == ms1 == 15.0                        # max over ranks
    assert v0 == v1 == pytest.approx(2e12 * 2 / 15e-3 / 1e12)
    assert s0 != s1                                  # each rank draws its own seeded inputs
    assert rc0 == rc1 == 0
    assert o1 == ""                                  # rank 1 does no reference work
    line = json.loads(o0.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"


def _dense_heads(q, k, v):
    """Plain softmax attention per query head (q [n*g, N, d], k, v [n, N, d]), fp64 on CPU."""
    import torch

    g = q.shape[0] // k.shape[0]
    kk = k.repeat_interleave(g, dim=0)
    vv = v.repeat_interleave(g, dim=0)
    s = (q @ kk.transpose(1, 2)) / q.shape[-1] ** 0.5
    return torch.softmax(s, dim=-1) @ vv


def _shard_worker(rank, world, port, out, B, Hq, Hkv):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    from free_block_sparse_sparsepr_b200.sharding import ShardedSparsePR

    try:
        dist.init_process_group("gloo", rank=rank, world_size=world)
        N, d = 24, 8
        gen = torch.Generator().manual_seed(11)                     # same full inputs on every rank
        Q = torch.randn(B, Hq, N, d, generator=gen, dtype=torch.float64)
        K = torch.randn(B, Hkv, N, d, generator=gen, dtype=torch.float64)
        V = torch.randn(B, Hkv, N, d, generator=gen, dtype=torch.float64)
        sh = ShardedSparsePR(B, Hq, Hkv, N, d, compute=_dense_heads)
        O_local = sh.attention(Q, K, V)
        O_all = sh.attention(Q, K, V, gather=True)
        ref = _dense_heads(Q.reshape(B * Hq, N, d), K.reshape(B * Hkv, N, d), V.reshape(B * Hkv, N, d))
        out.put((rank, sh.lo, sh.hi, bool(torch.equal(O_all, ref)),
                 bool(torch.equal(O_local, ref[sh.lo * (Hq // Hkv): sh.hi * (Hq // Hkv)]))))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world,B,Hq,Hkv", [(2, 1, 8, 2), (3, 2, 8, 4), (4, 1, 6, 3)])
def test_head_sharded_gather(world, B, Hq, Hkv):
    """Head sharding on gloo ranks: shards tile the flattened KV heads (sizes within one, a rank
    may hold none), each rank's output is its slice of the unsharded result, and the all-gather
    returns the whole output in head order on every rank."""
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, out, B, Hq, Hkv)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    P = B * Hkv
    assert res[0][1] == 0 and res[-1][2] == P
    assert all(res[i][2] == res[i + 1][1] for i in range(world - 1))
    sizes = [hi - lo for _, lo, hi, _, _ in res]
    assert max(sizes) - min(sizes) <= 1
    assert all(r[3] and r[4] for r in res)


def test_head_range_tiles():
    from free_block_sparse_sparsepr_b200.sharding import head_range

    for P in (1, 5, 24, 64):
        for world in (1, 2, 3, 8):
            ranges = [head_range(P, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == P
            assert all(ranges[i][1] == ranges[i + 1][0] for i in range(world - 1))
            assert max(b - a for a, b in ranges) - min(b - a for a, b in ranges) <= 1
