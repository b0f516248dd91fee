"""The multi-rank path of bench.py on CPU: two gloo ranks (no GPU) run the host logic the
driver's torchrun launch exercises — rendezvous, the max-over-ranks reduction of the timed
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
