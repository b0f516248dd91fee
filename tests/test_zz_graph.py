"""A SparsePR call captured in a CUDA graph: the call launches only kernels (no host
synchronisation, no allocation), so a stack of calls on two handles and two streams can be
captured once and replayed; the replay must reproduce the eager outputs bit for bit."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import free_block_sparse_sparsepr_b200 as spr  # noqa: E402
from synthetic import get_workload, video_qkv_device  # noqa: E402
from synthetic.workloads import stack_layer_locality  # noqa: E402

pytestmark = pytest.mark.gpu


def test_graph_replay_of_a_two_stream_stack():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    spr.load_library()
    w = get_workload("mid_n16384").replace(Hq=4, Hkv=4)
    L = 4
    ins = [video_qkv_device(w, layer=l, locality=stack_layer_locality(l)) for l in range(L)]
    eager = [torch.empty_like(q) for q, _, _ in ins]
    replay = [torch.empty_like(q) for q, _, _ in ins]
    hs = [spr.SparsePR.from_workload(w) for _ in range(2)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]

    def stack(outs):
        cur = torch.cuda.current_stream()
        fork = torch.cuda.Event()
        fork.record(cur)
        for s in streams:
            s.wait_event(fork)
        for l, (q, k, v) in enumerate(ins):
            with torch.cuda.stream(streams[l % 2]):
                hs[l % 2].attention(q, k, v, outs[l])
        for s in streams:
            join = torch.cuda.Event()
            join.record(s)
            cur.wait_event(join)

    stack(eager)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        stack(replay)
    for _ in range(2):
        for o in replay:
            o.zero_()
        g.replay()
        torch.cuda.synchronize()
        for l in range(L):
            assert torch.equal(eager[l], replay[l]), f"layer {l}"
    assert all(h.device_status() == 0 for h in hs)
    assert not torch.equal(eager[0], eager[1])          # layers differ
    del g
    for h in hs:
        h.close()
