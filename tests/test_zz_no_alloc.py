"""The allocation-free probe-row attention entry point, through the C ABI.

Callers that cannot allocate device memory (a framework that owns all device
allocations, code under an allocator lock, a process with a fixed memory
reservation) use sparsepr_probe_attention_noalloc instead of a handle. Its
output must match the handle-based probe pass of sparsepr_probe_fit within
the tolerance of the other parity tests, on two calls in a row (the second
call reuses the library's fixed scratch array left over from the first).
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import free_block_sparse_sparsepr_b200 as spr  # noqa: E402
from synthetic import get_workload, video_qkv  # noqa: E402

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def _entry():
    lib = spr.load_library()
    f = lib.sparsepr_probe_attention_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 6 + [ctypes.c_void_p]
    return f


def test_noalloc_probe_attention_matches_probe_fit_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = get_workload("mid_n16384").replace(Hq=4, Hkv=2)          # GQA: 2 query heads per KV head
    Qb, Kb, Vb = video_qkv(w)
    q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda() for x in (Qb, Kb, Vb))
    with spr.SparsePR.from_workload(w) as h:
        part = h.partition(q, k)
        route = h.route(q, part)
        Qp, Kp, Vp, Osp = (torch.empty_like(t) for t in (q, k, v, q))
        h.permute(q, k, v, part, Qp, Kp, Vp)
        h.blocksparse_attn(Qp, Kp, Vp, part, route, Osp)
        fit = h.probe_fit(q, k, v, part, Osp)
        torch.cuda.synchronize()
        ref = h.fit_views(fit)["Odense"].clone()
        rows = h.partition_views(part)["probe"].clone()
    f = _entry()
    stream = torch.cuda.current_stream().cuda_stream
    out = torch.empty_like(ref)
    results = []
    for _ in range(2):
        out.fill_(float("nan"))
        code = f(q.data_ptr(), k.data_ptr(), v.data_ptr(), rows.data_ptr(), out.data_ptr(),
                 w.B, w.Hq, w.Hkv, w.N, w.d, w.M, stream)
        assert code == 0, spr.STATUS.get(code, code)
        torch.cuda.synchronize()
        diff = (out - ref).abs()
        assert torch.isfinite(out).all()
        assert diff.max().item() <= MAX_ABS and diff.mean().item() <= MEAN_ABS, (diff.max().item(), diff.mean().item())
        results.append(out.clone())
    assert torch.equal(results[0], results[1])


def test_noalloc_rejects_requests_beyond_the_static_maximum():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    f = _entry()
    x = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    r = torch.zeros(4, dtype=torch.int32, device="cuda")
    o = torch.zeros(4, dtype=torch.float32, device="cuda")
    # 256 heads x 64 rows x (128 + 2) floats = 8.5 MB for a single split > 8 MiB
    code = f(x.data_ptr(), x.data_ptr(), x.data_ptr(), r.data_ptr(), o.data_ptr(), 1, 256, 256, 4096, 128, 64, None)
    assert code == 2
    code = f(x.data_ptr(), x.data_ptr(), x.data_ptr(), r.data_ptr(), o.data_ptr(), 1, 2, 2, 4096, 96, 64, None)
    assert code == 2
    code = f(0, x.data_ptr(), x.data_ptr(), r.data_ptr(), o.data_ptr(), 1, 2, 2, 4096, 128, 64, None)
    assert code == 1
