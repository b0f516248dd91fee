"""The allocation-free probe-row attention entry point, through the C ABI.

Some callers cannot allocate device memory: a framework whose memory manager owns every device
allocation, code that runs while an allocator lock is held, a process that reserves its device
memory up front. They call sparsepr_probe_attention_noalloc, which needs no handle and keeps its
scratch in a fixed array compiled into the library. Its output is checked against the oracle's
dense attention of the same rows (max-abs 2e-2, mean-abs 2e-3, the tolerance of the other parity
tests) on two calls in a row (the second call reuses the scratch the first left behind), on
three shapes: d=128 with grouped-query heads, d=64 with fewer than 64 rows, and a length whose
key splits are capped by the number of key tiles and partly empty.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import free_block_sparse_sparsepr_b200 as spr  # noqa: E402
from synthetic import Workload, bf16_bits_to_f64, get_workload, video_qkv  # noqa: E402

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3

CASES = {
    # 4 query heads on 2 KV heads, d=128, M=64: 10 key splits fit the 8 MiB array
    "mid_gqa_d128_m64": get_workload("mid_n16384").replace(Hq=4, Hkv=2),
    # d=64, M=40 < 64, N=1024: 16 key tiles cap the split count
    "tiny_d64_m40": get_workload("tiny_n1024").replace(M=40),
    # N=2080 = 32 x 65: 32 splits of two key tiles each, the last ones empty
    "n2080_empty_splits": Workload("n2080", B=1, Hq=2, Hkv=1, T=2, Hg=20, Wg=52, d=128, Gk=8, Gq=8, block=128,
                                   rho=0.3, M=17, r=8),
}


def _entry():
    lib = spr.load_library()
    f = lib.sparsepr_probe_attention_noalloc
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 6 + [ctypes.c_void_p]
    return f


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    spr.load_library()


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_probe_attention_matches_oracle_on_two_calls(name):
    w = CASES[name]
    Qb, Kb, Vb = video_qkv(w)
    Q, K, V = (bf16_bits_to_f64(x) for x in (Qb, Kb, Vb))
    q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda() for x in (Qb, Kb, Vb))
    rng = np.random.default_rng(11)
    P = w.B * w.Hkv
    rows_h = np.stack([np.sort(rng.choice(w.N, w.M, replace=False)) for _ in range(P)]).astype(np.int32)
    rows = torch.from_numpy(rows_h).cuda()
    ref = np.empty((w.B * w.Hq, w.M, w.d))
    for b in range(w.B):
        for hq in range(w.Hq):
            z = b * w.Hkv + hq // w.g
            ref[b * w.Hq + hq], _ = oracle.dense_attention_rows(Q[b, hq, rows_h[z]], K[b, hq // w.g], V[b, hq // w.g])
    f = _entry()
    stream = torch.cuda.current_stream().cuda_stream
    out = torch.empty((w.B * w.Hq, w.M, w.d), dtype=torch.float32, device="cuda")
    results = []
    for _ in range(2):
        out.fill_(float("nan"))
        code = f(q.data_ptr(), k.data_ptr(), v.data_ptr(), rows.data_ptr(), out.data_ptr(),
                 w.B, w.Hq, w.Hkv, w.N, w.d, w.M, stream)
        assert code == 0, spr.STATUS.get(code, code)
        torch.cuda.synchronize()
        o = out.cpu().numpy().astype(np.float64)
        assert np.isfinite(o).all()
        e = np.abs(o - ref)
        assert e.max() <= MAX_ABS and e.mean() <= MEAN_ABS, (e.max(), e.mean())
        results.append(out.clone())
    assert torch.equal(results[0], results[1])


def test_noalloc_row_outside_range_reads_nothing():
    """A row index outside [0, N) takes a zero query: its output row is the mean of V."""
    w = CASES["n2080_empty_splits"].replace(M=4)
    Qb, Kb, Vb = video_qkv(w)
    V = bf16_bits_to_f64(Vb)
    q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda() for x in (Qb, Kb, Vb))
    rows = torch.tensor([[0, w.N, -1, w.N - 1]], dtype=torch.int32, device="cuda")
    out = torch.empty((w.Hq, 4, w.d), dtype=torch.float32, device="cuda")
    code = _entry()(q.data_ptr(), k.data_ptr(), v.data_ptr(), rows.data_ptr(), out.data_ptr(),
                    w.B, w.Hq, w.Hkv, w.N, w.d, 4, None)
    assert code == 0
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    mean_v = V[0, 0].mean(axis=0)
    for hq in range(w.Hq):
        for m in (1, 2):
            assert np.abs(o[hq, m] - mean_v).max() <= 2e-3


def test_noalloc_rejects_requests_beyond_the_static_maximum():
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
    code = f(x.data_ptr(), x.data_ptr(), x.data_ptr(), r.data_ptr() + 2, o.data_ptr(), 1, 2, 2, 4096, 128, 4, None)
    assert code == 1      # rows pointer not 4-byte aligned
