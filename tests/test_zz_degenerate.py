"""Parity on the degenerate inputs the method has.

  - a target density below the probes' share (rho < M/N): the route budget rho N^2 - M N is
    negative, so every query group keeps only its mandatory top cell ([execution]: rho_exec =
    route density + M/N; every query group keeps at least one cell);
  - identical keys: every distance of the key k-means ties, all keys fall in group 0 (ties go to
    the lowest group), the other key groups are empty, the softmax over the keys is uniform, the
    sparse output equals the dense one and the probe residuals are zero (an empty residual
    subspace, a zero correction);
  - identical queries: every query falls in query group 0, the other query groups are empty, and
    the probe rows come from one group in index order (equal radial keys);
  - extreme sizes and group counts: a length below one row tile (N = 100, GQA), a single cell
    (Gk = Gq = 1: the route keeps everything, the query coordinates are all zero), as many key
    groups as keys (N = Gk = 256: groups of one key), every row a probe (M = N = 64: the output is
    the dense attention), no Lloyd round after the seeding assignment (the centroids are the seed
    rows), and an odd GQA group (three query heads on one KV head);
  - the other shapes the configuration allows: d = 64 under GQA with an even group (two query heads
    per attention CTA), the smallest ranks (rK = rQ = 8 with Gk > rQ, r = 1) and the largest
    (rK = rQ = 64, M = 64, r = 32).

Each runs the whole call on the GPU (fused and stage by stage, bit-identical) and checks it against
the oracle with the GPU's partition and route handed in (sampled rows and every probe row, max-abs
2e-2, mean-abs 2e-3), the cell scores and the selection (identical cells), and the group-major
orders; the labels are also checked against the tie rule directly.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import free_block_sparse_sparsepr_b200 as spr  # noqa: E402
from synthetic import Workload, video_qkv  # noqa: E402
from gpu_helpers import sampled_call_parity  # noqa: E402

pytestmark = pytest.mark.gpu

# d = 128 (tensor-core path), GQA with two query heads per KV head, Gk > rQ (projected coordinates)
W = Workload("degenerate_n4096", B=1, Hq=4, Hkv=2, T=4, Hg=32, Wg=32, d=128, Gk=96, Gq=80, block=128,
             rho=0.22, locality=1.0)


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    spr.load_library()


def _labels(w, Qb, Kb):
    q, k = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda() for x in (Qb, Kb))
    with spr.SparsePR.from_workload(w) as h:
        pv = {n: t.cpu().numpy() for n, t in h.partition_views(h.partition(q, k)).items()}
        assert h.device_status() == 0
    return pv


def test_density_below_the_probe_share():
    w = W.replace(rho=0.01)                               # M / N = 64 / 4096 = 1.56%
    assert oracle.budget_pairs(w.rho, w.N, w.M) < 0
    rv = sampled_call_parity(w, *video_qkv(w), kv_heads=[0, 1])
    for z in range(w.B * w.Hkv):
        cells = np.diff(rv["rowptr"][z])
        assert cells.max() <= 1                           # the mandatory cell only
    pv = _labels(w, *video_qkv(w)[:2])
    for z in range(w.B * w.Hkv):
        assert np.array_equal(np.diff(rv["rowptr"][z]), (np.diff(pv["qoff"][z]) > 0).astype(np.int32))


def test_identical_keys():
    Qb, Kb, Vb = video_qkv(W)
    Kb = np.ascontiguousarray(np.broadcast_to(Kb[:, :, :1, :], Kb.shape))
    sampled_call_parity(W, Qb, Kb, Vb, kv_heads=[0, 1])
    pv = _labels(W, Qb, Kb)
    for z in range(W.B * W.Hkv):
        assert np.all(pv["kgroup"][z] == 0)               # every distance ties: the lowest group
        assert pv["koff"][z][1] == W.N


def test_identical_queries():
    Qb, Kb, Vb = video_qkv(W)
    Qb = np.ascontiguousarray(np.broadcast_to(Qb[:, :, :1, :], Qb.shape))
    sampled_call_parity(W, Qb, Kb, Vb, kv_heads=[0, 1])
    pv = _labels(W, Qb, Kb)
    for z in range(W.B * W.Hkv):
        assert np.all(pv["qgroup"][z] == 0)
        probe = np.sort(pv["probe"][z])
        assert np.array_equal(probe, oracle.sample_rows(W.N, W.M))   # one group, index order


SMALL = [
    Workload("n100_gqa", B=1, Hq=2, Hkv=1, T=1, Hg=10, Wg=10, d=128, Gk=8, Gq=6, block=64, rho=0.4, M=16, r=4),
    Workload("single_cell_n512", B=1, Hq=2, Hkv=2, T=2, Hg=16, Wg=16, d=64, Gk=1, Gq=1, block=64, rho=0.22, M=32,
             r=8),
    Workload("one_key_per_group_n256", B=1, Hq=2, Hkv=2, T=1, Hg=16, Wg=16, d=128, Gk=256, Gq=128, block=128,
             rho=0.3, M=32, r=8),
    Workload("every_row_a_probe_n64", B=1, Hq=2, Hkv=2, T=1, Hg=8, Wg=8, d=128, Gk=4, Gq=4, block=64, rho=0.5, M=64,
             r=8),
    Workload("no_lloyd_rounds_n1024", B=1, Hq=2, Hkv=2, T=4, Hg=16, Wg=16, d=128, Gk=16, Gq=16, block=128,
             rho=0.25, kmeans_iters=0),
    Workload("gqa_odd_group_n1024", B=1, Hq=3, Hkv=1, T=4, Hg=16, Wg=16, d=128, Gk=16, Gq=12, block=128, rho=0.3),
    Workload("d64_even_gqa_n2048", B=1, Hq=4, Hkv=2, T=2, Hg=32, Wg=32, d=64, Gk=32, Gq=24, block=64, rho=0.25,
             M=32, r=8),
    Workload("low_ranks_n1024", B=1, Hq=2, Hkv=2, T=4, Hg=16, Wg=16, d=128, Gk=32, Gq=16, block=128, rho=0.25,
             rK=8, rQ=8, M=16, r=1),
    Workload("max_ranks_n2048", B=1, Hq=2, Hkv=2, T=2, Hg=32, Wg=32, d=128, Gk=64, Gq=48, block=128, rho=0.2,
             rK=64, rQ=64, M=64, r=32),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_and_extreme_group_counts(w):
    rv = sampled_call_parity(w, *video_qkv(w))
    if w.Gk == 1 and w.Gq == 1:
        for z in range(w.B * w.Hkv):
            assert int(rv["pairs"][z]) == w.N * w.N          # the one cell holds every pair
