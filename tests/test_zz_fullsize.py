"""Full-size parity on the 720p (N=118800, 24 heads) and GQA world-model (N=75600, 32 query
heads on 8 KV heads) calls, in the launch configuration bench.py times.

The whole call runs on the GPU once through `sparsepr_attention` and once stage by stage (the
same kernels; the outputs must agree bit for bit), and its intermediates are read back. The
oracle then checks, on two KV heads each, what it can afford at this size:
  - response features at sampled keys (brute-force dot products) and key-group means at sampled
    groups (means of the raw keys);
  - the group-major orders and offsets (bit-exact against a stable sort of the GPU's labels);
  - the cell scores (the oracle's formula on the GPU's partition) and the selected cells (the
    oracle's selection rule on the GPU's scores: identical cells);
  - the sparse output O_s and the final corrected output O at sampled query rows and at every
    probe row, with the GPU's partition and route handed to the oracle (its own dense probe
    rows, residuals, ridge fit and subspace): max-abs 2e-2, mean-abs 2e-3;
  - probe rows of O equal the GPU's dense rows (rounded to bf16) exactly.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import free_block_sparse_sparsepr_b200 as spr  # noqa: E402
from synthetic import bf16_bits_to_f64, get_workload, video_qkv  # noqa: E402
from gpu_helpers import MAX_ABS, MEAN_ABS  # noqa: E402

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

ROWS_PER_HEAD = 48


def _sel_from_csr(rowptr, kg, Gq, Gk):
    sel = np.zeros((Gq, Gk), dtype=bool)
    for a in range(Gq):
        sel[a, kg[rowptr[a]:rowptr[a + 1]]] = True
    return sel


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    spr.load_library()


@pytest.mark.parametrize("name", ["hunyuan720p_n118800", "worldmodel_gqa_n75600"])
def test_full_size_sampled(name):
    w = get_workload(name)
    Qb, Kb, Vb = video_qkv(w)
    q, k, v = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda() for x in (Qb, Kb, Vb))
    P, N, d, g = w.B * w.Hkv, w.N, w.d, w.g
    with spr.SparsePR.from_workload(w) as h:
        O_call = h.attention(q, k, v)
        part = h.partition(q, k)
        route = h.route(q, part)
        Qp, Kp, Vp = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        h.permute(q, k, v, part, Qp, Kp, Vp)
        Osp = torch.empty_like(q)
        h.blocksparse_attn(Qp, Kp, Vp, part, route, Osp)
        fit = h.probe_fit(q, k, v, part, Osp)
        O = torch.empty_like(q)
        h.writeback(part, Osp, fit, O)
        torch.cuda.synchronize()
        assert h.device_status() == 0
        assert torch.equal(O_call, O), "staged and fused calls differ"
        pv = {n: t.cpu().numpy() for n, t in h.partition_views(part).items()}
        rv = {n: t.cpu().numpy() for n, t in h.route_views(route).items()}
        fv = {n: t.cpu().numpy() for n, t in h.fit_views(fit).items()}
    O_h = O.float().cpu().numpy()
    Osp_h = Osp.float().cpu().numpy()
    del q, k, v, Qp, Kp, Vp, Osp, O, O_call
    torch.cuda.empty_cache()

    rng = np.random.default_rng(7)
    srows = oracle.sample_rows(N, w.rK)
    for z in sorted({0, P - 1}):
        b, hk = divmod(z, w.Hkv)
        Qg = bf16_bits_to_f64(Qb[b, hk * g:(hk + 1) * g])
        Kh = bf16_bits_to_f64(Kb[b, hk])
        Vh = bf16_bits_to_f64(Vb[b, hk])
        # (1) response features at sampled keys
        keys = rng.choice(N, 64, replace=False)
        Qs = Qg[np.arange(w.rK) % g, srows]
        Fref = (Kh[keys] @ Qs.T) / np.sqrt(d)
        F = pv["features"][z][keys, : w.rK]
        assert np.abs(F - Fref).max() <= 1e-5 * np.abs(Fref).max()
        # (2) group-major orders, offsets and key-group means
        for lab, perm, off, G in ((pv["kgroup"][z], pv["kperm"][z], pv["koff"][z], w.Gk),
                                  (pv["qgroup"][z], pv["qperm"][z], pv["qoff"][z], w.Gq)):
            assert np.array_equal(perm, np.argsort(lab, kind="stable"))
            assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(lab, minlength=G))]))
        kcent = pv["kcent"][z]
        for grp in rng.choice(np.nonzero(np.diff(pv["koff"][z]))[0], 8, replace=False):
            ref = Kh[pv["kgroup"][z] == grp].mean(axis=0)
            assert np.abs(kcent[grp] - ref).max() <= 1e-5 * max(1.0, np.abs(ref).max())
        # (3) cell scores (the oracle's formula on the GPU's partition) and the selection
        ksize, qsize = np.diff(pv["koff"][z]), np.diff(pv["qoff"][z])
        u_heads = [oracle.query_logits(Qg[j], kcent) for j in range(g)]
        S_ref = oracle.cell_scores(u_heads, ksize, pv["qgroup"][z], w.Gq)
        S = rv["scores"][z]
        assert np.abs(S - S_ref).max() <= 2e-3 * np.abs(S_ref).max()
        sel_ref, _, pairs_ref = oracle.select_cells(S, qsize, ksize, N, w.M, w.rho)
        sel = _sel_from_csr(rv["rowptr"][z], rv["kg"][z], w.Gq, w.Gk)
        assert np.array_equal(sel, sel_ref)
        assert int(rv["pairs"][z]) == int(pairs_ref)
        # (4) outputs at sampled rows and the probe rows, GPU partition and route handed in
        inv = np.empty(N, dtype=np.int64)
        inv[pv["qperm"][z]] = np.arange(N)
        hp = oracle.HeadPartition(
            kgroup=pv["kgroup"][z], qgroup=pv["qgroup"][z], kcent=kcent, kperm=pv["kperm"][z],
            koff=pv["koff"][z], qperm=pv["qperm"][z], qoff=pv["qoff"][z], radial=pv["radial"][z],
            probe=pv["probe"][z].astype(np.int64), probe_seq=pv["probe_pos"][z].astype(np.int64),
            weights=pv["weights"][z].astype(np.float64), features=None, z=None, ycoord=None)
        rowptr, kg = oracle.route_csr(sel)
        hr = oracle.HeadRoute(S, sel, None, int(pairs_ref), rowptr, kg, pairs_ref / float(N) ** 2)
        rows = np.union1d(rng.choice(N, ROWS_PER_HEAD, replace=False), hp.probe)
        cfg1 = w.replace(B=1, Hq=g, Hkv=1)
        res = oracle.sparsepr_attention(Qg[None], Kh[None, None], Vh[None, None], cfg1, rows=rows,
                                        partitions={(0, 0): hp}, routes={(0, 0): hr})
        for j in range(g):
            hq = hk * g + j
            x = b * w.Hq + hq
            Os_gpu = Osp_h[b, hq][inv[rows]]
            e = np.abs(Os_gpu - res["O_sparse"][0, j, rows])
            assert e.max() <= MAX_ABS and e.mean() <= MEAN_ABS, (z, j, e.max(), e.mean())
            e = np.abs(O_h[b, hq][rows] - res["O"][0, j, rows])
            assert e.max() <= MAX_ABS and e.mean() <= MEAN_ABS, (z, j, e.max(), e.mean())
            dense_bf16 = torch.from_numpy(fv["Odense"][x]).bfloat16().float().numpy()
            assert np.array_equal(O_h[b, hq][hp.probe], dense_bf16)
