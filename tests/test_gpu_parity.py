"""GPU parity: every step of the CUDA path against the CPU oracle on the same
seeded inputs, through the C ABI. Tolerances: bf16 outputs with fp32
accumulation match within max-abs 2e-2 and mean-abs 2e-3; permutations,
offsets and (where the oracle's partition is handed in) selected cells are
exact; end-to-end partitions agree on >= 99% of rows whose k-means margin
exceeds 1e-3."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
import free_block_sparse_sparsepr_b200 as spr  # noqa: E402
from synthetic import Workload, get_workload, video_qkv  # noqa: E402
from gpu_helpers import (MAX_ABS, MEAN_ABS, assert_close, bf16_to_f64, err, inputs, kmeans_margin,  # noqa: E402
                         partition_tensors, route_tensors, sampled_call_parity, selected_from_csr,
                         to_group_major)

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_n1024": get_workload("tiny_n1024"),
    "mid_n16384_h4": get_workload("mid_n16384").replace(Hq=4, Hkv=4),
    # ragged: N=1000 (not a multiple of any tile), GQA 4 query heads on 2 KV heads, B=2
    "ragged_gqa_n1000": Workload("ragged_gqa_n1000", B=2, Hq=4, Hkv=2, T=5, Hg=10, Wg=20, d=128, Gk=13, Gq=7,
                                 block=64, rho=0.3, M=40, r=8, locality=0.8, noise=0.4),
    # ragged d=64: N=777, more query groups than key groups
    "ragged_d64_n777": Workload("ragged_d64_n777", B=1, Hq=3, Hkv=3, T=3, Hg=7, Wg=37, d=64, Gk=20, Gq=24,
                                block=64, rho=0.35, M=32, r=12),
    # ragged N=1500 with Gk=40 (a ragged column chunk) and GQA, d=128: the logits kernel's tiled
    # stores must clip each head's last row tile at N and its last column chunk at Gk
    "ragged_gqa_n1500_g40": Workload("ragged_gqa_n1500_g40", B=1, Hq=4, Hkv=2, T=5, Hg=15, Wg=20, d=128, Gk=40,
                                     Gq=24, block=128, rho=0.3, M=48, r=16, locality=1.0, noise=0.3),
    # Gk > rQ: the query coordinates go through the +-1 projection
    "proj_n4096": Workload("proj_n4096", B=1, Hq=2, Hkv=2, T=4, Hg=32, Wg=32, d=128, Gk=96, Gq=80, block=128,
                           rho=0.25, locality=1.2),
}

_cache = {}


def _setup(name):
    if name not in _cache:
        w = CASES[name]
        host, dev = inputs(w)
        res = oracle.sparsepr_attention(*host, w)
        _cache[name] = (w, host, dev, res)
    return _cache[name]


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    spr.load_library()
    yield
    _cache.clear()


@pytest.mark.parametrize("name", list(CASES))
def test_dense_attention_matches_oracle(name):
    w, (Q, K, V), (q, k, v), _ = _setup(name)
    with spr.SparsePR.from_workload(w) as h:
        O = h.dense_attn(q, k, v)
        torch.cuda.synchronize()
        rows = np.arange(w.N) if w.N <= 4096 else np.unique(oracle.sample_rows(w.N, 512))
        ref = oracle.dense_attention(Q, K, V, rows=rows)
        assert_close(bf16_to_f64(O)[:, :, rows], ref, "dense attention")


@pytest.mark.parametrize("name", list(CASES))
def test_handed_in_partition_and_route(name):
    """Steps 4-7 with the oracle's partition and route handed in."""
    w, (Q, K, V), (q, k, v), res = _setup(name)
    pt = partition_tensors(res, w)
    rt = route_tensors(res, w)
    part = spr.partition_from_tensors(pt)
    route = spr.route_from_tensors(rt)
    with spr.SparsePR.from_workload(w) as h:
        Qp, Kp, Vp = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        h.permute(q, k, v, part, Qp, Kp, Vp)
        # (4) permutation: bit-exact gathers
        kperm = pt["kperm"].long()
        qperm = pt["qperm"].long()
        for b in range(w.B):
            for hq in range(w.Hq):
                z = b * w.Hkv + hq // w.g
                assert torch.equal(Qp[b, hq], q[b, hq][qperm[z]])
            for hk in range(w.Hkv):
                z = b * w.Hkv + hk
                assert torch.equal(Kp[b, hk], k[b, hk][kperm[z]])
                assert torch.equal(Vp[b, hk], v[b, hk][kperm[z]])
        # (5) block-sparse attention, group-major order
        Osp = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
        h.blocksparse_attn(Qp, Kp, Vp, part, route, Osp, lse)
        torch.cuda.synchronize()
        ref_s = to_group_major(res["O_sparse"], res, w)
        assert_close(bf16_to_f64(Osp), ref_s, "sparse output")
        ref_lse = to_group_major(res["lse"][..., None], res, w)[..., 0]
        assert np.abs(lse.cpu().numpy() - ref_lse).max() < 1e-3
        # (6) probes, residuals, fit
        fit = h.probe_fit(q, k, v, part, Osp)
        torch.cuda.synchronize()
        fv = h.fit_views(fit)
        R = fv["R"].cpu().numpy().reshape(w.B, w.Hq, w.M, w.d)
        Od = fv["Odense"].cpu().numpy().reshape(w.B, w.Hq, w.M, w.d)
        for b in range(w.B):
            for hq in range(w.Hq):
                f = res["fits"][(b, hq)]
                assert_close(Od[b, hq], f.Odense, "probe dense rows", max_abs=2e-3, mean_abs=2e-4)
                assert_close(R[b, hq], f.R, "probe residual")
                x = b * w.Hq + hq
                assert_close(fv["obar"][x].cpu().numpy(), f.obar, "obar", 1e-2, 1e-3)
                assert_close(fv["Rbar"][x].cpu().numpy(), f.Rbar, "Rbar", 1e-2, 1e-3)
                s = f.sing
                rk = int(fv["rank"][x])
                assert rk == min(w.r, f.U.shape[1]) or rk == w.r
                if len(s) > w.r and s[w.r - 1] > 1.2 * s[w.r]:       # projector well defined
                    Ug = fv["U"][x].cpu().numpy().astype(np.float64)
                    assert np.abs(Ug @ Ug.T - f.U @ f.U.T).max() < 5e-2
                # the fit on the GPU's own probe rows, against the oracle's closed forms in fp64:
                # the ridge map A, Bm = U^T A with the GPU's U, and the residual subspace
                Xg = fv["Osp"][x].cpu().numpy().astype(np.float64)
                Rg = fv["R"][x].cpu().numpy().astype(np.float64)
                wz = pt["weights"][b * w.Hkv + hq // w.g].cpu().numpy().astype(np.float64)
                A_ref, xb_ref, yb_ref = oracle.ridge_fit(Xg, Rg, wz, w.lam)
                scale = max(1e-3, np.abs(A_ref).max())
                assert np.abs(fv["A"][x].cpu().numpy() - A_ref).max() <= 2e-3 * scale, "ridge map"
                assert np.abs(fv["obar"][x].cpu().numpy() - xb_ref).max() <= 1e-5 * max(1.0, np.abs(xb_ref).max())
                Ug = fv["U"][x].cpu().numpy().astype(np.float64)
                Bm_ref = Ug.T @ A_ref
                assert np.abs(fv["Bm"][x].cpu().numpy() - Bm_ref).max() <= 2e-3 * scale, "Bm"
                U_ref, s_ref = oracle.residual_subspace(Rg, wz, w.r)
                if len(s_ref) > w.r and s_ref[w.r - 1] > 1.2 * s_ref[w.r]:
                    assert np.abs(Ug @ Ug.T - U_ref @ U_ref.T).max() < 1e-3, "residual subspace"
        # (7) correction and write-back
        O = torch.empty_like(q)
        h.writeback(part, Osp, fit, O)
        torch.cuda.synchronize()
        assert_close(bf16_to_f64(O), res["O"], "corrected output")
        Of = bf16_to_f64(O)
        for b in range(w.B):
            for hq in range(w.Hq):
                p = res["partitions"][(b, hq // w.g)].probe
                assert_close(Of[b, hq, p], res["fits"][(b, hq)].Odense, "probe rows = dense rows", 8e-3, 2e-3)
        assert h.device_status() == 0


@pytest.mark.parametrize("name", list(CASES))
def test_route_with_oracle_partition(name):
    w, (Q, K, V), (q, k, v), res = _setup(name)
    part = spr.partition_from_tensors(partition_tensors(res, w))
    with spr.SparsePR.from_workload(w) as h:
        route = h.route(q, part)
        torch.cuda.synchronize()
        rv = h.route_views(route)
        for b in range(w.B):
            for hk in range(w.Hkv):
                z = b * w.Hkv + hk
                ro = res["routes"][(b, hk)]
                S = rv["scores"][z].cpu().numpy()
                nz = ro.scores > 0
                rel = np.abs(S.astype(np.float64) - ro.scores) / np.maximum(ro.scores, 1e-30)
                assert rel[nz].max() < 2e-4, f"scores rel err {rel[nz].max()}"
                assert np.all(S[~nz] == 0)
                sel = selected_from_csr(rv["rowptr"][z].cpu().numpy(), rv["kg"][z].cpu().numpy(), w.Gq, w.Gk)
                # the selection rule ([execution]: whole cells to the budget) re-run by the oracle on
                # the GPU's own scores must pick exactly the GPU's cells and pair count
                po = res["partitions"][(b, hk)]
                sel_ref, _, pairs_ref = oracle.select_cells(S, np.diff(po.qoff), np.diff(po.koff), w.N, w.M,
                                                            w.rho)
                assert np.array_equal(sel, sel_ref), "selected cells differ from the oracle's rule"
                assert int(rv["pairs"][z]) == int(pairs_ref)
                # and where the oracle's own fp64 ranking has no near-tie at the budget cut (no two
                # free cells within 2e-4 relative of the cut score on either side of it), the GPU's
                # cells are the oracle's own cells exactly
                free = ~ro.mandatory & (np.outer(np.diff(po.qoff), np.diff(po.koff)) > 0)
                if (ro.sel & free).any() and (~ro.sel & free).any():
                    cut_in = ro.scores[ro.sel & free].min()
                    cut_out = ro.scores[~ro.sel & free].max()
                    near = np.abs(ro.scores[free] - cut_in) <= 2e-4 * cut_in
                    if near.sum() <= 1 and cut_in - cut_out > 2e-4 * cut_in:
                        assert np.array_equal(sel, ro.sel), "selected cells differ from the oracle's"
                        assert int(rv["pairs"][z]) == ro.pairs
                # CSR rows ascending
                rp = rv["rowptr"][z].cpu().numpy()
                kgz = rv["kg"][z].cpu().numpy()
                for a in range(w.Gq):
                    assert np.all(np.diff(kgz[rp[a]:rp[a + 1]]) > 0)


@pytest.mark.parametrize("name", list(CASES))
def test_partition_end_to_end(name):
    w, (Q, K, V), (q, k, v), res = _setup(name)
    with spr.SparsePR.from_workload(w) as h:
        part = h.partition(q, k)
        torch.cuda.synchronize()
        pv = {n: t.cpu().numpy() for n, t in h.partition_views(part).items()}
    for b in range(w.B):
        for hk in range(w.Hkv):
            z = b * w.Hkv + hk
            po = res["partitions"][(b, hk)]
            # (1) response features, fp32
            F = pv["features"][z][:, : w.rK]
            scale = np.abs(po.features).max()
            assert np.abs(F - po.features).max() <= 1e-5 * scale
            # (2a) key groups: agreement where the oracle's margin is clear
            _, Ck, _ = oracle.kmeans(po.features, w.Gk, w.kmeans_iters)
            mk = kmeans_margin(po.features, Ck) > 1e-3
            agree_k = (pv["kgroup"][z] == po.kgroup)[mk].mean()
            assert agree_k >= 0.99, f"key-group agreement {agree_k:.4f}"
            # (2b) query groups
            _, Cq, _ = oracle.kmeans(po.ycoord, w.Gq, w.kmeans_iters)
            mq = kmeans_margin(po.ycoord, Cq) > 1e-3
            agree_q = (pv["qgroup"][z] == po.qgroup)[mq].mean()
            assert agree_q >= 0.99, f"query-group agreement {agree_q:.4f}"
            # (4) group-major orders: the stable sort of the GPU's own labels, bit-exact
            for lab, perm, off, G in ((pv["kgroup"][z], pv["kperm"][z], pv["koff"][z], w.Gk),
                                      (pv["qgroup"][z], pv["qperm"][z], pv["qoff"][z], w.Gq)):
                assert np.array_equal(perm, np.argsort(lab, kind="stable"))
                assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(lab, minlength=G))]))
            if np.array_equal(pv["kgroup"][z], po.kgroup):
                assert np.array_equal(pv["kperm"][z], po.kperm)
                assert np.abs(pv["kcent"][z] - po.kcent).max() < 1e-5
            if np.array_equal(pv["qgroup"][z], po.qgroup):
                assert np.array_equal(pv["qperm"][z], po.qperm)
                # probe rows follow from the radial order; equal up to radial near-ties
                same = (pv["probe"][z] == po.probe).mean()
                assert same >= 0.9, f"probe rows agree on {same:.2f}"
            # probe rows: distinct, M of them, systematic positions of the radial sequence
            pr = pv["probe"][z]
            assert len(np.unique(pr)) == w.M
            assert abs(pv["weights"][z].sum() - w.M) < 1e-3


@pytest.mark.parametrize("name", list(CASES))
def test_attention_end_to_end(name):
    w, (Q, K, V), (q, k, v), res = _setup(name)
    with spr.SparsePR.from_workload(w, flags=spr.FLAG_STAGE_TIMING) as h:
        O = h.attention(q, k, v)
        st = h.stats()
        O2 = h.attention(q, k, v)
        torch.cuda.synchronize()
        assert torch.equal(O, O2), "two calls on the same input differ"
        assert st["device_status"] == 0
        assert h.last_launch_count() > 10
        Of = bf16_to_f64(O)
        # realised density follows the rho_exec formula; whole cells keep it near the target
        assert abs(st["rho_exec"] - (st["route_density"] + w.M / w.N)) < 1e-12
        assert abs(st["rho_exec"] - res["rho_exec"]) < 0.02
        assert st["stage_ms"]["total"] > 0
        # probe rows of the output are the exact dense rows
        probes = h.partition_views(h.partition(q, k))["probe"].cpu().numpy()
        torch.cuda.synchronize()
        for b in range(w.B):
            for hq in range(w.Hq):
                p = probes[b * w.Hkv + hq // w.g]
                ref, _ = oracle.dense_attention_rows(Q[b, hq, p], K[b, hq // w.g], V[b, hq // w.g])
                assert_close(Of[b, hq, p], ref, "probe rows = dense rows", 8e-3, 2e-3)
        # quality relative to dense attention is the oracle's, within rounding
        D = oracle.dense_attention(Q, K, V) if w.N <= 4096 else None
        if D is not None:
            e_gpu = np.abs(Of - D).mean()
            e_orc = np.abs(res["O"] - D).mean()
            assert e_gpu <= 1.1 * e_orc + 1e-3, (e_gpu, e_orc)
        mx, mn = err(Of, res["O"])
        assert mn <= 5 * MEAN_ABS, f"end-to-end mean-abs {mn}"


@pytest.mark.parametrize("name", list(CASES))
def test_call_on_its_own_partition_every_row(name):
    """The fused call element by element: the GPU's own partition and route handed to the oracle,
    every row of every query head within max-abs 2e-2 / mean-abs 2e-3 (O_s and O), plus the cell
    scores, the selection rule on the GPU's scores (identical cells) and the probe rows = the
    GPU's dense rows exactly. Complements the end-to-end test above, whose partitions may differ
    from the oracle's at k-means near ties and which therefore compares a mean only."""
    w = CASES[name]
    sampled_call_parity(w, *video_qkv(w), kv_heads=range(w.B * w.Hkv), rows_per_head=w.N)


def test_full_density_equals_dense():
    w = CASES["ragged_gqa_n1000"].replace(rho=1.0)
    (Q, K, V), (q, k, v) = inputs(w)
    with spr.SparsePR.from_workload(w) as h:
        O = h.attention(q, k, v)
        Od = h.dense_attn(q, k, v)
        torch.cuda.synchronize()
        st = h.stats()
    assert abs(st["route_density"] - 1.0) < 1e-12
    D = oracle.dense_attention(Q, K, V)
    assert_close(bf16_to_f64(O), D, "rho=1 output vs dense")
    assert_close(bf16_to_f64(Od), D, "dense kernel")


def test_hard_drop_only_flag():
    w = CASES["tiny_n1024"]
    (Q, K, V), (q, k, v) = inputs(w)

    class Cfg:
        pass

    cfg = Cfg()
    for f in ("rK", "Gk", "Gq", "rQ", "M", "r", "lam", "rho", "kmeans_iters", "seed"):
        setattr(cfg, f, getattr(w, f))
    cfg.flags = oracle.FLAG_HARD_DROP_ONLY
    res = oracle.sparsepr_attention(Q, K, V, cfg)
    pt = partition_tensors(res, w.replace(M=0))
    rt = route_tensors(res, w)
    with spr.SparsePR.from_workload(w, flags=spr.FLAG_HARD_DROP_ONLY) as h:
        part, route = spr.partition_from_tensors(pt), spr.route_from_tensors(rt)
        Qp, Kp, Vp, Osp, O = (torch.empty_like(t) for t in (q, k, v, q, q))
        h.permute(q, k, v, part, Qp, Kp, Vp)
        h.blocksparse_attn(Qp, Kp, Vp, part, route, Osp)
        h.writeback(part, Osp, None, O)
        torch.cuda.synchronize()
        assert_close(bf16_to_f64(O), res["O"], "hard-drop output")
        O2 = h.attention(q, k, v)
        torch.cuda.synchronize()
        st = h.stats()
        assert abs(st["rho_exec"] - st["route_density"]) < 1e-12


@pytest.mark.parametrize("name", ["mid_n16384_h4", "ragged_gqa_n1000", "ragged_gqa_n1500_g40"])
def test_support_diagnostic_matches_oracle(name):
    """The 90%-mass support fraction of every sampled row ([support]) against the oracle's
    full-sort definition applied to the same response row (the GPU's fp32 features): the key
    count agrees to 2 keys (fp32 mass sums may move the crossing across near-equal weights);
    against the oracle's own fp64 responses to 1e-3 of N."""
    w, (Q, K, V), (q, k, v), res = _setup(name)
    with spr.SparsePR.from_workload(w, flags=spr.FLAG_TOPMASS) as h:
        part = h.partition(q, k)
        torch.cuda.synchronize()
        pv = {n: t.cpu().numpy() for n, t in h.partition_views(part).items()}
    assert "topmass" in pv
    for z in range(w.B * w.Hkv):
        F = pv["features"][z][:, : w.rK].astype(np.float64)
        k_gpu = np.rint(pv["topmass"][z] * w.N).astype(np.int64)
        k_ref = np.array([round(oracle.top_mass_fraction(F[:, s]) * w.N) for s in range(w.rK)])
        assert np.abs(k_gpu - k_ref).max() <= 2, (k_gpu, k_ref)
        zo = res["partitions"][(z // w.Hkv, z % w.Hkv)].z
        k_o = np.array([round(oracle.top_mass_fraction(zo[s]) * w.N) for s in range(w.rK)])
        assert np.abs(k_gpu - k_o).max() <= max(2, 1e-3 * w.N), (k_gpu, k_o)



@pytest.mark.parametrize("name", ["mid_n16384_h4", "ragged_gqa_n1000", "ragged_gqa_n1500_g40"])
def test_shared_support_matches_oracle(name):
    """The shared-route support diagnostic ([support]) on the GPU's own partition against the
    oracle's definition in fp64: each row's 90%-mass key count within max(2, 1e-3 N) keys (fp32
    logits and mass sums move the crossing across near-equal weights), the union within that
    per row; the result does not depend on how many KV heads share a workspace pass."""
    w, (Q, K, V), (q, k, v), res = _setup(name)
    P, g, R = w.B * w.Hkv, w.g, spr.SHARED_ROWS
    with spr.SparsePR.from_workload(w) as h:
        part = h.partition(q, k)
        rf_all, uf_all = h.shared_support(q, k, part)
        rf_one, uf_one = h.shared_support(q, k, part, max_workspace_bytes=0)   # one KV head per pass
        torch.cuda.synchronize()
        pv = {n: t.cpu().numpy() for n, t in h.partition_views(part).items()}
    rf, uf = rf_all.cpu().numpy(), uf_all.cpu().numpy()
    tol = max(2.0, 1e-3 * w.N)
    assert np.abs(rf_one.cpu().numpy() - rf).max() * w.N <= tol
    assert np.abs(uf_one.cpu().numpy() - uf).max() * w.N <= R * tol
    for z in range(P):
        b, hk = divmod(z, w.Hkv)
        Qg = bf16_to_f64(q[b, hk * g:(hk + 1) * g])
        Kh = bf16_to_f64(k[b, hk])
        u_ref, s_ref = oracle.shared_support(Qg, Kh, pv["qperm"][z], pv["qoff"][z])
        assert np.abs(rf[z] - s_ref).max() * w.N <= tol, (z, np.abs(rf[z] - s_ref).max() * w.N)
        assert np.abs(uf[z] - u_ref).max() * w.N <= R * tol, (z, np.abs(uf[z] - u_ref).max() * w.N)
        sizes = np.diff(pv["qoff"][z])
        assert np.all(rf[z][np.arange(R)[None, :] >= np.minimum(sizes, R)[:, None]] == 0)
        ok = sizes > 0
        assert np.all(uf[z][ok] + 1e-6 >= rf[z][ok].max(axis=1))        # the union covers every row's set


@pytest.mark.parametrize("name", ["mid_n16384_h4", "ragged_gqa_n1000"])
def test_head_shards_reproduce_the_call(name):
    """Head sharding: every step is per KV head, so running the KV heads in shards (each shard
    its own handle, as each rank of a head-sharded group would) reproduces the unsharded call
    bit for bit."""
    from free_block_sparse_sparsepr_b200.sharding import ShardedSparsePR

    w, (Q, K, V), (q, k, v), res = _setup(name)
    kw = dict(Gk=w.Gk, Gq=w.Gq, block=w.block, rK=w.rK, rQ=w.rQ, M=w.M, r=w.r, kmeans_iters=w.kmeans_iters,
              lam=w.lam, rho_exec=w.rho, seed=w.seed)
    with spr.SparsePR.from_workload(w) as h:
        O_full = h.attention(q, k, v).reshape(w.B * w.Hq, w.N, w.d)
    world = min(3, w.B * w.Hkv)
    parts = []
    for rank in range(world):
        with ShardedSparsePR(w.B, w.Hq, w.Hkv, w.N, w.d, world=world, rank=rank, **kw) as sh:
            parts.append(sh.attention(q, k, v).clone())
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts), O_full)


@pytest.mark.parametrize("name", ["mid_n16384_h4", "ragged_gqa_n1000", "proj_n4096"])
def test_host_call_matches_device_call(name):
    """sparsepr_attention_host (host buffers; the KV heads run in chunks whose copies overlap the
    other chunks' compute) returns the device call's output bit for bit, with the same realised
    density and a clean device status."""
    w, (Q, K, V), (q, k, v), res = _setup(name)
    with spr.SparsePR.from_workload(w) as h:
        O_dev = h.attention(q, k, v)
        torch.cuda.synchronize()
        st_dev = h.stats()
        pin = [t.cpu().pin_memory() for t in (q, k, v)]
        Oh = torch.empty_like(pin[0]).pin_memory()
        for _ in range(2):                                     # the second call reuses the chunk handles
            Oh.zero_()
            h.attention_host(*pin, Oh)
            assert torch.equal(Oh, O_dev.cpu())
        st = h.stats()
        assert st["device_status"] == 0 and h.last_launch_count() > 10
        assert st["rho_exec"] == st_dev["rho_exec"]


@pytest.mark.parametrize("name", ["mid_n16384_h4", "ragged_gqa_n1000"])
def test_affine_diagnostics_match_oracle(name):
    """Affine diagnostics of the hard-drop residual: on the GPU's own uncorrected sparse output
    and dense output, the explained fraction and the orthogonal energy equal the oracle's
    least-squares formula (fp64 on both sides); the sparse output handed to it is the group-major
    output returned to the original order, and the dense one the dense kernel's."""
    w, (Q, K, V), (q, k, v), res = _setup(name)
    with spr.SparsePR.from_workload(w) as h:
        out, Os, Od = h.affine_diagnostics(q, k, v)
        part = h.partition(q, k)
        route = h.route(q, part)
        Qp, Kp, Vp, Osp = (torch.empty_like(t) for t in (q, k, v, q))
        h.permute(q, k, v, part, Qp, Kp, Vp)
        h.blocksparse_attn(Qp, Kp, Vp, part, route, Osp)
        torch.cuda.synchronize()
        assert h.device_status() == 0
        qperm = h.partition_views(part)["qperm"].long()
        Od2 = h.dense_attn(q, k, v)
        torch.cuda.synchronize()
    assert torch.equal(Od, Od2)
    for b in range(w.B):
        for hq in range(w.Hq):
            z = b * w.Hkv + hq // w.g
            back = torch.empty_like(Osp[b, hq])
            back[qperm[z]] = Osp[b, hq]
            assert torch.equal(Os[b, hq], back)
    o = out.cpu().numpy()
    Osf, Odf = bf16_to_f64(Os), bf16_to_f64(Od)
    for b in range(w.B):
        for hq in range(w.Hq):
            x = b * w.Hq + hq
            ex, orth = oracle.affine_diagnostics(Osf[b, hq], Odf[b, hq])
            assert abs(o[x, 0] - ex) <= 1e-6 and abs(o[x, 1] - orth) <= 1e-6, (x, o[x], ex, orth)
            assert 0.0 <= o[x, 1] <= 1.0 and o[x, 0] <= 1.0


@pytest.mark.parametrize("name", ["mid_n16384_h4", "ragged_gqa_n1000"])
def test_semantic_partition_ablation(name):
    """The semantic-partition ablation of [partition] (k-means on the raw keys and the raw mean
    query): the GPU's groups agree with the oracle's where the assignment margin is clear, its
    group-major orders are the stable sort of its own labels, and with the oracle's semantic
    partition handed in to both sides the corrected output matches the oracle."""
    import types

    w, (Q, K, V), (q, k, v), res = _setup(name)
    cfg = types.SimpleNamespace(rK=w.rK, Gk=w.Gk, Gq=w.Gq, rQ=w.rQ, M=w.M, r=w.r, lam=w.lam, rho=w.rho,
                                kmeans_iters=w.kmeans_iters, seed=w.seed, flags=oracle.FLAG_SEMANTIC_PARTITION)
    with spr.SparsePR.from_workload(w, flags=spr.FLAG_SEMANTIC_PARTITION) as h:
        part = h.partition(q, k)
        torch.cuda.synchronize()
        assert h.device_status() == 0
        pv = {n: t.cpu().numpy() for n, t in h.partition_views(part).items()}
    parts = {}
    for b in range(w.B):
        for hk in range(w.Hkv):
            z = b * w.Hkv + hk
            Qg = bf16_to_f64(q[b, hk * w.g:(hk + 1) * w.g])
            Kh = bf16_to_f64(k[b, hk])
            po = oracle.partition_head(Qg, Kh, cfg)
            parts[(b, hk)] = po
            assert np.array_equal(pv["features"][z], po.features)          # the raw keys, widened
            _, Ck, _ = oracle.kmeans(po.features, w.Gk, w.kmeans_iters)
            mk = kmeans_margin(po.features, Ck) > 1e-3
            assert (pv["kgroup"][z] == po.kgroup)[mk].mean() >= 0.99
            _, Cq, _ = oracle.kmeans(po.ycoord, w.Gq, w.kmeans_iters)
            mq = kmeans_margin(po.ycoord, Cq) > 1e-3
            assert (pv["qgroup"][z] == po.qgroup)[mq].mean() >= 0.99
            for lab, perm in ((pv["kgroup"][z], pv["kperm"][z]), (pv["qgroup"][z], pv["qperm"][z])):
                assert np.array_equal(perm, np.argsort(lab, kind="stable"))
    routes = {key: oracle.route_head(bf16_to_f64(q[key[0], key[1] * w.g:(key[1] + 1) * w.g]), hp, cfg)
              for key, hp in parts.items()}
    ref = oracle.sparsepr_attention(Q, K, V, cfg, partitions=parts, routes=routes)
    res2 = dict(res, partitions=parts, routes=routes)
    pt, rt = partition_tensors(res2, w), route_tensors(res2, w)
    with spr.SparsePR.from_workload(w, flags=spr.FLAG_SEMANTIC_PARTITION) as h:
        part, route = spr.partition_from_tensors(pt), spr.route_from_tensors(rt)
        Qp, Kp, Vp, Osp, O = (torch.empty_like(t) for t in (q, k, v, q, q))
        h.permute(q, k, v, part, Qp, Kp, Vp)
        h.blocksparse_attn(Qp, Kp, Vp, part, route, Osp)
        fit = h.probe_fit(q, k, v, part, Osp)
        h.writeback(part, Osp, fit, O)
        torch.cuda.synchronize()
        assert h.device_status() == 0
    assert_close(bf16_to_f64(O), ref["O"], "semantic-partition output")


@pytest.mark.parametrize("flag", ["FLAG_PROBES_UNIFORM", "FLAG_PROBES_RANDOM"])
@pytest.mark.parametrize("name", ["mid_n16384_h4", "ragged_gqa_n1000"])
def test_probe_sampling_ablations(name, flag):
    """The probe-sampling ablations of [probe]: the GPU's probe rows, positions and coverage
    weights equal the oracle's sampler applied to the GPU's own query groups (exact rows and
    positions); with the oracle's partition carrying those probes handed in to both sides, the
    corrected output matches the oracle."""
    w, (Q, K, V), (q, k, v), res = _setup(name)
    seed = w.seed
    with spr.SparsePR.from_workload(w, flags=getattr(spr, flag)) as h:
        part = h.partition(q, k)
        torch.cuda.synchronize()
        assert h.device_status() == 0
        pv = {n: t.cpu().numpy() for n, t in h.partition_views(part).items()}

    def sample(qperm):
        if flag == "FLAG_PROBES_UNIFORM":
            return oracle.probe_rows_uniform(qperm, w.M)
        return oracle.probe_rows_random(qperm, w.M, seed)

    for z in range(w.B * w.Hkv):
        rows, pos = sample(pv["qperm"][z])
        assert np.array_equal(pv["probe"][z], rows)
        assert np.array_equal(pv["probe_pos"][z], pos)
        wref = oracle.coverage_weights(pos, pv["qoff"][z], w.M, w.N)
        assert np.abs(pv["weights"][z] - wref).max() < 1e-4 * max(1.0, wref.max())
    # end to end on the oracle's partition with the ablation's probes
    parts = {}
    for key, hp in res["partitions"].items():
        rows, pos = sample(hp.qperm)
        parts[key] = oracle.HeadPartition(hp.kgroup, hp.qgroup, hp.kcent, hp.kperm, hp.koff, hp.qperm, hp.qoff,
                                          hp.radial, rows, pos, oracle.coverage_weights(pos, hp.qoff, w.M, w.N),
                                          hp.features, hp.z, hp.ycoord)

    class Cfg:
        pass

    cfg = Cfg()
    for f in ("rK", "Gk", "Gq", "rQ", "M", "r", "lam", "rho", "kmeans_iters", "seed"):
        setattr(cfg, f, getattr(w, f))
    cfg.flags = getattr(oracle, flag)
    ref = oracle.sparsepr_attention(Q, K, V, cfg, partitions=parts, routes=res["routes"])
    res2 = dict(res, partitions=parts)
    pt, rt = partition_tensors(res2, w), route_tensors(res, w)
    with spr.SparsePR.from_workload(w, flags=getattr(spr, flag)) as h:
        part, route = spr.partition_from_tensors(pt), spr.route_from_tensors(rt)
        Qp, Kp, Vp, Osp, O = (torch.empty_like(t) for t in (q, k, v, q, q))
        h.permute(q, k, v, part, Qp, Kp, Vp)
        h.blocksparse_attn(Qp, Kp, Vp, part, route, Osp)
        fit = h.probe_fit(q, k, v, part, Osp)
        h.writeback(part, Osp, fit, O)
        torch.cuda.synchronize()
        assert h.device_status() == 0
    assert_close(bf16_to_f64(O), ref["O"], f"{flag} output")


@pytest.mark.parametrize("flag", ["FLAG_RIDGE_ONLY", "FLAG_RBAR_UNPROJECTED"])
@pytest.mark.parametrize("name", ["mid_n16384_h4", "ragged_gqa_n1000"])
def test_ablation_corrections(name, flag):
    """The two correction ablations of [probe] (ridge without the subspace projection; the
    residual mean added unprojected) against the oracle, the oracle's partition and route handed
    in to both sides."""
    w, (Q, K, V), (q, k, v), res = _setup(name)

    class Cfg:
        pass

    cfg = Cfg()
    for f in ("rK", "Gk", "Gq", "rQ", "M", "r", "lam", "rho", "kmeans_iters", "seed"):
        setattr(cfg, f, getattr(w, f))
    cfg.flags = getattr(oracle, flag)
    ref = oracle.sparsepr_attention(Q, K, V, cfg, partitions=res["partitions"], routes=res["routes"])
    pt, rt = partition_tensors(res, w), route_tensors(res, w)
    with spr.SparsePR.from_workload(w, flags=getattr(spr, flag)) as h:
        part, route = spr.partition_from_tensors(pt), spr.route_from_tensors(rt)
        Qp, Kp, Vp, Osp, O = (torch.empty_like(t) for t in (q, k, v, q, q))
        h.permute(q, k, v, part, Qp, Kp, Vp)
        h.blocksparse_attn(Qp, Kp, Vp, part, route, Osp)
        fit = h.probe_fit(q, k, v, part, Osp)
        h.writeback(part, Osp, fit, O)
        torch.cuda.synchronize()
        assert h.device_status() == 0
    assert not np.allclose(ref["O"], res["O"])          # the ablation changes the output
    assert_close(bf16_to_f64(O), ref["O"], f"{flag} output")
