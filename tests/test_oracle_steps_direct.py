"""Direct pins of oracle steps that the other pins reach only through composite functions:
the centroid update, the query logits, the route CSR, the route of one head at full density and
the probe fit of one head. Each is checked against a plain loop or a closed form."""
import math
import types

import numpy as np

import oracle


def test_kmeans_update_is_the_member_mean():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((50, 5)).astype(np.float32)
    labels = rng.integers(0, 4, 50)
    labels[labels == 2] = 1                                  # group 2 empty: keeps its centroid
    C = rng.standard_normal((4, 5)).astype(np.float32)
    out = oracle.kmeans_update(X, labels, C)
    for g in range(4):
        rows = [X[i].astype(np.float64) for i in range(50) if labels[i] == g]
        want = (sum(rows) / len(rows)).astype(np.float32) if rows else C[g]
        assert np.array_equal(out[g], want)


def test_query_logits_by_loops():
    rng = np.random.default_rng(2)
    Qh = rng.standard_normal((7, 4))
    c = rng.standard_normal((3, 4))
    u = oracle.query_logits(Qh, c)
    for i in range(7):
        for g in range(3):
            ref = sum(Qh[i, t] * c[g, t] for t in range(4)) / 2.0        # sqrt(d) = 2; u is stored fp32
            assert u.dtype == np.float32 and abs(float(u[i, g]) - ref) <= 2.0 ** -24 * abs(ref) + 1e-30


def test_route_csr_round_trip():
    rng = np.random.default_rng(3)
    sel = rng.random((6, 9)) < 0.3
    sel[2] = False                                           # an empty row
    rowptr, kg = oracle.route_csr(sel)
    back = np.zeros_like(sel)
    for a in range(6):
        cols = kg[rowptr[a]:rowptr[a + 1]]
        assert list(cols) == sorted(cols)
        back[a, cols] = True
    assert np.array_equal(back, sel) and rowptr[-1] == sel.sum()


def _tiny_head(rng, g=2, N=96, d=8, Gk=6, Gq=5):
    Qg = rng.standard_normal((g, N, d))
    Kh = rng.standard_normal((N, d))
    Vh = rng.standard_normal((N, d))
    cfg = types.SimpleNamespace(rK=8, rQ=64, Gk=Gk, Gq=Gq, M=12, r=4, lam=0.1, rho=1.0, kmeans_iters=5, seed=0,
                                flags=0)
    return Qg, Kh, Vh, cfg


def test_route_head_at_full_density_keeps_every_nonempty_cell():
    Qg, Kh, Vh, cfg = _tiny_head(np.random.default_rng(4))
    hp = oracle.partition_head(Qg, Kh, cfg)
    hr = oracle.route_head(Qg, hp, cfg)
    qs, ks = np.diff(hp.qoff) > 0, np.diff(hp.koff) > 0
    assert np.array_equal(hr.sel, np.outer(qs, ks))
    assert hr.pairs == int(np.diff(hp.qoff).sum() * np.diff(hp.koff).sum())


def test_fit_head_closed_forms():
    """fit_head: dense probe rows by an explicit softmax loop, R = O_dense - O_sparse, the ridge
    map solving its normal equations, and a subspace spanning the top weighted residual directions."""
    rng = np.random.default_rng(5)
    Qg, Kh, Vh, cfg = _tiny_head(rng)
    hp = oracle.partition_head(Qg, Kh, cfg)
    Qh = Qg[0]
    Os = rng.standard_normal((cfg.M, Kh.shape[1]))
    f = oracle.fit_head(Qh, Kh, Vh, Os, hp, cfg)
    d = Kh.shape[1]
    for m, i in enumerate(hp.probe):
        s = [float(Qh[i] @ Kh[j]) / math.sqrt(d) for j in range(len(Kh))]
        mx = max(s)
        w = [math.exp(v - mx) for v in s]
        row = sum(w[j] * Vh[j] for j in range(len(Kh))) / sum(w)
        assert np.allclose(f.Odense[m], row, atol=1e-12)
    assert np.allclose(f.R, f.Odense - Os)
    w = np.asarray(hp.weights, dtype=np.float64)
    Xc, Yc = Os - f.obar, f.R - f.Rbar
    lhs = f.A @ (Xc.T @ (w[:, None] * Xc) + cfg.lam * np.eye(d))
    assert np.allclose(lhs, Yc.T @ (w[:, None] * Xc), atol=1e-9)
    Wm = np.sqrt(w)[:, None] * f.R                          # rows = columns of the weighted residual matrix
    P = f.U @ f.U.T
    kept = np.linalg.norm(Wm @ P) ** 2
    assert kept >= (np.sort(np.linalg.svd(Wm, compute_uv=False) ** 2)[::-1][: f.U.shape[1]].sum()) * (1 - 1e-9)
