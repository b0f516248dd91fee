"""Pins of the oracle's routing, block-sparse attention, probe fit and whole call.

Each check is against brute force, a closed form, a textbook special case or
an identity stated on the SparsePR page -- never a re-run of the same code.
"""
import itertools
import math
import os

import numpy as np
import pytest

import oracle
from synthetic import bf16_bits_to_f64, get_workload, video_qkv

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- routing

def test_cell_scores_brute_force_and_mass_identity():
    rng = np.random.default_rng(10)
    N, Gk, Gq = 40, 5, 4
    kgroup = rng.integers(0, Gk - 1, size=N)          # key group Gk-1 empty
    ksize = np.bincount(kgroup, minlength=Gk)
    qgroup = rng.integers(0, Gq, size=N)
    us = [rng.standard_normal((N, Gk)).astype(np.float32) for _ in range(2)]
    S = oracle.cell_scores(us, ksize, qgroup, Gq)
    for a in range(Gq):
        members = [i for i in range(N) if qgroup[i] == a]
        for gk in range(Gk):
            acc = 0.0
            for u in us:
                for i in members:
                    den = sum(ksize[t] * math.exp(float(u[i, t])) for t in range(Gk))
                    acc += math.exp(float(u[i, gk])) / den
            ref = acc / (len(us) * len(members)) if (members and ksize[gk]) else 0.0
            assert abs(float(S[a, gk]) - ref) <= 1e-6 * max(ref, 1e-30)
        # a query's weights over all keys sum to 1, so sum_g |K_g| S[a, g] = 1
        if members:
            assert abs(float((ksize * S[a].astype(np.float64)).sum()) - 1.0) < 1e-5


def _route_rule_by_prefixes(S, qsize, ksize, N, M, rho):
    """Independent statement of the rule: among the prefixes of the visiting order
    pick the one whose total is closest to the budget (ties -> the shorter)."""
    Gq, Gk = S.shape
    cost = np.outer(qsize, ksize).astype(np.int64)
    elig = cost > 0
    mand = set()
    for a in range(Gq):
        best = None
        for g in range(Gk):
            if elig[a, g] and (best is None or S[a, g] > S[a, best]):
                best = g
        if best is not None:
            mand.add((a, best))
    rest = [(a, g) for a in range(Gq) for g in range(Gk) if elig[a, g] and (a, g) not in mand]
    rest.sort(key=lambda c: (-float(S[c]), c[0], c[1]))
    base = sum(int(cost[c]) for c in mand)
    budget = math.floor(float(np.float32(rho)) * N * N) - M * N
    best_k, best_gap, tot = 0, abs(base - budget), base
    if base <= budget:
        for k in range(1, len(rest) + 1):
            tot += int(cost[rest[k - 1]])
            if tot - int(cost[rest[k - 1]]) > budget:
                break
            gap = abs(tot - budget)
            if gap < best_gap:
                best_k, best_gap = k, gap
    return mand | set(rest[:best_k])


def test_select_cells_matches_prefix_rule_exhaustive():
    rng = np.random.default_rng(11)
    for trial in range(60):
        Gq, Gk = rng.integers(1, 5), rng.integers(1, 5)
        qsize = rng.integers(0, 6, size=Gq)
        ksize = rng.integers(0, 6, size=Gk)
        N = int(max(qsize.sum(), ksize.sum(), 1))
        S = rng.integers(0, 4, size=(Gq, Gk)).astype(np.float32) / 4    # many ties
        rho = float(rng.choice([0.1, 0.3, 0.5, 0.8, 0.99]))
        M = int(rng.integers(0, 2))
        sel, mand, pairs = oracle.select_cells(S, qsize, ksize, N, M, rho)
        want = _route_rule_by_prefixes(S, qsize, ksize, N, M, rho)
        got = set(zip(*np.nonzero(sel)))
        assert got == want, (trial, got, want)
        assert pairs == sum(int(qsize[a] * ksize[g]) for a, g in got)


def test_select_cells_budget_and_order_invariants():
    rng = np.random.default_rng(12)
    Gq = Gk = 16
    qsize = rng.integers(20, 80, size=Gq)
    ksize = rng.integers(20, 80, size=Gk)
    N = int(qsize.sum())
    ksize = (ksize * N / ksize.sum()).astype(int)
    ksize[-1] += N - ksize.sum()
    S = rng.random((Gq, Gk)).astype(np.float32)
    for rho in (0.15, 0.25, 0.4):
        sel, mand, pairs = oracle.select_cells(S, qsize, ksize, N, 8, rho)
        budget = math.floor(float(np.float32(rho)) * N * N) - 8 * N
        cost = np.outer(qsize, ksize)
        assert abs(pairs - budget) <= cost.max() / 2                    # whole cells: within half a cell
        assert np.all(mand.sum(1) == 1)                                  # one mandatory cell per group
        assert np.all(S[mand] == S.max(1))                               # ... the group's top cell
        free = ~mand
        lo = S[sel & free].min()
        hi = S[~sel & free].max()
        assert lo >= hi                                                  # the kept set is a score prefix
    sel, _, pairs = oracle.select_cells(S, qsize, ksize, N, 8, 1.0)
    assert sel.all() and pairs == N * N


def test_budget_pairs_and_rho_exec_formula_with_page_numbers():
    # probe paragraph: 64 rows are 0.054% of the pairs at the 720p HunyuanVideo length
    rows = [l.split() for l in open(os.path.join(GOLDEN, "page_numbers.txt")) if not l.startswith("#")]
    frac = [r for r in rows if r[0] == "probe_pair_fraction_percent_low"][0]
    M, N = int(frac[2].split("=")[1]), int(frac[3].split("=")[1])
    assert round(100.0 * M / N, 3) == float(frac[1])
    assert oracle.budget_pairs(0.22, N, M) == math.floor(float(np.float32(0.22)) * N * N) - M * N
    # rho_exec = route pairs / N^2 + M / N (execution paragraph)
    b = oracle.budget_pairs(0.22, N, M)
    assert 0 <= float(np.float32(0.22)) - (b / N**2 + M / N) < 1.0 / N**2   # floor of the fp32 target


# ---------------------------------------------------------------- attention

def _naive_attention(Q, K, V, allowed):
    N, d = Q.shape
    O = np.zeros_like(Q)
    for i in range(N):
        z = [sum(Q[i, c] * K[j, c] for c in range(d)) / math.sqrt(d) if allowed(i, j) else None
             for j in range(K.shape[0])]
        m = max(v for v in z if v is not None)
        w = [math.exp(v - m) if v is not None else 0.0 for v in z]
        s = sum(w)
        for c in range(d):
            O[i, c] = sum(w[j] * V[j, c] for j in range(K.shape[0])) / s
    return O


def test_sparse_attention_full_density_is_dense_softmax():
    rng = np.random.default_rng(13)
    N, d = 24, 4
    Q, K, V = (rng.standard_normal((N, d)) for _ in range(3))
    qg = rng.integers(0, 3, size=N)
    kg = rng.integers(0, 4, size=N)
    sel = np.ones((3, 4), dtype=bool)
    O, _ = oracle.sparse_attention(Q, K, V, qg, kg, sel)
    ref = _naive_attention(Q, K, V, lambda i, j: True)
    assert np.abs(O - ref).max() < 1e-12
    Od, _ = oracle.dense_attention_rows(Q, K, V)
    assert np.abs(Od - ref).max() < 1e-12


def test_sparse_attention_brute_force_masking():
    rng = np.random.default_rng(14)
    N, d = 30, 5
    Q, K, V = (rng.standard_normal((N, d)) for _ in range(3))
    qg = rng.integers(0, 3, size=N)
    kg = rng.integers(0, 4, size=N)
    sel = rng.random((3, 4)) < 0.5
    sel[np.arange(3), rng.integers(0, 4, size=3)] = True
    for a in range(3):                          # every group keeps a non-empty key set
        if not np.any(np.isin(kg, np.nonzero(sel[a])[0])):
            sel[a, kg[0]] = True
    O, lse = oracle.sparse_attention(Q, K, V, qg, kg, sel)
    ref = _naive_attention(Q, K, V, lambda i, j: bool(sel[qg[i], kg[j]]))
    assert np.abs(O - ref).max() < 1e-12
    for i in range(N):
        z = [float(Q[i] @ K[j]) / math.sqrt(d) for j in range(N) if sel[qg[i], kg[j]]]
        assert abs(lse[i] - math.log(sum(math.exp(v) for v in z))) < 1e-12


def test_residual_identity_dropped_mass():
    """Residual paragraph: R = O_dense - O_sparse = m (O_drop - O_sparse)."""
    rng = np.random.default_rng(15)
    N, d = 80, 8
    Q, K, V = (rng.standard_normal((N, d)) for _ in range(3))
    qg = rng.integers(0, 4, size=N)
    kg = rng.integers(0, 5, size=N)
    sel = rng.random((4, 5)) < 0.5
    sel[:, 0] = True
    Os, _ = oracle.sparse_attention(Q, K, V, qg, kg, sel)
    Od, _ = oracle.dense_attention_rows(Q, K, V)
    drop = ~sel
    if not drop.any():
        drop[0, 1] = True
        sel[0, 1] = False
    Odrop, _ = oracle.sparse_attention(Q, K, V, qg, kg, drop)
    Z = Q @ K.T / math.sqrt(d)
    P = np.exp(Z - Z.max(1, keepdims=True))
    P /= P.sum(1, keepdims=True)
    m = np.array([P[i, ~sel[qg[i], kg]].sum() for i in range(N)])
    has_drop = m > 0
    lhs = (Od - Os)[has_drop]
    rhs = (m[:, None] * (Odrop - Os))[has_drop]
    assert np.abs(lhs - rhs).max() < 1e-10


# ---------------------------------------------------------------- probes and fit

def test_probe_rows_stratified_radial_brute_force():
    rng = np.random.default_rng(16)
    N, Gq, M = 97, 6, 10
    qgroup = rng.integers(0, Gq, size=N)
    radial = rng.integers(0, 5, size=N).astype(np.float32)      # many ties -> index breaks them
    probe, pos = oracle.probe_rows(qgroup, radial, M)
    seq = sorted(range(N), key=lambda i: (qgroup[i], radial[i], i))
    for m in range(M):
        p = math.floor((m + 0.5) * N / M)
        assert pos[m] == p and probe[m] == seq[p]
    assert len(set(probe.tolist())) == M
    cnt = np.bincount(qgroup, minlength=Gq)
    for a in range(Gq):
        if cnt[a] >= math.ceil(N / M):
            assert np.any(qgroup[probe] == a)                    # big groups are always probed


def test_coverage_weights_brute_force():
    rng = np.random.default_rng(17)
    for _ in range(20):
        Gq, M = int(rng.integers(2, 9)), int(rng.integers(1, 7))
        sizes = rng.integers(0, 9, size=Gq)
        sizes[0] += 1
        N = int(sizes.sum())
        if M > N:
            continue
        qoff = np.concatenate([[0], np.cumsum(sizes)])
        pos = oracle.sample_rows(N, M)
        w = oracle.coverage_weights(pos, qoff, M, N)
        raw = [0.0] * M
        for a in range(Gq):
            lo, hi = qoff[a], qoff[a + 1]
            if hi == lo:
                continue
            mine = [m for m in range(M) if lo <= pos[m] < hi]
            if mine:
                for m in mine:
                    raw[m] += (hi - lo) / len(mine)
            else:
                dist = [min(abs(pos[m] - x) for x in range(lo, hi)) for m in range(M)]
                raw[dist.index(min(dist))] += hi - lo
        assert np.allclose(w, np.array(raw) * M / N)
        assert abs(w.sum() - M) < 1e-9
    # equal groups with one probe each -> all weights 1
    qoff = np.arange(0, 65, 8)
    assert np.allclose(oracle.coverage_weights(oracle.sample_rows(64, 8), qoff, 8, 64), 1.0)


def test_ridge_primal_equals_dual():
    rng = np.random.default_rng(18)
    for M, d in [(64, 128), (64, 16), (10, 3)]:
        X = rng.standard_normal((M, d))
        Y = rng.standard_normal((M, d))
        w = rng.random(M) + 0.2
        A1, xb1, yb1 = oracle.ridge_fit(X, Y, w, 0.1)
        A2, xb2, yb2 = oracle.ridge_fit_dual(X, Y, w, 0.1)
        assert np.abs(A1 - A2).max() <= 1e-8 * max(1.0, np.abs(A1).max())
        assert np.allclose(xb1, xb2) and np.allclose(yb1, yb2)


def test_ridge_recovers_planted_affine_map():
    rng = np.random.default_rng(19)
    M, d = 64, 8                                           # M > d, lambda -> 0: least squares
    Astar = rng.standard_normal((d, 3)) @ rng.standard_normal((3, d))
    b = rng.standard_normal(d)
    X = rng.standard_normal((M, d))
    Y = X @ Astar.T + b
    w = rng.random(M) + 0.5
    A, xbar, ybar = oracle.ridge_fit(X, Y, w, 1e-12)
    assert np.abs(A - Astar).max() < 1e-8
    assert np.abs((ybar - A @ xbar) - b).max() < 1e-8      # recovered intercept
    A0, _, _ = oracle.ridge_fit(X, np.zeros_like(Y), w, 0.1)
    assert np.abs(A0).max() == 0.0


def test_residual_subspace_equals_gram_eigenvectors():
    rng = np.random.default_rng(20)
    M, d, r = 64, 32, 16
    R = rng.standard_normal((M, d)) * np.linspace(3, 0.1, d)
    w = rng.random(M) + 0.5
    U, s = oracle.residual_subspace(R, w, r)
    Gm = (R * w[:, None]).T @ R                            # sum_m w_m R_m R_m^T
    ev, V = np.linalg.eigh(Gm)
    Vr = V[:, ::-1][:, :r]
    assert np.abs(U @ U.T - Vr @ Vr.T).max() < 1e-8        # same projector
    assert np.allclose(np.sort(s ** 2)[::-1][:r], ev[::-1][:r])
    # rank-deficient residuals: the subspace shrinks to the rank
    R3 = rng.standard_normal((M, 3)) @ rng.standard_normal((3, d))
    U3, _ = oracle.residual_subspace(R3, w, r)
    assert U3.shape == (d, 3)
    U0, _ = oracle.residual_subspace(np.zeros((M, d)), w, r)
    assert U0.shape == (d, 0)


def test_correction_variants():
    rng = np.random.default_rng(21)
    d, n = 6, 5
    U, _ = np.linalg.qr(rng.standard_normal((d, 2)))
    A = rng.standard_normal((d, d))
    obar, Rbar = rng.standard_normal(d), rng.standard_normal(d)
    O = rng.standard_normal((n, d))
    full = oracle.correction(O, U, A, obar, Rbar)
    P = U @ U.T
    for i in range(n):
        assert np.allclose(full[i], P @ (Rbar + A @ (O[i] - obar)))
    assert np.allclose(oracle.correction(O, U, A, obar, Rbar, oracle.FLAG_RIDGE_ONLY),
                       Rbar + (O - obar) @ A.T)
    assert np.allclose(oracle.correction(O, U, A, obar, Rbar, oracle.FLAG_RBAR_UNPROJECTED),
                       Rbar + ((O - obar) @ A.T) @ P)
    assert np.allclose(oracle.correction(O, np.eye(d), A, obar, Rbar), Rbar + (O - obar) @ A.T)


# ---------------------------------------------------------------- whole call

def _small(name="tiny_n1024", **kw):
    w = get_workload(name).replace(**kw)
    Q, K, V = (bf16_bits_to_f64(x) for x in video_qkv(w))
    return w, Q, K, V


def test_full_density_call_equals_dense_attention():
    w, Q, K, V = _small(rho=1.0)
    res = oracle.sparsepr_attention(Q, K, V, w)
    D = oracle.dense_attention(Q, K, V)
    assert np.abs(res["O_sparse"] - D).max() < 1e-12
    assert np.abs(res["O"] - D).max() < 1e-12               # R = 0 -> correction 0
    assert abs(res["route_density"] - 1.0) < 1e-15


def test_probe_rows_of_output_are_dense_rows_exactly():
    w, Q, K, V = _small()
    res = oracle.sparsepr_attention(Q, K, V, w)
    for (b, hq), fit in res["fits"].items():
        part = res["partitions"][(b, hq // w.g)]
        Od, _ = oracle.dense_attention_rows(Q[b, hq, part.probe], K[b, hq // w.g], V[b, hq // w.g])
        assert np.array_equal(res["O"][b, hq, part.probe], Od)


def test_realised_density_and_rho_exec():
    w, Q, K, V = _small()
    res = oracle.sparsepr_attention(Q, K, V, w)
    N = w.N
    for (b, h), rt in res["routes"].items():
        part = res["partitions"][(b, h)]
        cmax = np.diff(part.qoff).max() * np.diff(part.koff).max()
        assert abs(rt.pairs - oracle.budget_pairs(w.rho, N, w.M)) <= cmax / 2
        assert rt.pairs == int(np.outer(np.diff(part.qoff), np.diff(part.koff))[rt.sel].sum())
    assert abs(res["rho_exec"] - (res["route_density"] + w.M / N)) < 1e-15


def test_hard_drop_only_flag_keeps_sparse_output():
    w, Q, K, V = _small()

    class Cfg:
        pass

    cfg = Cfg()
    for f in ("rK", "Gk", "Gq", "rQ", "M", "r", "lam", "rho", "kmeans_iters", "seed"):
        setattr(cfg, f, getattr(w, f))
    cfg.flags = oracle.FLAG_HARD_DROP_ONLY
    res = oracle.sparsepr_attention(Q, K, V, cfg)
    assert np.array_equal(res["O"], res["O_sparse"])
    assert res["rho_exec"] == res["route_density"]
    # the whole budget goes to the route
    rt = res["routes"][(0, 0)]
    part = res["partitions"][(0, 0)]
    cmax = np.diff(part.qoff).max() * np.diff(part.koff).max()
    assert abs(rt.pairs - oracle.budget_pairs(w.rho, w.N, 0)) <= cmax / 2


def test_probe_fit_reduces_error_on_tiny_call():
    """Ablation paragraph, qualitatively: the probe fit lowers the error of hard drop."""
    w, Q, K, V = _small()
    res = oracle.sparsepr_attention(Q, K, V, w)
    D = oracle.dense_attention(Q, K, V)
    assert np.abs(res["O"] - D).mean() < np.abs(res["O_sparse"] - D).mean()
