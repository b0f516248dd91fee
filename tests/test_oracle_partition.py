"""Pins of the oracle's partition steps (sampling, responses, k-means, coordinates, order).

Each test checks the oracle against something other than itself: brute force
on tiny inputs, a closed form, an invariant, or a published test vector.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_sample_rows_closed_form():
    for n in (1, 7, 64, 1000, 1024, 118800):
        for s in (1, 3, 16, 48, 64, 256):
            got = oracle.sample_rows(n, s)
            want = [math.floor((Fraction(i) + Fraction(1, 2)) * n / s) for i in range(s)]
            assert got.tolist() == want
            assert got.min() >= 0 and got.max() < n


def test_splitmix64_published_outputs():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "splitmix64.txt")) if not l.startswith("#")]
    assert rows
    for state, out in rows:
        assert oracle.splitmix64(int(state, 16)) == int(out, 16)


def test_rademacher_projection_properties():
    P = oracle.rademacher_projection(256, 64, seed=0)
    assert P.shape == (256, 64)
    assert np.all(np.isclose(np.abs(P), 1 / 8.0))
    frac_neg = (P < 0).mean()
    assert 0.45 < frac_neg < 0.55                       # balanced signs
    G = P.T @ P                                          # near-orthogonal columns (JL)
    assert np.allclose(np.diag(G), 256 / 64.0)
    assert np.abs(G - np.diag(np.diag(G))).max() < 1.2   # |off-diag| ~ 4/8 * sqrt(256)/8 scale
    # deterministic and seed dependent
    assert np.array_equal(P, oracle.rademacher_projection(256, 64, seed=0))
    assert not np.array_equal(P, oracle.rademacher_projection(256, 64, seed=1))
    # entry (g, t) depends on the counter g*rQ + t only
    for g, t in [(0, 0), (3, 5), (255, 63)]:
        bit = oracle.splitmix64(0 ^ (g * 64 + t)) & 1
        assert P[g, t] == (-1 / 8.0 if bit else 1 / 8.0)


def test_response_features_brute_force_gqa():
    rng = np.random.default_rng(1)
    g, N, d, S = 2, 37, 8, 5
    Qg = rng.standard_normal((g, N, d))
    K = rng.standard_normal((N, d))
    z, F = oracle.response_features(Qg, K, S)
    for s in range(S):
        i = math.floor((s + 0.5) * N / S)
        h = s % g
        for j in range(N):
            ref = sum(Qg[h, i, c] * K[j, c] for c in range(d)) / math.sqrt(d)
            assert abs(z[s, j] - ref) < 1e-12
            assert F[j, s] == np.float32(ref)


def test_top_mass_fraction_closed_forms():
    N = 1000
    assert oracle.top_mass_fraction(np.zeros(N)) == 900 / N        # uniform: ceil(0.9 N) keys
    z = np.full(N, -1e9)
    z[17] = 0.0
    assert oracle.top_mass_fraction(z) == 1 / N                      # one-hot
    # two levels: 10 keys of weight e^5, 990 of weight 1
    z = np.zeros(N)
    z[:10] = 5.0
    w_hi, total = 10 * math.exp(5.0), 10 * math.exp(5.0) + 990
    need = 0.9 * total - w_hi                                        # mass still needed from weight-1 keys
    assert oracle.top_mass_fraction(z) == (10 + math.ceil(need)) / N


def test_sq_dists_matches_direct_form():
    rng = np.random.default_rng(2)
    X = rng.standard_normal((50, 48)).astype(np.float32) * 4
    C = rng.standard_normal((9, 48)).astype(np.float32) * 4
    D = oracle.sq_dists_f32(X, C)
    direct = ((X[:, None, :].astype(np.float64) - C[None].astype(np.float64)) ** 2).sum(-1)
    assert np.array_equal(D, direct.astype(np.float32)) or np.abs(D - direct).max() < 1e-4
    assert np.abs(D.astype(np.float64) - direct).max() <= 2 * np.spacing(np.float32(direct.max()))


def test_kmeans_assign_brute_force_and_ties():
    rng = np.random.default_rng(3)
    X = rng.integers(-3, 4, size=(40, 3)).astype(np.float32)
    C = rng.integers(-3, 4, size=(6, 3)).astype(np.float32)
    C[4] = C[1]                                  # duplicate centroid: ties must go to the lower id
    lab, dist = oracle.kmeans_assign(X, C)
    for i in range(len(X)):
        ds = [float(((X[i] - C[g]) ** 2).sum()) for g in range(len(C))]
        best = min(ds)
        assert lab[i] == ds.index(best)
        assert dist[i] == np.float32(best)
    assert not np.any(lab == 4)


def _planted(n_per, G, D, sep, rng):
    centres = rng.standard_normal((G, D)) * sep
    X = np.concatenate([c + rng.standard_normal((n_per, D)) * 0.05 for c in centres])
    truth = np.repeat(np.arange(G), n_per)
    p = rng.permutation(len(X))
    return X[p].astype(np.float32), truth[p]


def test_kmeans_planted_clusters_exact_recovery():
    rng = np.random.default_rng(4)
    for G in (2, 5, 8):
        X, truth = _planted(30, G, 6, sep=10.0, rng=rng)
        # seeds land in distinct clusters only by chance; use a seeding that hits every cluster
        order = np.argsort(truth, kind="stable")
        X, truth = X[order], truth[order]
        lab, C, dist = oracle.kmeans(X, G, iters=10)
        # the partition equals the planted one up to relabelling
        pairs = set(zip(lab.tolist(), truth.tolist()))
        assert len(pairs) == G and len({a for a, _ in pairs}) == G
        # each centroid is its cluster's mean
        for g in range(G):
            assert np.allclose(C[g], X[lab == g].astype(np.float64).mean(0), atol=1e-5)
        assert np.all(dist < 0.2)                      # every row sits in its planted cluster


def test_kmeans_objective_non_increasing():
    rng = np.random.default_rng(5)
    X = rng.standard_normal((300, 4)).astype(np.float32)
    prev = None
    for it in range(0, 8):
        lab, C, dist = oracle.kmeans(X, 7, iters=it)
        obj = float(dist.astype(np.float64).sum())
        if prev is not None:
            assert obj <= prev + 1e-4
        prev = obj


def test_kmeans_empty_group_keeps_centroid_and_labels_consistent():
    X = np.array([[0, 0], [0, 0], [0, 0], [10, 10]], dtype=np.float32)
    lab, C, dist = oracle.kmeans(X, 3, iters=5)
    # seeds are rows 0, 1, 3 -> groups 0 and 1 start identical; ties go to group 0
    assert lab.tolist() == [0, 0, 0, 2]
    assert np.array_equal(C[1], X[1])                      # empty group 1 kept its seed
    lab2, _ = oracle.kmeans_assign(X, C)
    assert np.array_equal(lab, lab2)                       # labels are the assignment of C


def test_group_means_brute_force_and_empty():
    rng = np.random.default_rng(6)
    Y = rng.standard_normal((25, 5))
    lab = rng.integers(0, 4, size=25)
    lab[lab == 2] = 3                                      # group 2 empty
    Cm = oracle.group_means(Y, lab, 5)
    for g in range(5):
        if np.any(lab == g):
            assert np.allclose(Cm[g], Y[lab == g].mean(0), atol=1e-6)
        else:
            assert np.all(Cm[g] == 0)


def test_stable_group_order_is_stable_bijection():
    rng = np.random.default_rng(7)
    lab = rng.integers(0, 9, size=200)
    perm, off = oracle.stable_group_order(lab, 10)
    assert sorted(perm.tolist()) == list(range(200))
    assert off[0] == 0 and off[-1] == 200 and off[-2] == 200     # group 9 empty
    for g in range(10):
        seg = perm[off[g]:off[g + 1]]
        assert np.all(lab[seg] == g)
        assert np.all(np.diff(seg) > 0)                         # original order inside a group
    x = rng.standard_normal((200, 3))
    inv = np.empty_like(perm)
    inv[perm] = np.arange(200)
    assert np.array_equal(x[perm][inv], x)                      # inverse restores input bit-exactly


def test_query_coordinates_properties():
    rng = np.random.default_rng(8)
    g, N, d = 2, 60, 16
    Qg = rng.standard_normal((g, N, d))
    for Gk, rQ in [(5, 64), (80, 8)]:
        kc = rng.standard_normal((Gk, d)).astype(np.float32)
        u, y = oracle.query_coordinates(Qg, kc, rQ, seed=3)
        assert u.shape == (N, Gk) and y.shape == (N, min(Gk, rQ))
        assert np.allclose(np.linalg.norm(y.astype(np.float64), axis=1), 1.0, atol=1e-6)
        # brute force of u on the mean query
        for i in (0, 17, 59):
            for c in (0, Gk - 1):
                ref = sum(0.5 * (Qg[0, i, t] + Qg[1, i, t]) * float(kc[c, t]) for t in range(d)) / 4.0
                assert abs(float(u[i, c]) - ref) < 1e-5 * max(1.0, abs(ref))
        if Gk <= rQ:
            uc = u.astype(np.float64) - u.astype(np.float64).mean(1, keepdims=True)
            ref = uc / np.linalg.norm(uc, axis=1, keepdims=True)
            assert np.allclose(y, ref, atol=1e-6)
        else:
            P = oracle.rademacher_projection(Gk, rQ, 3)
            uc = u.astype(np.float64) - u.astype(np.float64).mean(1, keepdims=True)
            ref = uc @ P
            ref /= np.linalg.norm(ref, axis=1, keepdims=True)
            assert np.allclose(y, ref, atol=1e-6)
    # centring: moving every centroid by the same vector v shifts all of a query's
    # logits by q.v/sqrt(d), which the centring removes
    kc = rng.standard_normal((5, d)).astype(np.float32)
    _, y1 = oracle.query_coordinates(Qg, kc, 64, 0)
    kc2 = (kc + rng.standard_normal(d).astype(np.float32)).astype(np.float32)
    _, y2 = oracle.query_coordinates(Qg, kc2, 64, 0)
    assert np.abs(y1 - y2).max() < 1e-4


def test_partition_head_tiny_end_to_end():
    rng = np.random.default_rng(9)

    class Cfg:
        rK, Gk, Gq, rQ, M, r, lam, rho, kmeans_iters, seed, flags = 8, 4, 4, 64, 8, 2, 0.1, 0.5, 10, 0, 0

    Qg = rng.standard_normal((1, 64, 8))
    K = rng.standard_normal((64, 8))
    p = oracle.partition_head(Qg, K, Cfg)
    assert sorted(p.kperm.tolist()) == list(range(64)) and sorted(p.qperm.tolist()) == list(range(64))
    assert p.koff[-1] == 64 and p.qoff[-1] == 64
    assert len(set(p.probe.tolist())) == 8
    assert abs(p.weights.sum() - 8) < 1e-12
    # key centroids are means of the raw keys of each group
    for gk in range(4):
        if np.any(p.kgroup == gk):
            assert np.allclose(p.kcent[gk], K[p.kgroup == gk].mean(0), atol=1e-6)
