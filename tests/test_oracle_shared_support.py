"""Pins of the oracle's shared-route support diagnostic ([support]: a route shared by the
queries of a group must cover the union of their 90%-mass key sets), against closed forms and
an independent brute force on tiny inputs."""
import math

import numpy as np
import pytest

import oracle

GOLDEN = __file__.rsplit("/", 1)[0] + "/golden/splitmix64.txt"


def _brute_set(z, mass=0.9):
    """Independent restatement: walk the keys by descending weight with plain Python, stop at
    the first key where the running mass reaches `mass` of the total, then keep every key whose
    logit is not below that key's logit."""
    w = [math.exp(v - max(z)) for v in z]
    total = sum(w)
    order = sorted(range(len(z)), key=lambda j: -w[j])
    run, last = 0.0, None
    for j in order:
        run += w[j]
        last = j
        if run >= mass * total:
            break
    return {j for j in range(len(z)) if z[j] >= z[last]}


def test_top_mass_set_closed_forms():
    N = 1000
    z = np.full(N, -30.0)
    z[17] = 10.0
    m = oracle.top_mass_set(z)
    assert m.sum() == 1 and m[17]                      # one dominant key holds > 90%
    assert oracle.top_mass_set(np.zeros(N)).all()      # uniform: every key ties with the 900th
    z = np.arange(N, dtype=np.float64) * 1e-3          # distinct logits: exactly the count
    assert oracle.top_mass_set(z).sum() == oracle.top_mass_count(z)
    assert oracle.top_mass_count(np.zeros(N)) == 900


def test_shared_rows_positions():
    assert list(oracle.shared_rows(10, 13)) == [10, 11, 12]            # fewer rows than R: all
    assert list(oracle.shared_rows(0, 8)) == list(range(8))
    pos = oracle.shared_rows(100, 200)
    assert list(pos) == [100 + (2 * m + 1) * 100 // 16 for m in range(8)]
    assert len(set(pos)) == 8 and pos.min() >= 100 and pos.max() < 200


def test_shared_support_brute_force():
    rng = np.random.default_rng(3)
    g, N, d, Gq = 2, 96, 8, 4
    Qg = rng.standard_normal((g, N, d)) * 2.0
    Kh = rng.standard_normal((N, d))
    labels = rng.integers(0, Gq, N)
    labels[:Gq] = np.arange(Gq)
    qperm = np.argsort(labels, kind="stable")
    qoff = np.concatenate([[0], np.cumsum(np.bincount(labels, minlength=Gq))])
    union, single = oracle.shared_support(Qg, Kh, qperm, qoff)
    for a in range(Gq):
        lo, hi = int(qoff[a]), int(qoff[a + 1])
        sets = []
        for m, pos in enumerate(oracle.shared_rows(lo, hi)):
            z = [float(v) for v in (Qg[m % g, qperm[pos]] @ Kh.T) / math.sqrt(d)]
            sets.append(_brute_set(z))
            assert single[a, m] * N == pytest.approx(oracle.top_mass_count(np.array(z)))
        assert union[a] * N == len(set().union(*sets))
        assert max(len(x) for x in sets) <= union[a] * N <= sum(len(x) for x in sets)


def test_shared_support_identical_and_disjoint_rows():
    N, d = 64, 64
    rng = np.random.default_rng(5)
    Kh = rng.standard_normal((N, d)) * 3.0
    q = rng.standard_normal(d)
    Q = np.broadcast_to(q, (1, N, d)).copy()           # every query is the same vector
    qperm = np.arange(N)
    qoff = np.array([0, 16, N])
    union, single = oracle.shared_support(Q, Kh, qperm, qoff)
    own = oracle.top_mass_set(Kh @ q / math.sqrt(d)).sum() / N
    assert np.allclose(union, own) and np.allclose(single[:, :8], single[0, 0])   # union = one row's set
    Kh = np.eye(N, d) * 80.0                           # key j answers only to direction j (logit 10)
    Q = np.zeros((1, N, d))
    Q[0, np.arange(N), np.arange(N) % d] = 1.0         # query i points at key i
    union, single = oracle.shared_support(Q, Kh, qperm, qoff)
    assert union[0] * N == 8 and np.allclose(single[0] * N, 1)   # disjoint one-key sets add up


def test_alternative_probe_samplers():
    """The probe-sampling ablations of [probe]: the uniform grid is the original rows
    floor((m + 1/2) N / M); the random draw follows its stated generator (first draws checked
    against SplitMix64's published outputs from state 0, tests/golden/splitmix64.txt, when the
    seed cancels the salt), gives M
    distinct rows, and both come back in group-major order with their positions in qperm."""
    rng = np.random.default_rng(9)
    N, M = 500, 16
    qperm = rng.permutation(N)
    rows, pos = oracle.probe_rows_uniform(qperm, M)
    assert sorted(rows) == [(2 * m + 1) * N // (2 * M) for m in range(M)]
    assert np.all(np.diff(pos) > 0) and np.array_equal(qperm[pos], rows)
    rows, pos = oracle.probe_rows_random(qperm, M, seed=oracle.PROBE_SEED_SALT)   # state 0
    gold = [int(line.split()[1], 16) for line in open(GOLDEN).read().splitlines() if line.startswith("0x")]
    first = [g % N for g in gold]                                            # published first outputs
    assert set(first) <= set(rows.tolist())
    assert len(set(rows.tolist())) == M and np.all(np.diff(pos) > 0) and np.array_equal(qperm[pos], rows)


def test_semantic_partition_groups_raw_activations():
    """The semantic-partition ablation of [partition]: key groups are the k-means of the raw
    keys (recovered exactly on planted, well separated key clusters, whatever the queries), and
    query groups the k-means of the raw mean query of the KV group."""
    from synthetic import get_workload

    rng = np.random.default_rng(2)
    g, N, d, G = 2, 128, 16, 4
    centers = rng.standard_normal((G, d)) * 20.0
    lab = np.repeat(np.arange(G), N // G)
    Kh = centers[lab] + rng.standard_normal((N, d)) * 0.1
    qc = rng.standard_normal((G, d)) * 20.0
    rows = np.arange(N)
    qlab = (rows // 16 + rows // 64) % G          # another partition; the k-means seed rows fall in distinct clusters
    Qg = np.stack([qc[qlab] + rng.standard_normal((N, d)) * 0.1 for _ in range(g)])
    import types

    base = get_workload("tiny_n1024")
    cfg = types.SimpleNamespace(rK=base.rK, rQ=base.rQ, Gk=G, Gq=G, M=8, r=4, kmeans_iters=10, seed=0,
                                flags=oracle.FLAG_SEMANTIC_PARTITION)
    hp = oracle.partition_head(Qg, Kh, cfg)
    same = lambda a, b: all(len(set(b[a == v])) == 1 for v in np.unique(a)) and len(np.unique(a)) == len(np.unique(b))
    assert same(hp.kgroup, lab) and same(hp.qgroup, qlab)
    assert np.allclose(hp.features, Kh.astype(np.float32))
    assert np.allclose(hp.ycoord, Qg.mean(axis=0).astype(np.float32))


def test_affine_diagnostics_planted():
    """Residual = affine map of the sparse output + a part orthogonal to every affine function of
    it: the fit recovers the map, so the unexplained energy is exactly that part's energy."""
    rng = np.random.default_rng(4)
    n, d = 400, 6
    Os = rng.standard_normal((n, d))
    A = rng.standard_normal((d, d))
    b = rng.standard_normal(d)
    X = np.concatenate([Os, np.ones((n, 1))], axis=1)
    E = rng.standard_normal((n, d))
    Qx, _ = np.linalg.qr(X)
    E -= Qx @ (Qx.T @ E)                                   # orthogonal to the columns of [Os, 1]
    R = Os @ A.T + b + E
    explained, orthogonal = oracle.affine_diagnostics(Os, Os + R)
    sse = (E ** 2).sum()
    assert explained == pytest.approx(1 - sse / ((R - R.mean(axis=0)) ** 2).sum(), rel=1e-9)
    assert orthogonal == pytest.approx(sse / (R ** 2).sum(), rel=1e-9)
    ex0, or0 = oracle.affine_diagnostics(Os, Os + Os @ A.T + b)       # purely affine residual
    assert ex0 == pytest.approx(1.0, abs=1e-12) and or0 == pytest.approx(0.0, abs=1e-12)
