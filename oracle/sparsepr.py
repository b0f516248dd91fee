"""SparsePR attention call restated step by step on the CPU -- TEST INFRASTRUCTURE.

Only tests/, __graft_entry__.smoke() and bench.py (cpu_baseline leg and the
reference arm) may use this module. It shares no code with the CUDA library.

Source: the summary page of "Partition the Support, Reconstruct the Residual:
Training-Free Sparse Attention for Video Generation and World Models"
(Taghavi, Langari, Pandey, 2026-08-19). Its paragraphs are cited as
  [support]    single-row vs shared-route support of 90% of the attention mass
  [residual]   after a hard drop and renormalisation the residual is the dropped
               mass times (output on the dropped support - sparse output)
  [partition]  response-coupled partition: sampled queries' pre-softmax
               responses to all keys give key features (rank rK=48); key groups
               by similarity of those response curves, values follow keys;
               key-group centroids in the original space give the query
               coordinates (rank rQ=64); queries with similar response
               direction share a route; one asymmetric pass
  [probe]      probe residual fit: M=64 rows per query head attend to all keys,
               R = O_dense - O_sparse; group-coverage-weighted ridge
               (lambda=0.1) fits R as an affine function of O_sparse; the
               correction is projected onto the r=16 output subspace seen in
               the probe residuals; probes stratified by query group and drawn
               in within-group radial order around the centroid
  [execution]  Q/K/V in group-major order; exact attention on the selected
               cells, renormalised over the kept K/V groups; under GQA the K/V
               partition and the routing are shared by the query heads of a KV
               head; rho_exec = route density + M/Nq with the probe cost taken
               off the route budget first; whole cells are indivisible, so the
               realised density is reported

Where the page leaves a step open, the reading used is marked "Reading:".

Precision. bf16 inputs enter as exact fp64 values and all continuous
arithmetic is fp64. Wherever a floating-point value decides an integer (k-means
argmin, the cell order, the radial order of probes) that value is first rounded
to fp32 -- the precision the CUDA kernels decide in -- and the decision is taken
on the rounded value with the stated tie rule.

Pins. Each function below is checked in the CPU test-suite against something
other than itself (brute force on tiny inputs, a closed form, a textbook
special case, an invariant the page states, or a published test vector).
The end-to-end quality of the corrected output on real video models (the
page's PSNR / VBench / PBench numbers) is parity unpinned: it needs the page's
trained models, which are out of scope.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "FLAG_HARD_DROP_ONLY", "FLAG_RIDGE_ONLY", "FLAG_RBAR_UNPROJECTED", "FLAG_UNIFORM_WEIGHTS",
    "FLAG_PROBES_UNIFORM", "FLAG_PROBES_RANDOM", "FLAG_SEMANTIC_PARTITION", "PROBE_SEED_SALT",
    "affine_diagnostics", "probe_rows_uniform", "probe_rows_random",
    "sample_rows", "splitmix64", "rademacher_projection", "response_features", "top_mass_fraction",
    "top_mass_count", "top_mass_set", "SHARED_ROWS", "shared_rows", "shared_support",
    "sq_dists_f32", "kmeans_assign", "kmeans_update", "kmeans", "group_means",
    "stable_group_order", "query_coordinates", "query_logits", "cell_scores", "select_cells",
    "route_csr", "probe_rows", "coverage_weights", "sparse_attention", "dense_attention_rows",
    "ridge_fit", "ridge_fit_dual", "residual_subspace", "correction", "budget_pairs",
    "HeadPartition", "HeadRoute", "HeadFit", "partition_head", "route_head", "fit_head",
    "sparsepr_attention", "dense_attention",
]

# Ablation switches (the page's ablations compare these variants).
FLAG_HARD_DROP_ONLY = 1 << 0    # no probes, no correction; the whole budget goes to the route
FLAG_RIDGE_ONLY = 1 << 1        # ridge correction without the subspace projection
FLAG_RBAR_UNPROJECTED = 1 << 2  # project only the feature-dependent part A(o - obar)
FLAG_UNIFORM_WEIGHTS = 1 << 3   # all probe weights 1 instead of group-coverage weights
FLAG_PROBES_UNIFORM = 1 << 5    # probes on a uniform grid of the original token order
FLAG_PROBES_RANDOM = 1 << 6     # probes drawn at random (seeded)
FLAG_SEMANTIC_PARTITION = 1 << 7   # ablation: k-means on the raw keys and the raw mean query
PROBE_SEED_SALT = 0x70726F6265  # "probe": separates the probe draws from other uses of the seed

_MASK64 = (1 << 64) - 1


def _to_f32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


# --------------------------------------------------------------------------------------
# Small shared rules
# --------------------------------------------------------------------------------------

def sample_rows(n: int, s: int) -> np.ndarray:
    """Evenly strided indices floor((i + 1/2) * n / s), i = 0..s-1 (exact integer form).

    Reading: the page says a batch of the current call's queries is sampled
    ([partition]) but not which. The same systematic rule also places the
    k-means seeds and the probe positions.
    """
    i = np.arange(s, dtype=np.int64)
    return ((2 * i + 1) * np.int64(n)) // (2 * np.int64(s))


def splitmix64(x: int) -> int:
    """One output of SplitMix64 (Steele, Lea, Flood, OOPSLA 2014) from state x.

    The state is advanced by the odd constant 0x9E3779B97F4A7C15 and mixed by
    two xor-shift / multiply rounds and a final xor-shift (Stafford's mix13).
    """
    z = (x + 0x9E3779B97F4A7C15) & _MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
    return z ^ (z >> 31)


def rademacher_projection(Gk: int, rQ: int, seed: int) -> np.ndarray:
    """Fixed +-1/sqrt(rQ) matrix P[g, t]; the sign is bit 0 of splitmix64(seed ^ (g*rQ + t)).

    Reading: [partition] gives the query coordinates rank rQ=64 while the
    number of key groups may exceed it; coordinates against Gk > rQ centroids
    are reduced to rQ by this random projection (bit 0 set means -1).
    """
    P = np.empty((Gk, rQ), dtype=np.float64)
    inv = 1.0 / math.sqrt(rQ)
    for g in range(Gk):
        for t in range(rQ):
            bit = splitmix64((seed ^ (g * rQ + t)) & _MASK64) & 1
            P[g, t] = -inv if bit else inv
    return P


def budget_pairs(rho: float, N: int, M: int) -> int:
    """Route budget in (query, key) pairs: floor(rho * N^2) - M * N.

    [execution]: rho_exec = route density + M/Nq and the router takes the probe
    cost off first, so the route may use (rho - M/N) * N^2 pairs. rho is taken
    as the fp32 value the caller passes, widened to fp64, times N*N.
    """
    return int(math.floor(float(np.float32(rho)) * float(N * N))) - int(M) * int(N)


# --------------------------------------------------------------------------------------
# Step 1: sampled queries' pre-softmax responses  ([partition], [support])
# --------------------------------------------------------------------------------------

def response_features(Qg: np.ndarray, Kh: np.ndarray, S: int):
    """Pre-softmax responses z[s, j] = q_{i_s} . k_j / sqrt(d) of S sampled queries.

    Qg: [g, N, d] query heads of one KV group (fp64); Kh: [N, d].
    Sample s is row i_s = floor((s + 1/2) N / S) of query head (s mod g)
    (Reading: under GQA the samples cycle over the group's query heads).
    Returns z [S, N] (fp64) and the key features F = z^T rounded to fp32 [N, S]
    (the response curve of each key over the sample).
    """
    g, N, d = Qg.shape
    rows = sample_rows(N, S)
    heads = np.arange(S) % g
    Qs = Qg[heads, rows, :]                      # [S, d]
    z = (Qs @ Kh.T) / math.sqrt(d)               # [S, N]
    return z, _to_f32(z.T)


def top_mass_fraction(z_row: np.ndarray, mass: float = 0.9) -> float:
    """Fraction of keys a single query row needs to hold `mass` of its softmax mass.

    [support]: the number of largest-probability keys whose softmax mass first
    reaches `mass` of the total, divided by the number of keys.
    """
    z = np.asarray(z_row, dtype=np.float64)
    p = np.exp(z - z.max())
    p = np.sort(p)[::-1]
    c = np.cumsum(p)
    k = int(np.searchsorted(c, mass * c[-1], side="left")) + 1
    return min(k, len(p)) / len(p)


def top_mass_count(z_row: np.ndarray, mass: float = 0.9) -> int:
    """The key count behind top_mass_fraction: keys taken in descending probability until their
    softmax mass first reaches `mass` of the total ([support])."""
    z = np.asarray(z_row, dtype=np.float64)
    p = np.exp(z - z.max())
    c = np.cumsum(np.sort(p)[::-1])
    k = int(np.searchsorted(c, mass * c[-1], side="left")) + 1
    return min(k, len(p))


def top_mass_set(z_row: np.ndarray, mass: float = 0.9) -> np.ndarray:
    """Boolean mask of a row's 90%-mass support: the keys whose logit is at least the k-th
    largest, k = top_mass_count (reading: keys tied with the k-th largest logit all count)."""
    z = np.asarray(z_row, dtype=np.float64)
    k = top_mass_count(z, mass)
    tau = np.sort(z)[::-1][k - 1]
    return z >= tau


SHARED_ROWS = 8     # queries that share one route in the shared-support diagnostic


def shared_rows(lo: int, hi: int, R: int = SHARED_ROWS) -> np.ndarray:
    """Group-major positions of the rows of a query group [lo, hi) that stand for it in the
    shared-support diagnostic: min(R, size) systematic positions lo + floor((m + 1/2) size / R')."""
    size = hi - lo
    Rp = min(R, size)
    m = np.arange(Rp, dtype=np.int64)
    return lo + ((2 * m + 1) * size) // (2 * Rp)


def shared_support(Qg: np.ndarray, Kh: np.ndarray, qperm: np.ndarray, qoff: np.ndarray,
                   R: int = SHARED_ROWS, mass: float = 0.9):
    """Shared-route support ([support]): a route serves every query of its group, so it must
    cover the union of their 90%-mass key sets. For each query group a, the rows of shared_rows
    (row m in query head m mod g of the KV group; Qg [g, N, d], Kh [N, d] fp64) each get their
    90%-mass set over all N keys (top_mass_set of q.k / sqrt(d)); returns the union's size / N
    per group [Gq] (0 for an empty group) and each row's own count / N [Gq, R] (0 past R')."""
    g, N, d = Qg.shape
    Gq = len(qoff) - 1
    union = np.zeros(Gq, dtype=np.float64)
    single = np.zeros((Gq, R), dtype=np.float64)
    for a in range(Gq):
        lo, hi = int(qoff[a]), int(qoff[a + 1])
        if hi <= lo:
            continue
        mask = np.zeros(N, dtype=bool)
        for m, pos in enumerate(shared_rows(lo, hi, R)):
            z = (Qg[m % g, int(qperm[pos])] @ Kh.T) / math.sqrt(d)
            mask |= top_mass_set(z, mass)
            single[a, m] = top_mass_count(z, mass) / N
        union[a] = mask.sum() / N
    return union, single


# --------------------------------------------------------------------------------------
# Step 2: k-means (Lloyd) for key groups and query groups  ([partition])
# --------------------------------------------------------------------------------------

def sq_dists_f32(X: np.ndarray, C: np.ndarray) -> np.ndarray:
    """||x - c||^2 for every row pair, in fp64 as ||x||^2 - 2 x.c + ||c||^2, rounded to fp32.

    The fp64 cancellation error (about 1e-15 * ||x||^2) is far below the fp32
    rounding that follows, so the result is the fp32 value of the distance.
    """
    X64 = np.asarray(X, dtype=np.float64)
    C64 = np.asarray(C, dtype=np.float64)
    d = (X64 * X64).sum(1)[:, None] - 2.0 * (X64 @ C64.T) + (C64 * C64).sum(1)[None, :]
    return _to_f32(np.maximum(d, 0.0))


def kmeans_assign(X: np.ndarray, C: np.ndarray):
    """Nearest centroid of each row (Euclidean; ties -> lowest group id) and its distance."""
    D = sq_dists_f32(X, C)
    lab = D.argmin(axis=1)
    return lab.astype(np.int32), D[np.arange(len(lab)), lab]


def kmeans_update(X: np.ndarray, labels: np.ndarray, C: np.ndarray) -> np.ndarray:
    """Centroid = mean of the member rows (fp64, stored fp32); an empty group keeps its centroid."""
    G = C.shape[0]
    X64 = np.asarray(X, dtype=np.float64)
    sums = np.zeros((G, X64.shape[1]), dtype=np.float64)
    np.add.at(sums, labels, X64)
    cnt = np.bincount(labels, minlength=G)
    out = C.astype(np.float32).copy()
    nz = cnt > 0
    out[nz] = _to_f32(sums[nz] / cnt[nz, None])
    return out


def kmeans(X: np.ndarray, G: int, iters: int):
    """Lloyd's algorithm on fp32 rows X [n, D] into G groups.

    Reading (the page gives no k-means details): seeds are rows
    floor((g + 1/2) n / G); after the first assignment at most `iters`
    rounds of (update, re-assign), stopping as soon as no assignment changes.
    Returns labels [n] int32, the centroids that produced them [G, D] fp32,
    and each row's fp32 distance to its centroid (the radial key).
    """
    X = np.asarray(X, dtype=np.float32)
    C = X[sample_rows(X.shape[0], G)].copy()
    labels, dist = kmeans_assign(X, C)
    for _ in range(iters):
        C = kmeans_update(X, labels, C)
        new, dist = kmeans_assign(X, C)
        changed = not np.array_equal(new, labels)
        labels = new
        if not changed:
            break
    return labels, C, dist


def group_means(Y: np.ndarray, labels: np.ndarray, G: int) -> np.ndarray:
    """Mean of the rows of Y in each group (fp64, stored fp32); empty groups get 0.

    [partition]: the key groups' centroids are taken in the original key space.
    Reading: an empty key group has no keys; its centroid is set to 0.
    """
    Y64 = np.asarray(Y, dtype=np.float64)
    sums = np.zeros((G, Y64.shape[1]), dtype=np.float64)
    np.add.at(sums, labels, Y64)
    cnt = np.bincount(labels, minlength=G)
    out = np.zeros((G, Y64.shape[1]), dtype=np.float32)
    nz = cnt > 0
    out[nz] = _to_f32(sums[nz] / cnt[nz, None])
    return out


def stable_group_order(labels: np.ndarray, G: int):
    """Group-major order: stable sort by group id ([execution]).

    Returns perm [n] (position -> original index; inside a group, ascending
    original index) and offsets off [G+1] (group g occupies off[g]:off[g+1]).
    """
    labels = np.asarray(labels)
    perm = np.argsort(labels, kind="stable").astype(np.int32)
    cnt = np.bincount(labels, minlength=G)
    off = np.zeros(G + 1, dtype=np.int64)
    np.cumsum(cnt, out=off[1:])
    return perm, off.astype(np.int32)


# --------------------------------------------------------------------------------------
# Step 2b: query coordinates against the key-group centroids  ([partition])
# --------------------------------------------------------------------------------------

def query_logits(Qh: np.ndarray, kcent: np.ndarray) -> np.ndarray:
    """u[i, g] = q_i . c_g / sqrt(d), rounded to fp32 (Qh [N, d] fp64, kcent [Gk, d] fp32)."""
    d = Qh.shape[1]
    return _to_f32((Qh @ np.asarray(kcent, dtype=np.float64).T) / math.sqrt(d))


def query_coordinates(Qg: np.ndarray, kcent: np.ndarray, rQ: int, seed: int):
    """Query coordinates y_i: the direction of the query's responses to the key groups.

    Reading: u_i = (mean query over the KV group's g heads) . c_g / sqrt(d);
    centre u_i over the key groups; if Gk > rQ reduce to rQ dimensions with
    rademacher_projection; L2-normalise ("response direction"); zero vectors
    stay zero. Returns the logits u [N, Gk] fp32 and y [N, min(Gk, rQ)] fp32.
    """
    qm = Qg.mean(axis=0)
    u = query_logits(qm, kcent)
    u64 = u.astype(np.float64)
    uc = u64 - u64.mean(axis=1, keepdims=True)
    Gk = kcent.shape[0]
    y = uc @ rademacher_projection(Gk, rQ, seed) if Gk > rQ else uc
    nrm = np.sqrt((y * y).sum(axis=1, keepdims=True))
    y = np.where(nrm > 0, y / np.where(nrm > 0, nrm, 1.0), 0.0)
    return u, _to_f32(y)


# --------------------------------------------------------------------------------------
# Step 3: routing to the density budget  ([execution])
# --------------------------------------------------------------------------------------

def cell_scores(u_heads, ksize: np.ndarray, qgroup: np.ndarray, Gq: int) -> np.ndarray:
    """Score of cell (a, g): estimated softmax weight of one key of group g for a query of group a.

    Reading: a query i puts weight exp(u_ig) / sum_g' |K_g'| exp(u_ig') on
    each key of group g (keys replaced by their group centroid); the score
    is that weight averaged over the queries of group a and, under GQA, over
    the query heads of the KV group (u_heads holds one fp32 [N, Gk] logit
    array per head). A greedy order by score maximises estimated mass per
    executed pair. Returned as fp32 [Gq, Gk]; cells of empty groups score 0.
    """
    ksize = np.asarray(ksize, dtype=np.int64)
    Gk = len(ksize)
    nonempty = ksize > 0
    qgroup = np.asarray(qgroup)
    perm, off = stable_group_order(qgroup, Gq)
    acc = np.zeros((Gq, Gk), dtype=np.float64)
    logk = np.where(nonempty, np.log(np.maximum(ksize, 1)), -np.inf)
    for u in u_heads:
        u64 = np.asarray(u, dtype=np.float64)
        a = u64 + logk[None, :]
        m = a.max(axis=1, keepdims=True)
        lse = m[:, 0] + np.log(np.exp(a - m).sum(axis=1))
        p = np.exp(u64 - lse[:, None])[perm]
        for grp in range(Gq):
            lo, hi = off[grp], off[grp + 1]
            if hi > lo:
                acc[grp] += p[lo:hi].sum(axis=0)
    qsize = np.diff(off).astype(np.float64)
    S = acc / (len(u_heads) * np.maximum(qsize, 1.0))[:, None]
    S[:, ~nonempty] = 0.0
    S[qsize == 0] = 0.0
    return _to_f32(S)


def select_cells(S: np.ndarray, qsize: np.ndarray, ksize: np.ndarray, N: int, M: int, rho: float):
    """Choose whole (query-group, key-group) cells to the route budget ([execution]).

    Reading: every non-empty query group first keeps its top-scoring cell
    (ties -> lowest key group). The other cells are visited in descending
    fp32 score (ties -> lower query group, then lower key group) and added
    while the route's pairs stay within budget_pairs(rho, N, M); the first
    cell that would cross is kept only if its overshoot is smaller than the
    undershoot left without it, and the visit stops there. rho >= 1 keeps
    every cell. Returns selected [Gq, Gk] bool, mandatory [Gq, Gk] bool and
    the number of routed pairs.
    """
    S = np.asarray(S, dtype=np.float32)
    qsize = np.asarray(qsize, dtype=np.int64)
    ksize = np.asarray(ksize, dtype=np.int64)
    Gq, Gk = S.shape
    cost = qsize[:, None] * ksize[None, :]
    eligible = cost > 0
    mand = np.zeros((Gq, Gk), dtype=bool)
    if float(np.float32(rho)) >= 1.0:
        return eligible.copy(), mand, int(cost[eligible].sum())
    for a in range(Gq):
        if eligible[a].any():
            mand[a, int(np.where(eligible[a], S[a], -np.inf).argmax())] = True
    sel = mand.copy()
    total = int(cost[sel].sum())
    budget = budget_pairs(rho, N, M)
    ai, gi = np.nonzero(eligible & ~mand)
    order = np.lexsort((gi, ai, -S[ai, gi]))
    for c in order:
        a, g = int(ai[c]), int(gi[c])
        cc = int(cost[a, g])
        if total + cc <= budget:
            sel[a, g] = True
            total += cc
            continue
        over = total + cc - budget
        under = budget - total
        if over < under:
            sel[a, g] = True
            total += cc
        break
    return sel, mand, total


def route_csr(sel: np.ndarray):
    """Selected cells as CSR: rowptr [Gq+1], kept key groups of each query group ascending."""
    rowptr = np.zeros(sel.shape[0] + 1, dtype=np.int32)
    np.cumsum(sel.sum(axis=1), out=rowptr[1:])
    kg = np.nonzero(sel)[1].astype(np.int32)
    return rowptr, kg


# --------------------------------------------------------------------------------------
# Step 5: exact attention on the selected cells  ([execution], [residual])
# --------------------------------------------------------------------------------------

def sparse_attention(Qh, Kh, Vh, qgroup, kgroup, sel, rows=None):
    """Exact softmax attention of each query row over the union of its group's kept key groups.

    The softmax is renormalised over the kept keys only (hard drop +
    renormalise). Qh [N, d], Kh/Vh [N, d] fp64 in original order. Returns
    O [N, d] and lse [N] (natural log of the kept softmax sum of the scaled
    logits), filled for `rows` only when given (other rows are NaN).
    """
    N, d = Qh.shape
    scale = 1.0 / math.sqrt(d)
    O = np.full((N, d), np.nan)
    lse = np.full(N, np.nan)
    want = np.ones(N, dtype=bool) if rows is None else np.isin(np.arange(N), rows)
    for a in range(sel.shape[0]):
        qi = np.nonzero((qgroup == a) & want)[0]
        if qi.size == 0:
            continue
        kj = np.nonzero(np.isin(kgroup, np.nonzero(sel[a])[0]))[0]
        Z = (Qh[qi] @ Kh[kj].T) * scale
        m = Z.max(axis=1, keepdims=True)
        P = np.exp(Z - m)
        l = P.sum(axis=1, keepdims=True)
        O[qi] = (P @ Vh[kj]) / l
        lse[qi] = m[:, 0] + np.log(l[:, 0])
    return O, lse


def dense_attention_rows(Qrows, Kh, Vh):
    """Dense softmax attention (scale 1/sqrt(d)) of the given query rows over all keys."""
    d = Qrows.shape[1]
    Z = (Qrows @ Kh.T) / math.sqrt(d)
    m = Z.max(axis=1, keepdims=True)
    P = np.exp(Z - m)
    l = P.sum(axis=1, keepdims=True)
    return (P @ Vh) / l, m[:, 0] + np.log(l[:, 0])


# --------------------------------------------------------------------------------------
# Step 6: probes, coverage weights, ridge fit, residual subspace  ([probe])
# --------------------------------------------------------------------------------------

def probe_rows(qgroup: np.ndarray, radial: np.ndarray, M: int):
    """M probe rows, stratified by query group and drawn in within-group radial order.

    Reading: order the queries group-major, inside a group by fp32 distance to
    the group centroid (ascending; ties -> lower original index), and take
    the systematic sample of positions floor((m + 1/2) N / M). Every group
    of at least N/M rows gets a probe; smaller groups get one in proportion.
    Returns the probes' original indices [M] and their sequence positions [M].
    """
    N = len(qgroup)
    seq = np.lexsort((np.arange(N), np.asarray(radial, dtype=np.float32), np.asarray(qgroup)))
    pos = sample_rows(N, M)
    return seq[pos].astype(np.int32), pos.astype(np.int32)


def _by_sequence_position(rows: np.ndarray, qperm: np.ndarray):
    """The rows with their group-major positions (index in qperm), in ascending position."""
    inv = np.empty(len(qperm), dtype=np.int64)
    inv[np.asarray(qperm, dtype=np.int64)] = np.arange(len(qperm))
    pos = inv[np.asarray(rows, dtype=np.int64)]
    o = np.argsort(pos, kind="stable")
    return np.asarray(rows)[o].astype(np.int32), pos[o].astype(np.int32)


def probe_rows_uniform(qperm: np.ndarray, M: int):
    """Ablation of [probe] (uniform spatio-temporal sampling): the rows floor((m + 1/2) N / M) of
    the original token order, a uniform grid over (t, h, w) in t-major order, returned in
    group-major order with their sequence positions (for the coverage weights)."""
    return _by_sequence_position(sample_rows(len(qperm), M), qperm)


def probe_rows_random(qperm: np.ndarray, M: int, seed: int):
    """Ablation of [probe] (random sampling): M distinct rows from the SplitMix64 stream of state
    s = seed xor PROBE_SEED_SALT (output i = splitmix64(s + i * 0x9E3779B97F4A7C15)), each output
    taken mod N, an output equal to an earlier one skipped; returned in group-major order with
    their sequence positions."""
    N = len(qperm)
    s = (int(seed) ^ PROBE_SEED_SALT) & _MASK64
    rows, seen, i = [], set(), 0
    while len(rows) < M:
        c = splitmix64((s + i * 0x9E3779B97F4A7C15) & _MASK64) % N
        i += 1
        if c not in seen:
            seen.add(c)
            rows.append(c)
    return _by_sequence_position(np.array(rows, dtype=np.int64), qperm)


def coverage_weights(pos: np.ndarray, qoff: np.ndarray, M: int, N: int) -> np.ndarray:
    """Group-coverage weight of each probe, normalised to mean 1 ([probe]).

    Reading: a query group that holds probes splits its size equally among
    them; a group without a probe adds its size to the probe nearest to the
    group in sequence position (ties -> lower probe index). The weights sum
    to N before the scaling by M / N.
    """
    pos = np.asarray(pos, dtype=np.int64)
    qoff = np.asarray(qoff, dtype=np.int64)
    pg = np.searchsorted(qoff, pos, side="right") - 1     # group that holds each probe
    raw = np.zeros(len(pos), dtype=np.float64)
    for a in range(len(qoff) - 1):
        lo, hi = int(qoff[a]), int(qoff[a + 1])
        size = hi - lo
        if size == 0:
            continue
        mine = np.nonzero(pg == a)[0]
        if mine.size:
            raw[mine] += size / mine.size
        else:
            dist = np.where(pos < lo, lo - pos, np.where(pos >= hi, pos - (hi - 1), 0))
            raw[int(dist.argmin())] += size
    return raw * (M / float(N))


def ridge_fit(X: np.ndarray, Y: np.ndarray, w: np.ndarray, lam: float):
    """Weighted-centred affine ridge fit of Y on X (primal closed form).

    A = argmin_A sum_m w_m ||(Y_m - Ybar) - A (X_m - Xbar)||^2 + lam ||A||_F^2,
    with Xbar, Ybar the w-weighted means (the intercept is not penalised):
    A (Xc^T W Xc + lam I) = Yc^T W Xc. Returns A [d, d], Xbar [d], Ybar [d].
    """
    w = np.asarray(w, dtype=np.float64)
    W = w.sum()
    xbar = (w @ X) / W
    ybar = (w @ Y) / W
    Xc = X - xbar
    Yc = Y - ybar
    d = X.shape[1]
    Gm = Xc.T @ (w[:, None] * Xc) + lam * np.eye(d)
    Cyx = Yc.T @ (w[:, None] * Xc)
    A = np.linalg.solve(Gm, Cyx.T).T
    return A, xbar, ybar


def ridge_fit_dual(X: np.ndarray, Y: np.ndarray, w: np.ndarray, lam: float):
    """The same fit through the M x M (kernel) system:
    A = Yc^T W^1/2 (W^1/2 Xc Xc^T W^1/2 + lam I)^-1 W^1/2 Xc."""
    w = np.asarray(w, dtype=np.float64)
    W = w.sum()
    xbar = (w @ X) / W
    ybar = (w @ Y) / W
    s = np.sqrt(w)[:, None]
    Xs = s * (X - xbar)
    Ys = s * (Y - ybar)
    Kmat = Xs @ Xs.T + lam * np.eye(X.shape[0])
    A = Ys.T @ np.linalg.solve(Kmat, Xs)
    return A, xbar, ybar


def residual_subspace(R: np.ndarray, w: np.ndarray, r: int):
    """Top-r left singular vectors of the d x M matrix [sqrt(w_m) R_m] ([probe]).

    Reading: the "output subspace seen in the probe residuals" is spanned by
    the weighted, uncentred residuals; numerically zero singular values
    (below max(M, d) * eps * sigma_1) are dropped, so the rank may be < r.
    Returns U [d, k] with k = min(r, rank) and all singular values.
    """
    Rw = np.sqrt(np.asarray(w, dtype=np.float64))[:, None] * R
    U, s, _ = np.linalg.svd(Rw.T, full_matrices=False)
    if s.size == 0 or s[0] == 0.0:
        return U[:, :0], s
    rank = int((s > s[0] * max(Rw.shape) * np.finfo(np.float64).eps).sum())
    return U[:, : min(r, rank)], s


def affine_diagnostics(Os: np.ndarray, Od: np.ndarray):
    """How affine the hard-drop residual of one query head is ([partition] diagnostics, judged
    against dense outputs): R = Od - Os over all rows, and the least-squares affine map of the
    sparse output R ~ A Os + b (no penalty). Returns
      explained  = 1 - SSE / sum ||R_i - mean R||^2   (affine-explainable fraction)
      orthogonal = SSE / sum ||R_i||^2                 (affine-orthogonal energy)
    with SSE the residual energy of that fit (reading: the page names both and gives no formula)."""
    Os = np.asarray(Os, dtype=np.float64)
    R = np.asarray(Od, dtype=np.float64) - Os
    X = np.concatenate([Os, np.ones((Os.shape[0], 1))], axis=1)
    beta, *_ = np.linalg.lstsq(X, R, rcond=None)
    sse = float(((R - X @ beta) ** 2).sum())
    centred = float(((R - R.mean(axis=0)) ** 2).sum())
    total = float((R ** 2).sum())
    return 1.0 - sse / centred, sse / total


def correction(Os: np.ndarray, U: np.ndarray, A: np.ndarray, obar: np.ndarray, Rbar: np.ndarray,
               flags: int = 0) -> np.ndarray:
    """Predicted residual of rows Os [n, d] ([probe]).

    Reading: the whole affine prediction Rbar + A (o - obar) is projected onto
    span(U): delta(o) = U U^T (Rbar + A (o - obar)). FLAG_RBAR_UNPROJECTED
    projects only A (o - obar); FLAG_RIDGE_ONLY skips the projection.
    """
    F = (Os - obar) @ A.T
    if flags & FLAG_RIDGE_ONLY:
        return Rbar + F
    P = U @ U.T
    if flags & FLAG_RBAR_UNPROJECTED:
        return Rbar + F @ P
    return (Rbar + F) @ P


# --------------------------------------------------------------------------------------
# One KV head end to end
# --------------------------------------------------------------------------------------

@dataclasses.dataclass
class HeadPartition:
    kgroup: np.ndarray      # [N] int32
    qgroup: np.ndarray      # [N] int32
    kcent: np.ndarray       # [Gk, d] fp32, key-group means in the original space
    kperm: np.ndarray       # [N] int32 position -> original key index (group-major)
    koff: np.ndarray        # [Gk+1] int32
    qperm: np.ndarray       # [N] int32 position -> original query index (group-major)
    qoff: np.ndarray        # [Gq+1] int32
    radial: np.ndarray      # [N] fp32 squared distance of each query to its group centroid
    probe: np.ndarray       # [M] int32 original query index of each probe row
    probe_seq: np.ndarray   # [M] int32 position of each probe in the radial-ordered sequence
    weights: np.ndarray     # [M] fp64 coverage weights (mean 1)
    features: np.ndarray    # [N, rK] fp32 key response features
    z: np.ndarray           # [rK, N] fp64 sampled responses
    ycoord: np.ndarray      # [N, D] fp32 query coordinates


@dataclasses.dataclass
class HeadRoute:
    scores: np.ndarray      # [Gq, Gk] fp32
    sel: np.ndarray         # [Gq, Gk] bool
    mandatory: np.ndarray   # [Gq, Gk] bool
    pairs: int
    rowptr: np.ndarray
    kg: np.ndarray
    density: float          # pairs / N^2


@dataclasses.dataclass
class HeadFit:
    A: np.ndarray
    obar: np.ndarray
    Rbar: np.ndarray
    U: np.ndarray
    sing: np.ndarray
    R: np.ndarray           # [M, d] probe residuals
    Odense: np.ndarray      # [M, d]
    Os_probe: np.ndarray    # [M, d]


def _n_probes(cfg) -> int:
    return 0 if (getattr(cfg, "flags", 0) & FLAG_HARD_DROP_ONLY) else int(cfg.M)


def partition_head(Qg: np.ndarray, Kh: np.ndarray, cfg) -> HeadPartition:
    """Response-coupled partition of one KV head ([partition]) plus its probe rows ([probe]).

    Qg: [g, N, d] fp64 query heads of the KV group; Kh: [N, d] fp64.
    """
    N = Kh.shape[0]
    z, F = response_features(Qg, Kh, cfg.rK)
    if getattr(cfg, "flags", 0) & FLAG_SEMANTIC_PARTITION:
        # ablation ([partition]: grouping by activations instead of responses): k-means on the
        # raw keys, and on the mean query of the KV group, both as fp32 rows
        F = _to_f32(Kh)
        y = _to_f32(Qg.mean(axis=0))
        kgroup, _, _ = kmeans(F, cfg.Gk, cfg.kmeans_iters)
        kcent = group_means(Kh, kgroup, cfg.Gk)
    else:
        kgroup, _, _ = kmeans(F, cfg.Gk, cfg.kmeans_iters)
        kcent = group_means(Kh, kgroup, cfg.Gk)
        _, y = query_coordinates(Qg, kcent, cfg.rQ, getattr(cfg, "seed", 0))
    qgroup, _, radial = kmeans(y, cfg.Gq, cfg.kmeans_iters)
    kperm, koff = stable_group_order(kgroup, cfg.Gk)
    qperm, qoff = stable_group_order(qgroup, cfg.Gq)
    M = _n_probes(cfg)
    flags = getattr(cfg, "flags", 0)
    if M:
        if flags & FLAG_PROBES_UNIFORM:
            probe, pseq = probe_rows_uniform(qperm, M)
        elif flags & FLAG_PROBES_RANDOM:
            probe, pseq = probe_rows_random(qperm, M, getattr(cfg, "seed", 0))
        else:
            probe, pseq = probe_rows(qgroup, radial, M)
        if flags & FLAG_UNIFORM_WEIGHTS:
            w = np.ones(M)
        else:
            w = coverage_weights(pseq, qoff, M, N)
    else:
        probe = np.zeros(0, np.int32)
        pseq = np.zeros(0, np.int32)
        w = np.zeros(0)
    return HeadPartition(kgroup, qgroup, kcent, kperm, koff, qperm, qoff, radial, probe, pseq, w,
                         F, z, y)


def route_head(Qg: np.ndarray, part: HeadPartition, cfg) -> HeadRoute:
    """Cell scores from every query head of the KV group, then selection to the budget."""
    N = Qg.shape[1]
    ksize = np.diff(part.koff)
    qsize = np.diff(part.qoff)
    u_heads = [query_logits(Qg[j], part.kcent) for j in range(Qg.shape[0])]
    S = cell_scores(u_heads, ksize, part.qgroup, len(qsize))
    sel, mand, pairs = select_cells(S, qsize, ksize, N, _n_probes(cfg), cfg.rho)
    rowptr, kg = route_csr(sel)
    return HeadRoute(S, sel, mand, pairs, rowptr, kg, pairs / float(N) ** 2)


def fit_head(Qh, Kh, Vh, Os_probe, part: HeadPartition, cfg) -> HeadFit:
    """Probe residuals of one query head and the projected ridge fit ([probe])."""
    Od, _ = dense_attention_rows(Qh[part.probe], Kh, Vh)
    R = Od - Os_probe
    A, obar, Rbar = ridge_fit(Os_probe, R, part.weights, cfg.lam)
    U, s = residual_subspace(R, part.weights, cfg.r)
    return HeadFit(A, obar, Rbar, U, s, R, Od, Os_probe)


def sparsepr_attention(Q, K, V, cfg, rows=None, partitions=None, routes=None):
    """One SparsePR attention call (all seven steps) on fp64 copies of bf16 inputs.

    Q [B, Hq, N, d], K/V [B, Hkv, N, d] (fp64 arrays of bf16 values). `rows`
    restricts the output to those query rows (the partition, route and probe
    fit still use the whole call). `partitions` / `routes` (dicts keyed by
    (b, kv_head)) replace the computed ones. Returns a dict with O [B, Hq, N, d]
    (NaN outside `rows`), O_sparse, lse, and the per-head partition, route and
    fit objects, the realised route density and rho_exec.
    """
    B, Hq, N, d = Q.shape
    Hkv = K.shape[1]
    g = Hq // Hkv
    flags = getattr(cfg, "flags", 0)
    M = _n_probes(cfg)
    O = np.full(Q.shape, np.nan)
    Os = np.full(Q.shape, np.nan)
    LSE = np.full(Q.shape[:3], np.nan)
    parts, rts, fits = {}, {}, {}
    dens = []
    for b in range(B):
        for h in range(Hkv):
            Qg = Q[b, h * g:(h + 1) * g]
            part = partitions[(b, h)] if partitions else partition_head(Qg, K[b, h], cfg)
            rt = routes[(b, h)] if routes else route_head(Qg, part, cfg)
            parts[(b, h)], rts[(b, h)] = part, rt
            dens.append(rt.density)
            need = np.arange(N) if rows is None else np.union1d(rows, part.probe)
            for j in range(g):
                hq = h * g + j
                o, l = sparse_attention(Q[b, hq], K[b, h], V[b, h], part.qgroup, part.kgroup, rt.sel,
                                        rows=need)
                Os[b, hq], LSE[b, hq] = o, l
                out = o.copy()
                if M:
                    fit = fit_head(Q[b, hq], K[b, h], V[b, h], o[part.probe], part, cfg)
                    fits[(b, hq)] = fit
                    if not (flags & FLAG_HARD_DROP_ONLY):
                        ok = ~np.isnan(o[:, 0])
                        out[ok] = o[ok] + correction(o[ok], fit.U, fit.A, fit.obar, fit.Rbar, flags)
                        out[part.probe] = fit.Odense
                O[b, hq] = out
    route_density = float(np.mean(dens))
    return {
        "O": O, "O_sparse": Os, "lse": LSE, "partitions": parts, "routes": rts, "fits": fits,
        "route_density": route_density, "rho_exec": route_density + M / float(N),
    }


def dense_attention(Q, K, V, rows=None):
    """Dense softmax attention for every head (the baseline the method is measured against)."""
    B, Hq, N, d = Q.shape
    g = Hq // K.shape[1]
    idx = np.arange(N) if rows is None else np.asarray(rows)
    O = np.empty((B, Hq, len(idx), d))
    for b in range(B):
        for hq in range(Hq):
            O[b, hq], _ = dense_attention_rows(Q[b, hq, idx], K[b, hq // g], V[b, hq // g])
    return O
