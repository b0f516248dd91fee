"""Planted mistakes in the oracle, on the CPU: the pins must notice them.

Each case below replaces one oracle function by a copy that carries one plausible mistake --
a dropped term, a wrong sign or scale, an index off by one, a transposed operand, a wrong tie
or ordering rule -- and runs the pins written for that function (the brute-force, closed-form
and invariant tests in the other ``test_oracle_*`` files). At least one of them must fail with
an assertion. This shows that the pins tie the oracle to the page's definitions closely enough
that such a mistake cannot pass unnoticed; it runs the oracle only, never the GPU path.

The replacement is made both in the package namespace (``oracle.f``, which the pins call) and
in the implementing module (``oracle.sparsepr.f``, which the oracle's own composite functions
call), and undone after each case.
"""
import importlib
import math

import numpy as np
import pytest

import oracle
import oracle.sparsepr as osp

_f32 = osp._to_f32
# the oracle's functions as written; the mutants that change one step of a function call it here
_ORIG = dict(vars(osp))


# ---------------------------------------------------------------- mutants

def m_sample_rows_no_half(n, s):
    """Strided sample without the half-step offset: floor(i n / s)."""
    i = np.arange(s, dtype=np.int64)
    return (i * np.int64(n)) // np.int64(s)


def m_rademacher_wrong_scale(Gk, rQ, seed):
    """Entries of magnitude 1/sqrt(Gk) instead of 1/sqrt(rQ)."""
    return _ORIG["rademacher_projection"](Gk, rQ, seed) * math.sqrt(rQ) / math.sqrt(Gk)


def m_splitmix64_wrong_shift(x):
    """First xor-shift by 31 instead of 30."""
    M = (1 << 64) - 1
    z = (x + 0x9E3779B97F4A7C15) & M
    z = ((z ^ (z >> 31)) * 0xBF58476D1CE4E5B9) & M
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & M
    return z ^ (z >> 31)


def m_budget_no_probe_cost(rho, N, M):
    """Route budget without the probes' M N pairs taken off."""
    return int(math.floor(float(np.float32(rho)) * float(N * N)))


def m_response_features_head0(Qg, Kh, S):
    """Every sample from query head 0 (the GQA cycling over heads dropped)."""
    g, N, d = Qg.shape
    Qs = Qg[0, osp.sample_rows(N, S), :]
    z = (Qs @ Kh.T) / math.sqrt(d)
    return z, _f32(z.T)


def m_response_features_no_scale(Qg, Kh, S):
    """Responses without the 1/sqrt(d) scale."""
    z, _ = _ORIG["response_features"](Qg, Kh, S)
    z = z * math.sqrt(Qg.shape[2])
    return z, _f32(z.T)


def m_top_mass_floor(z_row, mass=0.9):
    """Key count one short: the keys strictly before the cumulative mass reaches the target."""
    z = np.asarray(z_row, dtype=np.float64)
    p = np.sort(np.exp(z - z.max()))[::-1]
    c = np.cumsum(p)
    k = int(np.searchsorted(c, mass * c[-1], side="left"))
    return max(min(k, len(p)), 1) / len(p)


def m_sq_dists_no_cc(X, C):
    """Distance without the ||c||^2 term."""
    X64, C64 = np.asarray(X, np.float64), np.asarray(C, np.float64)
    return _f32((X64 * X64).sum(1)[:, None] - 2.0 * (X64 @ C64.T))


def m_sq_dists_sign(X, C):
    """Cross term with the wrong sign: ||x||^2 + 2 x.c + ||c||^2."""
    X64, C64 = np.asarray(X, np.float64), np.asarray(C, np.float64)
    return _f32((X64 * X64).sum(1)[:, None] + 2.0 * (X64 @ C64.T) + (C64 * C64).sum(1)[None, :])


def m_kmeans_assign_ties_high(X, C):
    """Ties between centroids go to the highest group id."""
    D = osp.sq_dists_f32(X, C)
    G = D.shape[1]
    lab = G - 1 - D[:, ::-1].argmin(axis=1)
    return lab.astype(np.int32), D[np.arange(len(lab)), lab]


def m_kmeans_update_off_by_one(X, labels, C):
    """Member sum divided by the count plus one."""
    G = C.shape[0]
    X64 = np.asarray(X, dtype=np.float64)
    sums = np.zeros((G, X64.shape[1]))
    np.add.at(sums, labels, X64)
    cnt = np.bincount(labels, minlength=G)
    out = C.astype(np.float32).copy()
    nz = cnt > 0
    out[nz] = _f32(sums[nz] / (cnt[nz, None] + 1))
    return out


def m_kmeans_update_empty_zero(X, labels, C):
    """An empty group's centroid reset to zero instead of kept."""
    out = _ORIG["kmeans_update"](X, labels, C)
    out[np.bincount(labels, minlength=C.shape[0]) == 0] = 0.0
    return out


def m_group_means_over_n(Y, labels, G):
    """Group sums divided by the row count of the whole head."""
    Y64 = np.asarray(Y, dtype=np.float64)
    sums = np.zeros((G, Y64.shape[1]))
    np.add.at(sums, labels, Y64)
    return _f32(sums / len(Y64))


def m_stable_order_reversed_within(labels, G):
    """Group-major order with descending original index inside a group."""
    labels = np.asarray(labels)
    n = len(labels)
    perm = np.lexsort((-np.arange(n), labels)).astype(np.int32)
    off = np.zeros(G + 1, dtype=np.int64)
    np.cumsum(np.bincount(labels, minlength=G), out=off[1:])
    return perm, off.astype(np.int32)


def m_query_logits_no_scale(Qh, kcent):
    """Logits without the 1/sqrt(d) scale."""
    return _f32(Qh @ np.asarray(kcent, np.float64).T)


def m_query_coordinates_no_centring(Qg, kcent, rQ, seed):
    """Coordinates from the uncentred logits."""
    u = osp.query_logits(Qg.mean(axis=0), kcent)
    y = u.astype(np.float64)
    Gk = kcent.shape[0]
    if Gk > rQ:
        y = y @ osp.rademacher_projection(Gk, rQ, seed)
    y = y / np.linalg.norm(y, axis=1, keepdims=True)
    return u, _f32(y)


def m_query_coordinates_head0(Qg, kcent, rQ, seed):
    """Coordinates of the first query head instead of the mean over the KV group's heads."""
    return _ORIG["query_coordinates"](Qg[:1], kcent, rQ, seed)


def m_cell_scores_no_group_size(u_heads, ksize, qgroup, Gq):
    """Softmax normaliser over centroids without the key-group sizes |K_g|."""
    return _ORIG["cell_scores"](u_heads, np.where(np.asarray(ksize) > 0, 1, 0), qgroup, Gq)


def m_cell_scores_sum_not_mean(u_heads, ksize, qgroup, Gq):
    """Scores summed over the query group's rows instead of averaged."""
    S = _ORIG["cell_scores"](u_heads, ksize, qgroup, Gq).astype(np.float64)
    qsize = np.bincount(np.asarray(qgroup), minlength=Gq)
    return _f32(S * np.maximum(qsize, 1)[:, None])


def _select_with(S, qsize, ksize, N, M, rho, *, tie_high=False, keep_crossing=False, no_mandatory=False):
    S = np.asarray(S, dtype=np.float32)
    qsize, ksize = np.asarray(qsize, np.int64), np.asarray(ksize, np.int64)
    Gq, Gk = S.shape
    cost = qsize[:, None] * ksize[None, :]
    elig = cost > 0
    mand = np.zeros((Gq, Gk), dtype=bool)
    if float(np.float32(rho)) >= 1.0:
        return elig.copy(), mand, int(cost[elig].sum())
    if not no_mandatory:
        for a in range(Gq):
            if elig[a].any():
                mand[a, int(np.where(elig[a], S[a], -np.inf).argmax())] = True
    sel = mand.copy()
    total = int(cost[sel].sum())
    budget = osp.budget_pairs(rho, N, M)
    ai, gi = np.nonzero(elig & ~mand)
    order = np.lexsort(((-gi if tie_high else gi), ai, -S[ai, gi]))
    for c in order:
        a, g = int(ai[c]), int(gi[c])
        cc = int(cost[a, g])
        if total + cc <= budget:
            sel[a, g] = True
            total += cc
            continue
        if keep_crossing or total + cc - budget < budget - total:
            sel[a, g] = True
            total += cc
        break
    return sel, mand, total


def m_select_ties_high_key(S, qsize, ksize, N, M, rho):
    """Equal scores visited from the higher key group."""
    return _select_with(S, qsize, ksize, N, M, rho, tie_high=True)


def m_select_keeps_crossing_cell(S, qsize, ksize, N, M, rho):
    """The cell that crosses the budget always kept."""
    return _select_with(S, qsize, ksize, N, M, rho, keep_crossing=True)


def m_select_no_mandatory(S, qsize, ksize, N, M, rho):
    """No mandatory top cell per query group."""
    return _select_with(S, qsize, ksize, N, M, rho, no_mandatory=True)


def m_sparse_attention_transposed_mask(Qh, Kh, Vh, qgroup, kgroup, sel, rows=None):
    """Kept cells read from the transposed selection (sel[g, a] for query group a, key group g)."""
    Gq, Gk = sel.shape
    n = max(Gq, Gk)
    big = np.zeros((n, n), dtype=bool)
    big[:Gk, :Gq] = sel.T
    for a in range(n):                          # keep every query group's key set non-empty
        if not big[a].any():
            big[a, 0] = True
    return _ORIG["sparse_attention"](Qh, Kh, Vh, qgroup, kgroup, big[:Gq, :Gk], rows)


def m_sparse_attention_lse_no_max(Qh, Kh, Vh, qgroup, kgroup, sel, rows=None):
    """Log-sum-exp without the row maximum added back."""
    O, lse = _ORIG["sparse_attention"](Qh, Kh, Vh, qgroup, kgroup, sel, rows)
    d = Qh.shape[1]
    out = lse.copy()
    for a in range(sel.shape[0]):
        qi = np.nonzero(qgroup == a)[0]
        kj = np.nonzero(np.isin(kgroup, np.nonzero(sel[a])[0]))[0]
        if qi.size and kj.size:
            out[qi] -= ((Qh[qi] @ Kh[kj].T) / math.sqrt(d)).max(axis=1)
    return O, out


def m_dense_rows_scale_d(Qrows, Kh, Vh):
    """Dense attention scaled by 1/d instead of 1/sqrt(d)."""
    d = Qrows.shape[1]
    Z = (Qrows @ Kh.T) / d
    m = Z.max(axis=1, keepdims=True)
    P = np.exp(Z - m)
    l = P.sum(axis=1, keepdims=True)
    return (P @ Vh) / l, m[:, 0] + np.log(l[:, 0])


def m_probe_rows_radial_descending(qgroup, radial, M):
    """Within-group order by descending distance to the centroid."""
    N = len(qgroup)
    seq = np.lexsort((np.arange(N), -np.asarray(radial, np.float32), np.asarray(qgroup)))
    pos = osp.sample_rows(N, M)
    return seq[pos].astype(np.int32), pos.astype(np.int32)


def m_coverage_orphans_dropped(pos, qoff, M, N):
    """Groups without a probe give their size to nobody."""
    pos, qoff = np.asarray(pos, np.int64), np.asarray(qoff, np.int64)
    pg = np.searchsorted(qoff, pos, side="right") - 1
    raw = np.zeros(len(pos))
    for a in range(len(qoff) - 1):
        mine = np.nonzero(pg == a)[0]
        if mine.size:
            raw[mine] += (qoff[a + 1] - qoff[a]) / mine.size
    return raw * (M / float(N))


def m_ridge_uncentred(X, Y, w, lam):
    """Ridge map fitted on the raw rows (the weighted means not taken off)."""
    w = np.asarray(w, dtype=np.float64)
    xbar, ybar = (w @ X) / w.sum(), (w @ Y) / w.sum()
    Gm = X.T @ (w[:, None] * X) + lam * np.eye(X.shape[1])
    A = np.linalg.solve(Gm, (Y.T @ (w[:, None] * X)).T).T
    return A, xbar, ybar


def m_ridge_unweighted(X, Y, w, lam):
    """Ridge map with the coverage weights left out of the normal equations."""
    return _ORIG["ridge_fit"](X, Y, np.ones(len(w)), lam)


def m_ridge_dual_no_lambda(X, Y, w, lam):
    """Kernel system without the ridge term."""
    return _ORIG["ridge_fit_dual"](X, Y, w, 1e-300)


def m_subspace_unweighted(R, w, r):
    """Residual subspace of the unweighted residuals."""
    return _ORIG["residual_subspace"](R, np.ones(len(w)), r)


def m_subspace_right_vectors(R, w, r):
    """Right singular vectors (over probes) taken for the output directions (a transposed operand)."""
    Rw = np.sqrt(np.asarray(w, np.float64))[:, None] * R
    _, s, Vt = np.linalg.svd(Rw.T, full_matrices=False)
    k = min(r, int((s > s[0] * max(Rw.shape) * np.finfo(np.float64).eps).sum())) if s.size and s[0] else 0
    V = Vt.T
    out = np.zeros((R.shape[1], k))
    m = min(V.shape[0], R.shape[1])
    out[:m] = V[:m, :k]
    return out, s


def m_correction_rbar_unprojected(Os, U, A, obar, Rbar, flags=0):
    """Default path leaves the mean residual outside the projection."""
    if flags:
        return _ORIG["correction"](Os, U, A, obar, Rbar, flags)
    return Rbar + ((Os - obar) @ A.T) @ (U @ U.T)


def m_correction_sign(Os, U, A, obar, Rbar, flags=0):
    """Centring with the wrong sign: A (o + obar)."""
    return _ORIG["correction"](Os, U, A, -obar, Rbar, flags)


def m_top_mass_set_strict(z_row, mass=0.9):
    """Keys tied with the k-th largest logit left out (strict comparison)."""
    z = np.asarray(z_row, dtype=np.float64)
    k = osp.top_mass_count(z, mass)
    return z > np.sort(z)[::-1][k - 1]


def m_top_mass_count_right(z_row, mass=0.9):
    """Cumulative-mass search from the right: one key too many when the mass lands exactly."""
    z = np.asarray(z_row, dtype=np.float64)
    c = np.cumsum(np.sort(np.exp(z - z.max()))[::-1])
    return min(int(np.searchsorted(c, mass * c[-1], side="right")) + 1, len(z))


def m_shared_rows_no_half(lo, hi, R=osp.SHARED_ROWS):
    """Shared-route rows without the half-step offset."""
    size = hi - lo
    Rp = min(R, size)
    return lo + (np.arange(Rp, dtype=np.int64) * size) // Rp


def m_shared_support_largest_not_union(Qg, Kh, qperm, qoff, R=osp.SHARED_ROWS, mass=0.9):
    """The group's support taken as its largest single-row set instead of the union."""
    union, single = _ORIG["shared_support"](Qg, Kh, qperm, qoff, R, mass)
    return single.max(axis=1), single


def m_shared_support_head0(Qg, Kh, qperm, qoff, R=osp.SHARED_ROWS, mass=0.9):
    """Every shared row taken from query head 0 (the cycling over the KV group's heads dropped)."""
    return _ORIG["shared_support"](Qg[:1], Kh, qperm, qoff, R, mass)


def m_probe_uniform_no_half(qperm, M):
    """Uniform probe grid without the half-step offset."""
    rows = (np.arange(M, dtype=np.int64) * len(qperm)) // M
    return osp._by_sequence_position(rows, qperm)


def m_probe_random_no_salt(qperm, M, seed):
    """Random probes drawn from the seed without the salt."""
    return _ORIG["probe_rows_random"](qperm, M, seed ^ osp.PROBE_SEED_SALT)


def m_affine_total_denominator(Os, Od):
    """Explained fraction over the uncentred residual energy."""
    Os = np.asarray(Os, dtype=np.float64)
    R = np.asarray(Od, dtype=np.float64) - Os
    X = np.concatenate([Os, np.ones((Os.shape[0], 1))], axis=1)
    beta, *_ = np.linalg.lstsq(X, R, rcond=None)
    sse = float(((R - X @ beta) ** 2).sum())
    return 1.0 - sse / float((R ** 2).sum()), sse / float((R ** 2).sum())


def m_affine_no_intercept(Os, Od):
    """Affine fit without the constant column (a linear fit)."""
    Os = np.asarray(Os, dtype=np.float64)
    R = np.asarray(Od, dtype=np.float64) - Os
    beta, *_ = np.linalg.lstsq(Os, R, rcond=None)
    sse = float(((R - Os @ beta) ** 2).sum())
    return 1.0 - sse / float(((R - R.mean(axis=0)) ** 2).sum()), sse / float((R ** 2).sum())


def m_call_no_probe_override(Q, K, V, cfg, rows=None, partitions=None, routes=None):
    """Probe rows of the output left as corrected sparse rows instead of the exact dense rows."""
    res = _ORIG["sparsepr_attention"](Q, K, V, cfg, rows, partitions, routes)
    g = Q.shape[1] // K.shape[1]
    for (b, hq), fit in res["fits"].items():
        p = res["partitions"][(b, hq // g)].probe
        o = res["O_sparse"][b, hq, p]
        res["O"][b, hq, p] = o + osp.correction(o, fit.U, fit.A, fit.obar, fit.Rbar, getattr(cfg, "flags", 0))
    return res


def m_call_rho_exec_without_probes(Q, K, V, cfg, rows=None, partitions=None, routes=None):
    """Execution density reported without the probes' share M/N."""
    res = _ORIG["sparsepr_attention"](Q, K, V, cfg, rows, partitions, routes)
    res["rho_exec"] = res["route_density"]
    return res


# ---------------------------------------------------------------- cases

P = "test_oracle_partition"
R = "test_oracle_route_attn_fit"
D = "test_oracle_steps_direct"
SS = "test_oracle_shared_support"

CASES = [
    ("sample_rows", m_sample_rows_no_half, [(P, "test_sample_rows_closed_form")]),
    ("rademacher_projection", m_rademacher_wrong_scale, [(P, "test_rademacher_projection_properties")]),
    ("splitmix64", m_splitmix64_wrong_shift, [(P, "test_splitmix64_published_outputs")]),
    ("budget_pairs", m_budget_no_probe_cost, [(R, "test_budget_pairs_and_rho_exec_formula_with_page_numbers")]),
    ("response_features", m_response_features_head0, [(P, "test_response_features_brute_force_gqa")]),
    ("response_features", m_response_features_no_scale, [(P, "test_response_features_brute_force_gqa")]),
    ("top_mass_fraction", m_top_mass_floor, [(P, "test_top_mass_fraction_closed_forms")]),
    ("sq_dists_f32", m_sq_dists_no_cc, [(P, "test_sq_dists_matches_direct_form")]),
    ("sq_dists_f32", m_sq_dists_sign, [(P, "test_sq_dists_matches_direct_form")]),
    ("kmeans_assign", m_kmeans_assign_ties_high, [(P, "test_kmeans_assign_brute_force_and_ties")]),
    ("kmeans_update", m_kmeans_update_off_by_one, [(D, "test_kmeans_update_is_the_member_mean"),
                                                   (P, "test_kmeans_planted_clusters_exact_recovery")]),
    ("kmeans_update", m_kmeans_update_empty_zero, [(D, "test_kmeans_update_is_the_member_mean")]),
    ("group_means", m_group_means_over_n, [(P, "test_group_means_brute_force_and_empty")]),
    ("stable_group_order", m_stable_order_reversed_within, [(P, "test_stable_group_order_is_stable_bijection")]),
    ("query_logits", m_query_logits_no_scale, [(D, "test_query_logits_by_loops")]),
    ("query_coordinates", m_query_coordinates_no_centring, [(P, "test_query_coordinates_properties")]),
    ("query_coordinates", m_query_coordinates_head0, [(P, "test_query_coordinates_properties")]),
    ("cell_scores", m_cell_scores_no_group_size, [(R, "test_cell_scores_brute_force_and_mass_identity")]),
    ("cell_scores", m_cell_scores_sum_not_mean, [(R, "test_cell_scores_brute_force_and_mass_identity")]),
    ("select_cells", m_select_ties_high_key, [(R, "test_select_cells_matches_prefix_rule_exhaustive")]),
    ("select_cells", m_select_keeps_crossing_cell, [(R, "test_select_cells_matches_prefix_rule_exhaustive"),
                                                    (R, "test_select_cells_budget_and_order_invariants")]),
    ("select_cells", m_select_no_mandatory, [(R, "test_select_cells_matches_prefix_rule_exhaustive"),
                                             (R, "test_select_cells_budget_and_order_invariants")]),
    ("sparse_attention", m_sparse_attention_transposed_mask, [(R, "test_sparse_attention_brute_force_masking")]),
    ("sparse_attention", m_sparse_attention_lse_no_max, [(R, "test_sparse_attention_brute_force_masking")]),
    ("dense_attention_rows", m_dense_rows_scale_d, [(R, "test_sparse_attention_full_density_is_dense_softmax")]),
    ("probe_rows", m_probe_rows_radial_descending, [(R, "test_probe_rows_stratified_radial_brute_force")]),
    ("coverage_weights", m_coverage_orphans_dropped, [(R, "test_coverage_weights_brute_force")]),
    ("ridge_fit", m_ridge_uncentred, [(R, "test_ridge_recovers_planted_affine_map"),
                                      (R, "test_ridge_primal_equals_dual")]),
    ("ridge_fit", m_ridge_unweighted, [(R, "test_ridge_primal_equals_dual")]),
    ("ridge_fit_dual", m_ridge_dual_no_lambda, [(R, "test_ridge_primal_equals_dual")]),
    ("residual_subspace", m_subspace_unweighted, [(R, "test_residual_subspace_equals_gram_eigenvectors")]),
    ("residual_subspace", m_subspace_right_vectors, [(R, "test_residual_subspace_equals_gram_eigenvectors")]),
    ("correction", m_correction_rbar_unprojected, [(R, "test_correction_variants")]),
    ("correction", m_correction_sign, [(R, "test_correction_variants")]),
    ("top_mass_set", m_top_mass_set_strict, [(SS, "test_top_mass_set_closed_forms")]),
    ("top_mass_count", m_top_mass_count_right, [(SS, "test_top_mass_set_closed_forms")]),
    ("shared_rows", m_shared_rows_no_half, [(SS, "test_shared_rows_positions")]),
    ("shared_support", m_shared_support_largest_not_union, [(SS, "test_shared_support_brute_force")]),
    ("shared_support", m_shared_support_head0, [(SS, "test_shared_support_brute_force")]),
    ("probe_rows_uniform", m_probe_uniform_no_half, [(SS, "test_alternative_probe_samplers")]),
    ("probe_rows_random", m_probe_random_no_salt, [(SS, "test_alternative_probe_samplers")]),
    ("affine_diagnostics", m_affine_total_denominator, [(SS, "test_affine_diagnostics_planted")]),
    ("affine_diagnostics", m_affine_no_intercept, [(SS, "test_affine_diagnostics_planted")]),
    ("sparsepr_attention", m_call_no_probe_override, [(R, "test_probe_rows_of_output_are_dense_rows_exactly")]),
    ("sparsepr_attention", m_call_rho_exec_without_probes, [(R, "test_realised_density_and_rho_exec")]),
]


@pytest.mark.parametrize("target,mutant,pins", CASES, ids=[m.__name__[2:] for _, m, _ in CASES])
def test_pins_catch_planted_mistake(target, mutant, pins, monkeypatch):
    monkeypatch.setattr(osp, target, mutant)
    monkeypatch.setattr(oracle, target, mutant)
    caught = []
    for mod, name in pins:
        fn = getattr(importlib.import_module(mod), name)
        try:
            fn()
        except AssertionError:
            caught.append(name)
    assert caught, f"no pin noticed the mistake '{mutant.__doc__.strip()}' planted in oracle.{target}"


def test_pins_pass_on_the_oracle_as_written():
    """Control: the same pins pass with the oracle unchanged."""
    for mod, name in sorted({pin for _, _, ps in CASES for pin in ps}):
        getattr(importlib.import_module(mod), name)()
