"""Shared helpers of the GPU parity tests: seeded inputs on both sides, the
oracle's partition and route converted into device tensors to hand them in,
and the comparison metrics."""
from __future__ import annotations

import numpy as np

import oracle
from synthetic import bf16_bits_to_f64, video_qkv

MAX_ABS = 2e-2    # element-wise tolerance on bf16 outputs with fp32 accumulation
MEAN_ABS = 2e-3


def inputs(w, layer=0):
    """Seeded bf16 Q/K/V: (numpy fp64 copies for the oracle, torch bf16 CUDA tensors)."""
    import torch

    Qb, Kb, Vb = video_qkv(w, layer=layer)
    host = tuple(bf16_bits_to_f64(x) for x in (Qb, Kb, Vb))
    dev = tuple(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda() for x in (Qb, Kb, Vb))
    return host, dev


def bf16_to_f64(t):
    import torch

    return t.detach().float().cpu().double().numpy() if t.dtype != torch.float64 else t.cpu().numpy()


def partition_tensors(res, w):
    """Oracle partitions of every (b, kv head) as device tensors in the C ABI layout."""
    import torch

    P, N, M = w.B * w.Hkv, w.N, w.M
    keys = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    parts = [res["partitions"][k] for k in keys]

    def stack(f, dt):
        return torch.from_numpy(np.stack([f(p) for p in parts]).astype(dt)).cuda()

    def probe_pos(p):
        inv = np.empty(N, dtype=np.int64)
        inv[p.qperm] = np.arange(N)
        return inv[p.probe]

    t = {
        "kgroup": stack(lambda p: p.kgroup, np.int32), "qgroup": stack(lambda p: p.qgroup, np.int32),
        "kperm": stack(lambda p: p.kperm, np.int32), "koff": stack(lambda p: p.koff, np.int32),
        "qperm": stack(lambda p: p.qperm, np.int32), "qoff": stack(lambda p: p.qoff, np.int32),
        "kcent": stack(lambda p: p.kcent, np.float32), "radial": stack(lambda p: p.radial, np.float32),
    }
    if M:
        t["probe"] = stack(lambda p: p.probe, np.int32)
        t["probe_pos"] = stack(probe_pos, np.int32)
        t["weights"] = stack(lambda p: p.weights, np.float32)
    assert all(v.shape[0] == P for v in t.values())
    return t


def route_tensors(res, w):
    import torch

    keys = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    rowptr = np.stack([res["routes"][k].rowptr for k in keys]).astype(np.int32)
    kg = np.zeros((len(keys), w.Gq * w.Gk), dtype=np.int32)
    for i, k in enumerate(keys):
        r = res["routes"][k]
        kg[i, : len(r.kg)] = r.kg
    pairs = np.array([res["routes"][k].pairs for k in keys], dtype=np.int64)
    return {"rowptr": torch.from_numpy(rowptr).cuda(), "kg": torch.from_numpy(kg).cuda(),
            "pairs": torch.from_numpy(pairs).cuda()}


def to_group_major(O, res, w):
    """Oracle [B, Hq, N, d] in original order -> each head's group-major order."""
    out = np.empty_like(O)
    for b in range(w.B):
        for hq in range(w.Hq):
            out[b, hq] = O[b, hq, res["partitions"][(b, hq // w.g)].qperm]
    return out


def err(a, b):
    d = np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64))
    return float(d.max()), float(d.mean())


def assert_close(a, b, what, max_abs=MAX_ABS, mean_abs=MEAN_ABS):
    mx, mn = err(a, b)
    assert mx <= max_abs and mn <= mean_abs, f"{what}: max-abs {mx:.3e} (<= {max_abs}), mean-abs {mn:.3e} (<= {mean_abs})"
    return mx, mn


def kmeans_margin(X, C):
    """Relative margin (d2 - d1) / d2 of each row's two nearest centroids (oracle distances)."""
    D = oracle.sq_dists_f32(X, C).astype(np.float64)
    s = np.sort(D, axis=1)
    d1, d2 = s[:, 0], s[:, 1] if s.shape[1] > 1 else s[:, 0] + 1.0
    return (d2 - d1) / np.maximum(d2, 1e-30)


def selected_from_csr(rowptr, kg, Gq, Gk):
    sel = np.zeros((Gq, Gk), dtype=bool)
    for a in range(Gq):
        sel[a, kg[rowptr[a]:rowptr[a + 1]]] = True
    return sel


def sampled_call_parity(w, Qb, Kb, Vb, kv_heads=None, rows_per_head=48, seed=7):
    """Parity of one whole call at a size where the oracle can only afford samples.

    The call runs on the GPU once fused (sparsepr_attention) and once stage by stage (the outputs
    must agree bit for bit). On the KV heads `kv_heads` (default: the first and the last) the
    oracle then checks the response features at sampled keys, the group-major orders and offsets
    (a stable sort of the GPU's labels), key-group means at sampled groups, the cell scores (its
    formula on the GPU's partition), the selected cells (its selection rule on the GPU's scores:
    identical cells and pair count), and, with the GPU's partition and route handed to it, the
    sparse output O_s and the corrected output O at sampled query rows and every probe row
    (max-abs 2e-2, mean-abs 2e-3). Probe rows of O must equal the GPU's dense rows rounded to
    bf16 exactly. Qb, Kb, Vb are the bf16 bit patterns of the inputs.
    """
    import torch

    import free_block_sparse_sparsepr_b200 as spr

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

    rng = np.random.default_rng(seed)
    srows = oracle.sample_rows(N, w.rK)
    heads = sorted({0, P - 1}) if kv_heads is None else list(kv_heads)
    for z in heads:
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
        nonempty = np.nonzero(np.diff(pv["koff"][z]))[0]
        for grp in rng.choice(nonempty, min(8, len(nonempty)), replace=False):
            ref = Kh[pv["kgroup"][z] == grp].mean(axis=0)
            assert np.abs(kcent[grp] - ref).max() <= 1e-5 * max(1.0, np.abs(ref).max())
        # (3) cell scores (the oracle's formula on the GPU's partition) and the selection
        ksize, qsize = np.diff(pv["koff"][z]), np.diff(pv["qoff"][z])
        u_heads = [oracle.query_logits(Qg[j], kcent) for j in range(g)]
        S_ref = oracle.cell_scores(u_heads, ksize, pv["qgroup"][z], w.Gq)
        S = rv["scores"][z]
        assert np.abs(S - S_ref).max() <= 2e-3 * np.abs(S_ref).max()
        sel_ref, _, pairs_ref = oracle.select_cells(S, qsize, ksize, N, w.M, w.rho)
        sel = selected_from_csr(rv["rowptr"][z], rv["kg"][z], w.Gq, w.Gk)
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
        rows = np.union1d(rng.choice(N, rows_per_head, replace=False), hp.probe)
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
    return rv
