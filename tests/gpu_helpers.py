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
