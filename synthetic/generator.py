"""Seeded synthetic Q/K/V with the structure of video-DiT attention.

Recipe (per batch element b and KV head h, one independent random stream each):
  * token n = t*Hg*Wg + y*Wg + x sits at position p = (t/T, y/Hg, x/Wg);
  * 8 random-phase Fourier features phi_j(p) = cos(2*pi*w_j.p + theta_j), with
    every component of w_j ~ U[0.5, 3] and theta_j ~ U[0, 2*pi);
  * one Gaussian matrix G ~ N(0, 1/8) of shape 8 x d shared by Q and K, so
    q.k reflects positional similarity;
  * K = a*phi(p)G + s*eps_K and, for every query head of the KV group,
    Q = a*phi(p)G + s*eps_Q, with s = noise. Workloads that state a locality
    target (the 720p, world-model, sweep and stack calls) use
    a = 0.8*sqrt(2)*locality**0.4: the locality scale enters the amplitude
    through that power law, fitted so that one law meets both stated targets
    (at locality 1.2, noise 0.3 and N=118800 a single query row needs a
    median 5-10% of the keys for 90% of its softmax mass; at locality 0.4,
    noise 0.6 and N=75600 about 50%). The tiny and mid calls, which state the
    amplitude 0.8 and no target, use a = 0.8*locality;
  * V ~ N(0, 1);
  * everything rounded to bf16 (round to nearest even) and returned as the
    16-bit patterns, so both consumers see identical bits.
"""
from __future__ import annotations

import concurrent.futures as _cf
import os

import numpy as np

AMPLITUDE = 0.8
LOCALITY_GAIN = 2.0 ** 0.5
LOCALITY_EXPONENT = 0.4
N_FEATURES = 8


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = u + np.uint32(0x7FFF) + lsb
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


def amplitude(w, locality: float | None = None) -> float:
    """Amplitude a of the positional part of Q and K for workload w (locality override optional)."""
    loc = w.locality if locality is None else locality
    if getattr(w, "calibrated", True):
        return AMPLITUDE * LOCALITY_GAIN * loc ** LOCALITY_EXPONENT
    return AMPLITUDE * loc


def _positions(T: int, Hg: int, Wg: int) -> np.ndarray:
    t, y, x = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(Wg), indexing="ij")
    return np.stack([t.ravel() / T, y.ravel() / Hg, x.ravel() / Wg], axis=1)  # [N, 3]


def _one_kv_head(args):
    (seed, layer, b, h, g, pos, d, amp, noise) = args
    rng = np.random.default_rng(np.random.SeedSequence([seed, layer, b, h]))
    omega = rng.uniform(0.5, 3.0, size=(N_FEATURES, 3))
    theta = rng.uniform(0.0, 2.0 * np.pi, size=(N_FEATURES,))
    G = rng.normal(0.0, np.sqrt(1.0 / N_FEATURES), size=(N_FEATURES, d))
    phi = np.cos(2.0 * np.pi * (pos @ omega.T) + theta)          # [N, 8]
    base = (amp * (phi @ G)).astype(np.float32)                   # [N, d]
    N = pos.shape[0]
    k = base + noise * rng.standard_normal((N, d), dtype=np.float32)
    qs = [base + noise * rng.standard_normal((N, d), dtype=np.float32) for _ in range(g)]
    v = rng.standard_normal((N, d), dtype=np.float32)
    return (b, h, [bf16_bits_from_f32(q) for q in qs], bf16_bits_from_f32(k), bf16_bits_from_f32(v))


def video_qkv(w, layer: int = 0, locality: float | None = None, threads: int | None = None):
    """Draw (Q, K, V) for workload ``w`` as bf16 bit patterns (uint16).

    Shapes: Q [B, Hq, N, d], K and V [B, Hkv, N, d]. Query head hq belongs to
    KV head hq // (Hq // Hkv).
    """
    amp = amplitude(w, locality)
    pos = _positions(w.T, w.Hg, w.Wg)
    N, d, g = w.N, w.d, w.g
    Q = np.empty((w.B, w.Hq, N, d), dtype=np.uint16)
    K = np.empty((w.B, w.Hkv, N, d), dtype=np.uint16)
    V = np.empty((w.B, w.Hkv, N, d), dtype=np.uint16)
    jobs = [(w.seed, layer, b, h, g, pos, d, amp, w.noise) for b in range(w.B) for h in range(w.Hkv)]
    nthreads = threads or min(len(jobs), os.cpu_count() or 1)
    with _cf.ThreadPoolExecutor(max_workers=nthreads) as ex:
        for b, h, qs, k, v in ex.map(_one_kv_head, jobs):
            for j, q in enumerate(qs):
                Q[b, h * g + j] = q
            K[b, h] = k
            V[b, h] = v
    return Q, K, V


def video_qkv_device(w, layer: int = 0, locality: float | None = None, device: str = "cuda"):
    """The same recipe drawn on the GPU with torch's generator, as bf16 tensors Q [B, Hq, N, d],
    K, V [B, Hkv, N, d]. Its random streams differ from video_qkv's (same distributions, other
    values); it serves stacks of many layers, whose inputs would take minutes on the host."""
    import torch

    amp = amplitude(w, locality)
    pos = torch.from_numpy(_positions(w.T, w.Hg, w.Wg)).to(device=device, dtype=torch.float64)
    N, d, g = w.N, w.d, w.g
    Q = torch.empty((w.B, w.Hq, N, d), dtype=torch.bfloat16, device=device)
    K = torch.empty((w.B, w.Hkv, N, d), dtype=torch.bfloat16, device=device)
    V = torch.empty((w.B, w.Hkv, N, d), dtype=torch.bfloat16, device=device)
    for b in range(w.B):
        for h in range(w.Hkv):
            seed = int(np.random.SeedSequence([w.seed, layer, b, h]).generate_state(1, dtype=np.uint64)[0] >> 1)
            gen = torch.Generator(device=device).manual_seed(seed)
            omega = torch.rand((N_FEATURES, 3), generator=gen, device=device, dtype=torch.float64) * 2.5 + 0.5
            theta = torch.rand((N_FEATURES,), generator=gen, device=device, dtype=torch.float64) * (2.0 * np.pi)
            G = torch.randn((N_FEATURES, d), generator=gen, device=device, dtype=torch.float64) * np.sqrt(1.0 / N_FEATURES)
            phi = torch.cos(2.0 * np.pi * (pos @ omega.T) + theta)
            base = (amp * (phi @ G)).float()
            K[b, h] = (base + w.noise * torch.randn((N, d), generator=gen, device=device)).bfloat16()
            for j in range(g):
                Q[b, h * g + j] = (base + w.noise * torch.randn((N, d), generator=gen, device=device)).bfloat16()
            V[b, h] = torch.randn((N, d), generator=gen, device=device).bfloat16()
    return Q, K, V
