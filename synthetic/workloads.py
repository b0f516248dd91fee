"""Named workloads: attention shapes of the video DiTs and world models that the
SparsePR page evaluates, plus the method's hyper-parameters for each call.

The shapes stand in for the page's models (HunyuanVideo-13B at 720p, a
world model with grouped-query attention); no weights or datasets are used.
Hyper-parameters rK=48, rQ=64, M=64, lambda=0.1, r=16 and the 22% / 26%
execution densities are the ones the page states for the method.
"""
from __future__ import annotations

import dataclasses


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    T: int          # latent frames
    Hg: int         # latent grid height
    Wg: int         # latent grid width
    d: int          # head dimension
    Gk: int         # key groups
    Gq: int         # query groups
    block: int      # tile rows used by the kernels (no effect on the result)
    rho: float      # target execution density (route density + M/N)
    locality: float = 1.0   # amplitude scale of the positional part of Q and K
    noise: float = 0.3      # standard deviation of the i.i.d. part of Q and K
    rK: int = 48
    rQ: int = 64
    M: int = 64
    r: int = 16
    lam: float = 0.1
    kmeans_iters: int = 10
    seed: int = 0
    calibrated: bool = True  # amplitude 0.8*sqrt(2)*locality**0.4 (locality targets); else 0.8*locality

    @property
    def N(self) -> int:
        return self.T * self.Hg * self.Wg

    @property
    def g(self) -> int:
        return self.Hq // self.Hkv

    def dense_equiv_flops(self) -> float:
        """4*B*Hq*N^2*d: QK^T and PV of dense attention, 2 flops per MAC."""
        return 4.0 * self.B * self.Hq * float(self.N) ** 2 * self.d

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # Tiny single call: 2 heads, d=64, grid 4x16x16.
    # Amplitude 0.8 as stated for this call (no locality target to calibrate to).
    "tiny_n1024": Workload("tiny_n1024", B=1, Hq=2, Hkv=2, T=4, Hg=16, Wg=16, d=64,
                           Gk=16, Gq=16, block=64, rho=0.25, locality=1.0, noise=0.3,
                           calibrated=False),
    # Mid call: 12 heads MHA, d=128, grid 16x32x32.
    # Amplitude 0.8 as stated for this call (no locality target to calibrate to).
    "mid_n16384": Workload("mid_n16384", B=1, Hq=12, Hkv=12, T=16, Hg=32, Wg=32, d=128,
                           Gk=64, Gq=64, block=64, rho=0.22, locality=1.0, noise=0.3,
                           calibrated=False),
    # HunyuanVideo-shaped 720p call: 24 heads MHA, d=128, latent grid 33x45x80.
    "hunyuan720p_n118800": Workload("hunyuan720p_n118800", B=1, Hq=24, Hkv=24, T=33, Hg=45,
                                    Wg=80, d=128, Gk=256, Gq=256, block=128, rho=0.22,
                                    locality=1.2, noise=0.3),
    # World-model-shaped GQA call: 32 query heads on 8 KV heads, grid 21x45x80.
    "worldmodel_gqa_n75600": Workload("worldmodel_gqa_n75600", B=1, Hq=32, Hkv=8, T=21, Hg=45,
                                      Wg=80, d=128, Gk=256, Gq=256, block=128, rho=0.26,
                                      locality=0.4, noise=0.6),
}

# Density / length sweep at 24 heads, d=128 (grids for 8192 and 32760 are our choice).
SWEEP_GRIDS = {8192: (8, 32, 32), 32760: (13, 45, 56), 75600: (21, 45, 80), 118800: (33, 45, 80)}
SWEEP_GROUPS = {8192: 64, 32760: 128, 75600: 256, 118800: 256}
SWEEP_RHOS = (0.10, 0.15, 0.22, 0.30, 0.50, 1.00)


def sweep_workload(N: int, rho: float) -> Workload:
    T, Hg, Wg = SWEEP_GRIDS[N]
    G = SWEEP_GROUPS[N]
    return Workload(f"sweep_n{N}_rho{int(round(rho * 100))}", B=1, Hq=24, Hkv=24, T=T, Hg=Hg,
                    Wg=Wg, d=128, Gk=G, Gq=G, block=128, rho=rho, locality=1.2, noise=0.3)


def stack_layer_locality(layer: int, seed: int = 0) -> float:
    """Locality scale of one layer of the 40-layer denoising-step stack, U[0.4, 1.2]."""
    import numpy as np

    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x57AC, layer]))
    return float(rng.uniform(0.4, 1.2))


def get_workload(name: str) -> Workload:
    """A named workload, or a sweep point named sweep_n<N>_rho<percent>."""
    if name in WORKLOADS:
        return WORKLOADS[name]
    if name.startswith("sweep_n") and "_rho" in name:
        n_part, rho_part = name[len("sweep_n"):].split("_rho")
        return sweep_workload(int(n_part), int(rho_part) / 100.0)
    raise KeyError(f"unknown workload {name!r}; known: {sorted(WORKLOADS)} or sweep_n<N>_rho<pct>")
