"""Voronoi-center video-token workloads.

The pages evaluate SparsePR inside HunyuanVideo-13B, Wan2.2-I2V-A14B and two
Cosmos models (paperlayer.ai summary, §5 "Models and benchmarks"); none of those
weights exist here, so these seeded synthetic tokens stand in for their
attention inputs.  Every token sits on a (t, h, w) latent grid in raster order
(t major).  Each head draws C latent centers mu_c ~ N(0, I_d) and C seed points
uniform in [0, 1)^3; a token takes the label of the seed nearest to its
normalised grid position ((t+1/2)/T, (h+1/2)/H, (w+1/2)/W) (ties to the lower
seed index), then a fraction f of tokens is relabelled uniformly at random.
With independent eps ~ N(0, I):  q = a*mu + eps,  k = a*mu + eps,  v = mu + eps,
a = 2.  Values are drawn in fp32 with torch's CPU generator, seeded per
(workload, batch*heads + head), and rounded to bf16 (round to nearest even).

Nothing here computes any step of the method.
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic attention call plus the method's parameters for it."""

    name: str
    index: int  # seeds are 1000*index + (b*H + h)
    B: int
    H: int
    grid: tuple  # (T, H, W) latent grid
    d: int
    centers: int
    relabel: float
    Ms: int
    p: int
    Gk: int
    Gq: int
    iters: int
    route_mode: str  # "tau" or "budget"
    tau: float
    rho_target: float
    M: int
    r: int
    lam: float
    center_scale: float = 2.0
    partition: str = "response"  # or "semantic" (the comparator)
    weights: str = "coverage"  # or "uniform" (probe weights of the fit)
    probes: str = "stratified"  # or "ranked" (probe rows nearest their centroid)

    @property
    def N(self) -> int:
        t, h, w = self.grid
        return t * h * w

    @property
    def BH(self) -> int:
        return self.B * self.H

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five workloads: a tiny oracle check, a single-layer mid size, a
# HunyuanVideo-13B-shaped call, a Wan2.2-14B-shaped call and a density/probe
# sweep shape.  Query/key group counts for the sweep shape are not given
# anywhere; they equal the center count.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, (4, 16, 16), 64, 32, 0.10,
                     128, 16, 16, 16, 10, "tau", 0.9, 0.0, 64, 8, 1e-3),
    "mid": Workload("mid", 2, 1, 24, (8, 32, 32), 128, 64, 0.10,
                    512, 32, 64, 64, 10, "budget", 1.0, 0.25, 256, 16, 1e-3),
    "hunyuan": Workload("hunyuan", 3, 1, 24, (33, 45, 80), 128, 256, 0.10,
                        2048, 32, 256, 256, 10, "budget", 1.0, 0.25, 1024, 32, 1e-3),
    "wan": Workload("wan", 4, 1, 40, (21, 45, 80), 128, 192, 0.15,
                    2048, 32, 192, 192, 10, "budget", 1.0, 0.25, 1024, 32, 1e-3),
    "sweep": Workload("sweep", 5, 1, 16, (8, 64, 64), 128, 128, 0.10,
                      2048, 32, 128, 128, 10, "budget", 1.0, 0.25, 256, 8, 1e-3),
}


def workload(name: str, **overrides) -> Workload:
    wl = WORKLOADS[name]
    return wl.replace(**overrides) if overrides else wl


def _grid_positions(grid) -> torch.Tensor:
    T, H, W = grid
    t = (torch.arange(T, dtype=torch.float32) + 0.5) / T
    h = (torch.arange(H, dtype=torch.float32) + 0.5) / H
    w = (torch.arange(W, dtype=torch.float32) + 0.5) / W
    tt, hh, ww = torch.meshgrid(t, h, w, indexing="ij")
    return torch.stack([tt.reshape(-1), hh.reshape(-1), ww.reshape(-1)], dim=1)


def voronoi_head(wl: Workload, bh: int, N: int | None = None):
    """Draw one head's (q, k, v) as fp32 [N, d] tensors (before bf16 rounding).

    ``N`` may truncate the grid's raster order (for ragged-size tests); the
    default is the whole grid.
    """
    g = torch.Generator().manual_seed(1000 * wl.index + bh)
    C, d = wl.centers, wl.d
    mu = torch.randn(C, d, generator=g)
    seeds = torch.rand(C, 3, generator=g)
    pos = _grid_positions(wl.grid)
    if N is not None:
        pos = pos[:N]
    n = pos.shape[0]
    lab = torch.empty(n, dtype=torch.long)
    for s in range(0, n, 16384):  # bounded temporary
        dist = ((pos[s:s + 16384, None, :] - seeds[None, :, :]) ** 2).sum(-1)
        lab[s:s + 16384] = torch.argmin(dist, dim=1)  # first minimum: lower index
    relab = torch.rand(n, generator=g) < wl.relabel
    lab = torch.where(relab, torch.randint(0, C, (n,), generator=g), lab)
    a = wl.center_scale
    m = mu[lab]
    q = a * m + torch.randn(n, d, generator=g)
    k = a * m + torch.randn(n, d, generator=g)
    v = m + torch.randn(n, d, generator=g)
    return q, k, v


def voronoi_qkv(wl: Workload, heads=None, N: int | None = None):
    """Q, K, V as bf16 [B, H, N, d] CPU tensors (contiguous).

    ``heads`` restricts generation to a list of flat (b*H + h) indices; the
    result then has shape [1, len(heads), N, d].
    """
    idx = list(range(wl.BH)) if heads is None else list(heads)
    n = wl.N if N is None else N
    shape = (wl.B, wl.H) if heads is None else (1, len(idx))
    Q = torch.empty(len(idx), n, wl.d, dtype=torch.bfloat16)
    K = torch.empty_like(Q)
    V = torch.empty_like(Q)
    for i, bh in enumerate(idx):
        q, k, v = voronoi_head(wl, bh, N=N)
        Q[i] = q.to(torch.bfloat16)
        K[i] = k.to(torch.bfloat16)
        V[i] = v.to(torch.bfloat16)
    return (Q.reshape(*shape, n, wl.d), K.reshape(*shape, n, wl.d),
            V.reshape(*shape, n, wl.d))
