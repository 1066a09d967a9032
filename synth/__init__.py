"""Seeded synthetic workloads for exact Lloyd k-means.

This module is shared by the tests, the benchmark and the smoke check. It holds
random draws only: mixture sampling, weight sampling and the choice of initial
centroids among the points. It contains none of the k-means arithmetic (no
distances, no means, no grid initialisation); that lives on the CUDA side and,
independently, in the CPU oracle.

Every generator takes a ``device`` and a ``seed`` and draws from one
``torch.Generator`` on that device, so the same call always returns the same
bits on the same kind of device. Tests that compare the CUDA path with the
oracle generate once and hand the identical tensors to both sides.

The five workloads follow the shapes the Flash-KMeans write-ups measure on
(B=32, N=65536, K=1024, d=128; N=1M, K=8192; N=33M, K=4096; fp16, d=128) and
the per-row weighted 1-D codebook setting of the LeanQuant "1D k-means" issue
(rows of quantisation weights with a per-weight importance, uniform-grid
init). No public dataset is named for this path; these distributions stand in.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

__all__ = ["WORKLOADS", "Workload", "make_workload", "gaussian_mixture", "student_t_rows",
           "pick_init_points"]


@dataclass(frozen=True)
class Workload:
    """Shape and distribution recipe of one synthetic workload."""
    idx: int
    name: str
    B: int
    N: int
    d: int
    K: tuple
    dtype: torch.dtype
    iters: int
    init: str            # "shuffle_first" | "random_points" | "grid"
    weighted: bool
    recipe: str
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    1: Workload(1, "tiny_exact", 1, 4096, 16, (32,), torch.float32, 20, "shuffle_first", False,
                "32-component isotropic Gaussian mixture, means U(-5,5)^16, sigma=0.5, equal weights",
                {"n_comp": 32, "mean": "uniform", "lo": -5.0, "hi": 5.0, "sigma": 0.5}),
    2: Workload(2, "rows_weighted_1d", 4096, 4096, 1, (16, 8), torch.float16, 30, "grid", True,
                "per row Student-t(nu=5)*0.02 values; weights N(0,1)^2+1e-3",
                {"nu": 5, "scale": 0.02}),
    3: Workload(3, "batched_assign_bound", 32, 65536, 128, (1024,), torch.float16, 10, "random_points",
                False, "per batch 1024-component Gaussian mixture, means N(0,1)^128, sigma=0.3",
                {"n_comp": 1024, "mean": "normal", "sigma": 0.3, "mix": "equal"}),
    4: Workload(4, "large_k_assign", 1, 1 << 20, 128, (8192,), torch.float16, 5, "random_points", False,
                "8192-component Gaussian mixture, means N(0,1)^128, sigma=0.25, Dirichlet(1) weights",
                {"n_comp": 8192, "mean": "normal", "sigma": 0.25, "mix": "dirichlet"}),
    5: Workload(5, "contention_update", 1, 1 << 25, 128, (4096,), torch.float16, 3, "random_points",
                False, "4096 Gaussian components, Zipf(1.1) sizes, means N(0,1)^128, sigma=0.3",
                {"n_comp": 4096, "mean": "normal", "sigma": 0.3, "mix": "zipf", "zipf_s": 1.1}),
}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _component_draw(n, mix, n_comp, g, device, zipf_s=1.1):
    """Component label per point: equal weights, Dirichlet(1) weights or Zipf sizes."""
    if mix in ("equal", None):
        return torch.randint(0, n_comp, (n,), generator=g, device=device)
    if mix == "dirichlet":
        # Dirichlet(alpha=1) = normalised unit exponentials.
        e = -torch.log1p(-torch.rand(n_comp, generator=g, device=device, dtype=torch.float64))
        p = e / e.sum()
    elif mix == "zipf":
        k = torch.arange(1, n_comp + 1, device=device, dtype=torch.float64)
        p = k.pow(-zipf_s)
        p = p / p.sum()
    else:
        raise ValueError(mix)
    cdf = torch.cumsum(p, 0)
    u = torch.rand(n, generator=g, device=device, dtype=torch.float64)
    return torch.searchsorted(cdf, u).clamp_(max=n_comp - 1)


def gaussian_mixture(B, N, d, n_comp, sigma, *, mean="normal", lo=-5.0, hi=5.0, mix="equal",
                     zipf_s=1.1, dtype=torch.float16, device="cpu", seed=0, chunk_rows=1 << 20,
                     return_labels=False):
    """X[B,N,d] drawn from an isotropic Gaussian mixture (one mixture per batch).

    Rows are generated in chunks so that the fp32 temporaries stay bounded. With
    ``return_labels`` the component each point was drawn from is returned too (int32 [B,N]):
    a draw of the generator, not a clustering.
    """
    g = _gen(device, seed)
    X = torch.empty((B, N, d), dtype=dtype, device=device)
    labels = torch.empty((B, N), dtype=torch.int32, device=device) if return_labels else None
    for b in range(B):
        if mean == "uniform":
            mu = lo + (hi - lo) * torch.rand((n_comp, d), generator=g, device=device)
        else:
            mu = torch.randn((n_comp, d), generator=g, device=device)
        comp = _component_draw(N, mix, n_comp, g, device, zipf_s)
        if labels is not None:
            labels[b] = comp.to(torch.int32)
        for s in range(0, N, chunk_rows):
            e = min(N, s + chunk_rows)
            rows = mu[comp[s:e]]
            rows.add_(torch.randn((e - s, d), generator=g, device=device), alpha=sigma)
            X[b, s:e] = rows.to(dtype)
    return (X, labels) if return_labels else X


def student_t_rows(B, N, nu=5, scale=0.02, *, dtype=torch.float16, device="cpu", seed=0):
    """X[B,N,1]: Student-t(nu) * scale, built as Z / sqrt(chi2_nu / nu) with integer nu."""
    g = _gen(device, seed)
    X = torch.empty((B, N, 1), dtype=dtype, device=device)
    rows_per = max(1, (1 << 22) // max(N, 1))
    for s in range(0, B, rows_per):
        e = min(B, s + rows_per)
        z = torch.randn((e - s, N), generator=g, device=device)
        chi2 = torch.zeros_like(z)
        for _ in range(nu):
            chi2.add_(torch.randn((e - s, N), generator=g, device=device).square())
        X[s:e, :, 0] = (z / torch.sqrt(chi2 / nu) * scale).to(dtype)
    return X


def importance_weights(B, N, *, device="cpu", seed=0):
    """w[B,N] = Z^2 + 1e-3 (fp32), a positive per-point weight."""
    g = _gen(device, seed)
    z = torch.randn((B, N), generator=g, device=device)
    return z.square() + 1e-3


def pick_init_points(X, K, mode, *, seed=0):
    """Initial centroids C0[B,K,d] (fp32) chosen among the points of each batch.

    ``shuffle_first``: the first K points after a seeded shuffle of the batch.
    ``random_points``: K distinct points drawn at random (without replacement).
    Both are a seeded permutation of the point indices; they differ only in
    the seed stream used. The values are the points' own (exact) values.
    """
    B, N, d = X.shape
    if K > N:
        raise ValueError("K > N: cannot pick K distinct points")
    g = _gen(X.device, seed + (0 if mode == "shuffle_first" else 7919))
    C0 = torch.empty((B, K, d), dtype=torch.float32, device=X.device)
    for b in range(B):
        perm = torch.randperm(N, generator=g, device=X.device)[:K]
        C0[b] = X[b, perm].float()
    return C0


def make_workload(idx, *, device="cpu", seed=None, B=None, N=None, K=None, labels=False):
    """Build inputs for workload ``idx`` (1..5), optionally shrunk along B and N.

    Returns a dict with X, w (or None), C0 (fp32, or None for grid init),
    K, iters and the Workload record. The shrunk variants keep the recipe
    (distribution, d, dtype, K unless overridden) and change only sizes.
    With ``labels`` (mixture workloads) the dict also holds "labels": the component index
    each point was drawn from (int32 [B,N]); the same seed gives the same X either way.
    """
    wl = WORKLOADS[idx]
    seed = 1234 + idx if seed is None else seed
    B = wl.B if B is None else B
    N = wl.N if N is None else N
    K = wl.K[0] if K is None else K
    ex = wl.extra
    w = None
    lab = None
    if idx == 2:
        X = student_t_rows(B, N, ex["nu"], ex["scale"], dtype=wl.dtype, device=device, seed=seed)
        w = importance_weights(B, N, device=device, seed=seed + 1)
        C0 = None
    else:
        X = gaussian_mixture(B, N, wl.d, ex["n_comp"], ex["sigma"], mean=ex["mean"],
                             lo=ex.get("lo", -5.0), hi=ex.get("hi", 5.0), mix=ex.get("mix", "equal"),
                             zipf_s=ex.get("zipf_s", 1.1), dtype=wl.dtype, device=device, seed=seed,
                             return_labels=labels)
        if labels:
            X, lab = X
        C0 = pick_init_points(X, K, wl.init, seed=seed + 2)
    out = {"X": X, "w": w, "C0": C0, "K": K, "iters": wl.iters, "workload": wl,
           "B": B, "N": N, "d": wl.d}
    if labels:
        out["labels"] = lab
    return out


def describe(idx):
    wl = WORKLOADS[idx]
    return (f"{wl.name}: B={wl.B} N={wl.N} d={wl.d} K={'/'.join(map(str, wl.K))} "
            f"{str(wl.dtype).replace('torch.', '')}, {wl.recipe}; init={wl.init}; {wl.iters} iterations")


def nbytes_estimate(idx):
    wl = WORKLOADS[idx]
    return wl.B * wl.N * wl.d * torch.tensor([], dtype=wl.dtype).element_size()

