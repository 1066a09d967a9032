"""CPU oracle for 1-D codebooks: encoding to uint8 indices and k-means++ seeding.
TEST INFRASTRUCTURE ONLY: imported by ``tests/`` (and nothing in the product path).

* Encoding follows the weight-clustering proposal reposted on wpnews.pro ("Cache-Aware Weight
  Clustering ...", the compressed-representation and 100-million-weight examples): every value
  is replaced by the index of its cluster's shared value, 8-bit indices for up to 256 values.
  The index is the exact nearest centroid (centroids rounded to the values' dtype, as every
  assignment here), lowest index on ties: the assignment stage of ``oracle.assign`` with d = 1.
* k-means++ seeding is what the LeanQuant issue "1D k-means" uses for rows with more than 8
  clusters (its ``KMeans(init=...)`` line): the first centre is drawn with probability
  proportional to the sample weight, each next one proportional to weight times the squared
  distance to the nearest centre chosen so far. Readings: the plain one-draw-per-centre form;
  each draw takes its uniform u (an input) and picks the first point whose running mass exceeds
  u * (total mass); when the total mass is 0 (every point sits on a chosen centre) the draw
  picks point 0.
"""
from __future__ import annotations

import numpy as np

from . import as_f64, assign, round_to_dtype


def encode1d(X, C, dtype=None):
    """X [B,N] values, C [B,K] centroids -> (codes [B,N] uint8, d1, d2) for K <= 256."""
    X = as_f64(X)
    C = as_f64(C)
    assert C.shape[1] <= 256
    ids, d1, d2, _ = assign(X[..., None], round_to_dtype(C[..., None], dtype))
    return ids.astype(np.uint8), d1, d2


def kmeanspp1d(X, K, u, w=None):
    """X [B,N] values, u [B,K] uniforms -> (C [B,K], chosen [B,K] point indices)."""
    X = as_f64(X)
    B, N = X.shape
    C = np.zeros((B, K))
    chosen = np.zeros((B, K), np.int64)
    for b in range(B):
        wb = np.ones(N) if w is None else as_f64(w)[b]
        D2 = np.ones(N)                      # first draw: proportional to the weights alone
        for k in range(K):
            mass = wb * D2
            total = mass.sum()
            i = 0
            if total > 0:
                run = np.cumsum(mass)
                hit = np.nonzero(run > u[b, k] * total)[0]
                i = int(hit[0]) if hit.size else int(np.nonzero(mass > 0)[0][-1])
            chosen[b, k] = i
            C[b, k] = X[b, i]
            D2 = np.minimum(D2 if k else np.full(N, np.inf), (X[b] - X[b, i]) ** 2)
    return C, chosen
