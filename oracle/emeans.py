"""CPU oracle for e-means and dead-cluster splitting: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg import this
module; the product path never does. Arithmetic in fp64 (numpy), the assignment through the C
oracle's exact argmin (``oracle.assign``) against centroids rounded to the points' dtype.

What the method computes follows the steinslab daily on e-means ("Beating 25 Lloyd Iterations
in 2 Epochs"):
* section "Breaking 70 Years of Full-Batch Inertia...": every cluster keeps a sum vector S_j and
  a count N_j whose quotient is the centroid; instead of resetting them every pass, each
  mini-batch's own per-cluster sum s_j (and count n_j) enters an exponential moving average
  S_j <- (1 - alpha) S_j + alpha s_j;
* section "Mini-Batch Stochastic Noise...": alpha follows a cosine decay from alpha0 to
  0.1 alpha0 over the run;
* section "Matching 25 Iterations...": after the last epoch the centroids are moved to the
  empirical mean of that epoch;
* section "Proportional Splitting Resurrects Thousands of Dead Centers": a centroid left without
  points is revived by splitting a large cluster, donors drawn in proportion to cluster size.

Readings where the page leaves a step open (each is listed with the design notes):
* the count gets the same average as the sum, N_j <- (1 - alpha) N_j + alpha n_j, and the
  centroid is S_j / N_j (a cluster with no points in a batch keeps its centroid: both decay);
* state starts at S_j = C0_j, N_j = 1;
* mini-batches are consecutive ranges of `batch` points in the order given (the caller shuffles);
  step t of T = epochs * ceil(N / batch) uses
  alpha_t = alpha0 * (0.1 + 0.9 * (1 + cos(pi * t / T)) / 2);
* with weights, s_j = sum w x and n_j = sum w over the batch's points of cluster j;
* "empirical mean of the final epoch" = per cluster, the (weighted) mean of the points the final
  epoch assigned to it, each labelled when its batch was processed; clusters the final epoch
  left empty keep their centroid;
* dead = a cluster that received no point during an epoch; splitting runs between epochs (not
  after the last one), dead clusters in index order, each drawing its donor with its own uniform
  u (an input): the first j whose running size sum exceeds u * (total size); the donor's size,
  its average count N and (through C * N) its sum are halved between the two; the centroids
  become c_dead = c_donor * (1 + eps * s_k), c_donor = c_donor * (1 - eps * s_k) per coordinate
  k, with s_k = +1 for even k and -1 for odd k. Sizes are the epoch's point counts (weights
  sums when weighted).
"""
from __future__ import annotations

import numpy as np

from . import as_f64, assign, round_to_dtype


def alpha_schedule(T, alpha0):
    """Step sizes alpha_0..alpha_{T-1} of the cosine decay from alpha0 towards 0.1 * alpha0."""
    t = np.arange(T, dtype=np.float64)
    return alpha0 * (0.1 + 0.9 * (1.0 + np.cos(np.pi * t / T)) / 2.0)


def batch_stats(X, ids, K, w=None):
    """Per-cluster sums s [B,K,d] and sizes n [B,K] (point counts, or weight sums) of a batch."""
    X = as_f64(X)
    B, n, d = X.shape
    s = np.zeros((B, K, d))
    cnt = np.zeros((B, K))
    for b in range(B):
        wb = np.ones(n) if w is None else as_f64(w)[b]
        np.add.at(s[b], ids[b], wb[:, None] * X[b])
        np.add.at(cnt[b], ids[b], wb)
    return s, cnt


def ema_update(S, Ncnt, C, s, n, alpha):
    """One moving-average step of the sums and counts; returns (S, Ncnt, C)."""
    S = (1.0 - alpha) * S + alpha * s
    Ncnt = (1.0 - alpha) * Ncnt + alpha * n
    C = np.where((Ncnt > 0)[..., None], S / np.where(Ncnt > 0, Ncnt, 1.0)[..., None], C)
    return S, Ncnt, C


def split_dead(C, sizes, u, eps, Ncnt=None):
    """Revive the clusters with size 0 by proportional splitting (one problem, C [K,d]).

    Returns (C, sizes, Ncnt, donors) with donors[i] = the donor of dead cluster i (-1 if alive).
    """
    C = np.array(C, dtype=np.float64)
    sizes = np.array(sizes, dtype=np.float64)
    Ncnt = None if Ncnt is None else np.array(Ncnt, dtype=np.float64)
    K, d = C.shape
    sign = np.where(np.arange(d) % 2 == 0, 1.0, -1.0)
    donors = np.full(K, -1, np.int64)
    for i in range(K):
        if sizes[i] != 0:
            continue
        total = sizes.sum()
        if total <= 0:
            break
        target = u[i] * total
        run = 0.0
        j = -1
        for k in range(K):
            run += sizes[k]
            if run > target:
                j = k
                break
        if j < 0:   # rounding left the target at the total: the last cluster with mass
            j = int(np.nonzero(sizes > 0)[0][-1])
        donors[i] = j
        cj = C[j].copy()
        C[i] = cj * (1.0 + eps * sign)
        C[j] = cj * (1.0 - eps * sign)
        sizes[i] = sizes[j] / 2.0
        sizes[j] -= sizes[i]
        if Ncnt is not None:
            Ncnt[i] = Ncnt[j] / 2.0
            Ncnt[j] -= Ncnt[i]
    return C, sizes, Ncnt, donors


def fit(X, C0, batch, epochs, alpha0, w=None, split_u=None, eps=1.0 / 1024, assign_dtype=None):
    """The whole e-means run. Returns dict(C, sse_hist [epochs,B], C_epochs [epochs,B,K,d]
    (centroids after each epoch's last step and splitting), sizes_last [B,K], donors [epochs,B,K]).
    """
    X = as_f64(X)
    w = None if w is None else as_f64(w)
    B, N, d = X.shape
    C = as_f64(C0).copy()
    K = C.shape[1]
    steps = -(-N // batch)
    alphas = alpha_schedule(epochs * steps, alpha0)
    S = C.copy()
    Ncnt = np.ones((B, K))
    sse = np.zeros((epochs, B))
    C_epochs = []
    donors_all = np.full((epochs, B, K), -1, np.int64)
    eS = eN = None
    for e in range(epochs):
        eS = np.zeros((B, K, d))
        eN = np.zeros((B, K))
        for st in range(steps):
            lo, hi = st * batch, min(N, (st + 1) * batch)
            Xb = X[:, lo:hi]
            wb = None if w is None else w[:, lo:hi]
            ids, _, _, inertia = assign(Xb, round_to_dtype(C, assign_dtype), wb)
            sse[e] += inertia
            s, n = batch_stats(Xb, ids, K, wb)
            S, Ncnt, C = ema_update(S, Ncnt, C, s, n, alphas[e * steps + st])
            eS += s
            eN += n
        if split_u is not None and e < epochs - 1:
            for b in range(B):
                C[b], _, Ncnt[b], donors_all[e, b] = split_dead(C[b], eN[b], split_u[e, b], eps,
                                                                Ncnt[b])
                S[b] = C[b] * Ncnt[b][:, None]
        C_epochs.append(C.copy())
    if epochs:
        C = np.where((eN > 0)[..., None], eS / np.where(eN > 0, eN, 1.0)[..., None], C)
    return {"C": C, "sse_hist": sse, "C_epochs": np.array(C_epochs), "sizes_last": eN,
            "donors": donors_all}
