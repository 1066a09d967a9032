"""Shared helpers for the GPU-vs-oracle parity tests (not a test module).

Tolerances (fixed by the specification of this path):
  ids / counts   bit-exact, except points whose best and second-best squared distances (oracle,
                 fp64, against the centroids rounded to the points' dtype) differ by less than
                 1e-3 relative; those are counted and reported.
  centroids      per batch ||C_gpu - C_ref||_F / ||C_ref||_F <= 1e-3
  inertia        relative error <= 1e-4 per batch
"""
import numpy as np
import torch

import oracle

CENTROID_RTOL = 1e-3
INERTIA_RTOL = 1e-4


def to_np(t):
    return t.detach().cpu().numpy()


def check_assign(X, C32, ids_gpu, *, w=None, mind_gpu=None, inertia_gpu=None, dtype=None,
                 rows=None):
    """Compare a GPU assignment with the oracle. ``rows`` restricts to sampled (b, i) pairs.

    Returns the number of near-tie points (allowed to differ).
    """
    dtype = X.dtype if dtype is None else dtype
    Cr = oracle.round_to_dtype(C32.detach().cpu(), dtype)
    if rows is not None:
        bsel, isel = to_np(rows[0]), to_np(rows[1])
        nnear = 0
        for b in np.unique(bsel):
            ii = isel[bsel == b]
            Xs = oracle.as_f64(X[int(b), torch.as_tensor(ii, device=X.device)].cpu())[None]
            ids, d1, d2, _ = oracle.assign(Xs, Cr[int(b)][None], None)
            ids, d1, d2 = ids[0], d1[0], d2[0]
            g = to_np(ids_gpu[int(b)])[ii]
            near = oracle.near_tie(d1, d2)
            bad = (g != ids) & ~near
            assert not bad.any(), f"batch {b}: {bad.sum()} non-near-tie mismatches of {len(g)}"
            if mind_gpu is not None:
                m = to_np(mind_gpu[int(b)])[ii].astype(np.float64)
                scale = (Xs[0] ** 2).sum(-1) + (Cr[int(b)][ids] ** 2).sum(-1) + 1e-30
                ok = np.abs(m - d1) <= 1e-5 * scale + 1e-6 * np.abs(d1)
                assert ok[g == ids].all()
            nnear += int(near.sum())
        return nnear
    X64 = oracle.as_f64(X.cpu())
    w64 = None if w is None else oracle.as_f64(w.cpu())
    ids, d1, d2, inertia = oracle.assign(X64, Cr, w64)
    g = to_np(ids_gpu)
    near = oracle.near_tie(d1, d2)
    bad = (g != ids) & ~near
    assert not bad.any(), f"{bad.sum()} non-near-tie mismatches of {g.size}"
    if mind_gpu is not None:
        m = to_np(mind_gpu).astype(np.float64)
        cn = (Cr ** 2).sum(-1)
        scale = (X64 ** 2).sum(-1) + np.take_along_axis(cn, ids, 1) + 1e-30
        ok = np.abs(m - d1) <= 1e-5 * scale + 1e-6 * np.abs(d1)
        assert ok[g == ids].all(), f"mind off at {(~ok & (g == ids)).sum()} points"
    if inertia_gpu is not None:
        gi = to_np(inertia_gpu)
        np.testing.assert_allclose(gi, inertia, rtol=INERTIA_RTOL, atol=0)
    return int(near.sum())


def check_update(X, ids_gpu, C_prev, C_new_gpu, counts_gpu, *, w=None, wsum_gpu=None):
    """The GPU update fed the GPU's ids: counts exact, centroids within the relative L2 bound."""
    X64 = oracle.as_f64(X.cpu())
    w64 = None if w is None else oracle.as_f64(w.cpu())
    C_ref, counts, wsum = oracle.update(X64, to_np(ids_gpu), oracle.as_f64(C_prev.cpu()), w64)
    np.testing.assert_array_equal(to_np(counts_gpu), counts)
    Cg = oracle.as_f64(C_new_gpu.cpu())
    for b in range(Cg.shape[0]):
        den = max(np.linalg.norm(C_ref[b]), 1e-30)
        assert np.linalg.norm(Cg[b] - C_ref[b]) / den <= CENTROID_RTOL
    empty = counts == 0
    if w64 is not None:
        empty |= wsum <= 0
    # empty clusters keep the previous centroid exactly
    np.testing.assert_array_equal(Cg[empty], oracle.as_f64(C_prev.cpu())[empty])
    if wsum_gpu is not None:
        np.testing.assert_allclose(to_np(wsum_gpu), wsum, rtol=1e-5, atol=1e-6)
    return C_ref


def oracle_update_chunked(X, ids, C_prev, chunk=1 << 21):
    """The oracle's update of all of X (on the device) fed the given assignment, chunk by chunk.

    Each chunk's per-cluster means and counts come from ``oracle.update``; the chunk's sums are
    rebuilt as mean x count (an fp64 rounding, 2^-52 relative) and added in fp64, so the
    whole-set means are the oracle's own, only regrouped. Returns (C_ref, counts)."""
    Bx, Nx, dx = X.shape
    Kx = C_prev.shape[1]
    C64 = oracle.as_f64(C_prev.cpu())
    S = np.zeros((Bx, Kx, dx))
    cnt = np.zeros((Bx, Kx), np.int64)
    for b in range(Bx):
        for s in range(0, Nx, chunk):
            Xc = oracle.as_f64(X[b:b + 1, s:s + chunk].cpu())
            Cc, nc, _ = oracle.update(Xc, to_np(ids[b:b + 1, s:s + chunk]), C64[b:b + 1])
            S[b] += Cc[0] * nc[0][:, None]
            cnt[b] += nc[0]
    nz = cnt > 0
    C_ref = C64.copy()
    C_ref[nz] = S[nz] / cnt[nz][:, None]
    return C_ref, cnt


def oracle_inertia_of(X, ids, C, dtype, chunk=1 << 21):
    """sum_i ||x_i - c_{ids_i}||^2 per batch element, every distance from the oracle: the
    points of each cluster are assigned against that one (rounded) centroid."""
    Bx, Nx, _ = X.shape
    Cr = oracle.round_to_dtype(C.cpu(), dtype)
    tot = np.zeros(Bx)
    for b in range(Bx):
        for s in range(0, Nx, chunk):
            Xc = oracle.as_f64(X[b, s:s + chunk].cpu())
            ic = to_np(ids[b, s:s + chunk])
            order = np.argsort(ic, kind="stable")
            ks, starts = np.unique(ic[order], return_index=True)
            ends = np.append(starts[1:], len(order))
            for k, a, e in zip(ks, starts, ends):
                _, _, _, inert = oracle.assign(Xc[order[a:e]][None], Cr[b, k][None, None])
                tot[b] += inert[0]
    return tot


def mixture(B, N, d, K, dtype, device, seed=0, sigma=0.3, c_noise=0.3):
    """Clustered points plus K initial centroids drawn among them (plus ``c_noise`` noise)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    ncomp = max(1, min(K, 64))
    mu = torch.randn((B, ncomp, d), generator=g)
    comp = torch.randint(0, ncomp, (B, N), generator=g)
    X = torch.gather(mu, 1, comp[..., None].expand(B, N, d)) + sigma * torch.randn((B, N, d), generator=g)
    idx = torch.stack([torch.randperm(N, generator=g)[:K] if K <= N else torch.randint(0, N, (K,), generator=g)
                       for _ in range(B)])
    C = torch.gather(X, 1, idx[..., None].expand(B, K, d)) + c_noise * torch.randn((B, K, d), generator=g)
    return X.to(dtype).to(device), C.float().to(device)
