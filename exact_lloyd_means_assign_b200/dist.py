"""Multi-GPU Lloyd iterations: one process per GPU, ``torch.distributed`` for the exchange.

The pages describe a single-GPU method; how it splits over ranks follows from the iteration
itself (the Lloyd recap in the technologypulse.uk Flash-KMeans article and the steinslab e-means
daily: the assignment is independent per point and the update is a per-cluster sum divided by a
count). Two ways:

* Batch sharding. Every batch element is an independent k-means problem, so each rank owns a
  contiguous range of whole problems and runs the full iteration on it. There is no exchange
  at all; ``batch_shard`` gives the range.
* Point sharding (one large problem). Each rank holds a contiguous slice of the points and a
  replica of the centroids. It assigns its slice and forms partial per-cluster sums, weight
  sums and counts; one all-reduce of those partials (K * (d + 1) fp32 values plus K int32
  counts per problem, a few MB at most) makes every rank hold the global statistics, and every
  rank then runs the same divide on the same reduced bits, so the replicas stay identical
  without a broadcast.

The device work is done by the library's kernels through ``LibraryOps``. The functions here
only slice, reduce and call; the operations are passed in so the exchange logic can be
exercised by CPU process groups with any implementation of the same four calls.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import km_assign, km_finalize, km_prep, km_update_partial


def _block(n: int, rank: int, world: int) -> tuple[int, int]:
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if n < 0:
        raise ValueError("negative extent")
    q, r = divmod(n, world)
    start = rank * q + min(rank, r)
    return start, start + q + (1 if rank < r else 0)


def point_shard(N: int, rank: int, world: int) -> tuple[int, int]:
    """[start, stop) of the points rank ``rank`` owns: contiguous, sizes differ by at most one."""
    return _block(N, rank, world)


def batch_shard(B: int, rank: int, world: int) -> tuple[int, int]:
    """[start, stop) of the problems rank ``rank`` owns (may be empty when B < world)."""
    return _block(B, rank, world)


class LibraryOps:
    """The four device calls of a point-sharded iteration, on the library's CUDA kernels."""

    def __init__(self, stream=None):
        self.stream = stream

    def assign(self, X, C, w):
        Cx, cn = km_prep(C, X.dtype, stream=self.stream)
        ids, _, inertia = km_assign(X, Cx, cn, w=w, want_inertia=True, stream=self.stream)
        return ids, inertia

    def partial(self, X, ids, K, w):
        sums, wsum, counts = km_update_partial(X, ids, K, w=w, stream=self.stream)
        if wsum is None:
            wsum = counts.to(torch.float32)
        return sums, wsum, counts

    def finalize(self, sums, wsum, counts, C_prev, weighted):
        C_new, _, _ = km_finalize(sums, counts, C_prev, wsum=wsum if weighted else None,
                                  stream=self.stream)
        return C_new


def lloyd_step_point_sharded(X_local, C, w_local=None, group=None, ops=None):
    """One exact Lloyd iteration over points split across the ranks of ``group``.

    X_local [B, n_r, d]: this rank's slice of the points (``point_shard``); C [B, K, d] fp32:
    the centroids, identical on every rank; w_local [B, n_r] or None: the slice's weights.
    Returns (C_new, ids_local, inertia) where inertia [B] fp64 is the global objective of the
    assignment made with C, and C_new is identical on every rank (empty clusters keep C).
    Every rank must call this the same number of times, in the same order.
    """
    ops = ops or LibraryOps()
    B, K, d = C.shape
    if X_local.shape[0] != B or X_local.shape[2] != d:
        raise ValueError("X_local and C disagree on B or d")
    ids, inertia = ops.assign(X_local, C, w_local)
    sums, wsum, counts = ops.partial(X_local, ids, K, w_local)
    # One fp32 buffer for the sums and weight sums, one int32 buffer for the counts (exact),
    # one fp64 value per problem for the objective.
    flat = torch.cat([sums.reshape(-1).to(torch.float32), wsum.reshape(-1).to(torch.float32)])
    counts = counts.to(torch.int32).contiguous()
    inertia = inertia.to(torch.float64).contiguous()
    dist.all_reduce(flat, group=group)
    dist.all_reduce(counts, group=group)
    dist.all_reduce(inertia, group=group)
    sums = flat[: B * K * d].view(B, K, d)
    wsum = flat[B * K * d:].view(B, K)
    C_new = ops.finalize(sums, wsum, counts, C, w_local is not None)
    return C_new, ids, inertia


def fit_point_sharded(X_local, C0, iters, w_local=None, group=None, ops=None):
    """``iters`` point-sharded iterations from C0. Returns (C, inertia_hist [iters, B])."""
    C = C0.clone()
    hist = []
    for _ in range(iters):
        C, _, inertia = lloyd_step_point_sharded(X_local, C, w_local, group=group, ops=ops)
        hist.append(inertia)
    return C, torch.stack(hist) if hist else torch.empty((0, C0.shape[0]), dtype=torch.float64)
