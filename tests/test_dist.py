"""Multi-process (gloo, world size 2, CPU) tests of the point- and batch-sharded iteration.

The device calls are replaced by plain numpy / oracle implementations of the same four
operations, so what is tested here is the exchange: slicing, the all-reduce of the partial
statistics and the identical divide on every rank. The result must equal one iteration of the
oracle over all points in one process.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from exact_lloyd_means_assign_b200 import dist as kdist


def test_point_shard_covers_every_point_once():
    for n in [0, 1, 7, 64, 65537]:
        for world in [1, 2, 3, 8]:
            spans = [kdist.point_shard(n, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1


def test_batch_shard_and_bad_ranks():
    assert [kdist.batch_shard(32, r, 8) for r in range(8)] == [(4 * r, 4 * r + 4) for r in range(8)]
    assert kdist.batch_shard(1, 1, 2) == (1, 1)          # fewer problems than ranks: empty
    for bad in [(5, 2, 2), (5, -1, 2), (5, 0, 0)]:
        with pytest.raises(ValueError):
            kdist.point_shard(*bad)


class OracleOps:
    """The four calls of an iteration in fp64 numpy (oracle assignment, np.add.at sums)."""

    def assign(self, X, C, w):
        ids, _, _, inertia = oracle.assign(X, C, w)
        return torch.from_numpy(ids), torch.from_numpy(np.asarray(inertia, dtype=np.float64))

    def partial(self, X, ids, K, w):
        X = oracle.as_f64(X)
        B, n, d = X.shape
        ids = ids.numpy()
        wt = np.ones((B, n)) if w is None else oracle.as_f64(w)
        sums = np.zeros((B, K, d))
        wsum = np.zeros((B, K))
        counts = np.zeros((B, K), dtype=np.int32)
        for b in range(B):
            np.add.at(sums[b], ids[b], X[b] * wt[b][:, None])
            np.add.at(wsum[b], ids[b], wt[b])
            np.add.at(counts[b], ids[b], 1)
        return torch.from_numpy(sums), torch.from_numpy(wsum), torch.from_numpy(counts)

    def finalize(self, sums, wsum, counts, C_prev, weighted):
        div = wsum if weighted else counts.to(torch.float64)
        upd = (counts > 0) & (div > 0)
        out = torch.where(upd[..., None], sums.double() / torch.where(upd, div.double(), 1.0)[..., None],
                          C_prev.double())
        return out.to(torch.float32)


def _problem(weighted):
    g = np.random.default_rng(1234)
    B, N, K, d = 2, 1001, 9, 5          # odd N: the two slices differ in size
    X = g.normal(size=(B, N, d)) + 4.0 * g.integers(0, 3, size=(B, N, 1))
    C = g.normal(size=(B, K, d)).astype(np.float32)
    C[:, -1] = 1e3                      # a centroid no point is nearest to: stays where it is
    w = g.uniform(0.1, 2.0, size=(B, N)).astype(np.float32) if weighted else None
    return X, C, w


def _worker(rank, world, port, out_dir, weighted):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        X, C, w = _problem(weighted)
        s0, s1 = kdist.point_shard(X.shape[1], rank, world)
        Xl = torch.from_numpy(X[:, s0:s1].copy())
        wl = None if w is None else torch.from_numpy(w[:, s0:s1].copy())
        Cn, ids, inertia = kdist.lloyd_step_point_sharded(Xl, torch.from_numpy(C), wl, ops=OracleOps())
        C2, hist = kdist.fit_point_sharded(Xl, torch.from_numpy(C), 3, wl, ops=OracleOps())
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), C=Cn.numpy(), ids=ids.numpy(),
                 inertia=inertia.numpy(), C3=C2.numpy(), hist=hist.numpy())
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("weighted", [False, True])
def test_point_sharded_step_equals_one_process_oracle(tmp_path, weighted):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path), weighted), nprocs=world, join=True)
    r = [np.load(tmp_path / f"r{k}.npz") for k in range(world)]
    X, C, w = _problem(weighted)
    ids, _, _, inertia = oracle.assign(X, C, w)
    C_ref, counts, _ = oracle.update(X, ids, C, w)
    assert counts[:, -1].sum() == 0
    # every rank holds the same centroids, equal to the one-process update
    np.testing.assert_array_equal(r[0]["C"], r[1]["C"])
    np.testing.assert_allclose(r[0]["C"], C_ref, rtol=1e-6, atol=1e-6)
    np.testing.assert_array_equal(r[0]["C"][:, -1], C[:, -1])
    # the slices' assignments concatenate to the full one; the objective is global
    np.testing.assert_array_equal(np.concatenate([r[0]["ids"], r[1]["ids"]], axis=1), ids)
    np.testing.assert_allclose(r[0]["inertia"], inertia, rtol=1e-12)
    np.testing.assert_array_equal(r[0]["inertia"], r[1]["inertia"])
    # three iterations: monotone objective, same as three one-process oracle iterations
    ref = oracle.fit(X, C, 3, w)
    np.testing.assert_allclose(r[0]["C3"], ref["C_hist"][-1], rtol=1e-5, atol=1e-5)
    # the sharded step keeps C in fp32 between iterations, the oracle in fp64: the objective
    # of later iterations differs by the fp32 rounding of the centroids (~1e-8 relative)
    np.testing.assert_allclose(r[0]["hist"], ref["inertia_hist"], rtol=1e-6)
    assert np.all(np.diff(r[0]["hist"], axis=0) <= 1e-9 * r[0]["hist"][:-1])


def test_mismatched_shapes_are_rejected():
    with pytest.raises(ValueError):
        kdist.lloyd_step_point_sharded(torch.zeros(2, 5, 3), torch.zeros(1, 4, 3), ops=OracleOps())
