"""Full-size workloads on the GPU, in the launch configuration the benchmark times.

The oracle cannot evaluate B*N*K*d fp64 work at these sizes in seconds, so the assignment is
checked on sampled points (each one computed exactly by the oracle), the counts are checked for
every cluster against a host bincount of the GPU's assignment, and centroids are checked for
sampled clusters (the largest included) against the fp64 mean of their members.
"""
import numpy as np
import pytest
import torch

import exact_lloyd_means_assign_b200 as km
import oracle
import synth
from parity import check_assign, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    torch.cuda.set_device(cuda_device)
    yield
    torch.cuda.empty_cache()
    assert km.km_device_error() == 0


def _sample_rows(B, N, m, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(0, B, (m,), generator=g), torch.randint(0, N, (m,), generator=g)


def _check_centroids(X, ids, C_prev, C_new, counts, clusters, b=0):
    """Each sampled non-empty cluster's centroid is the fp64 mean of its members."""
    idb = ids[b]
    for k in clusters:
        k = int(k)
        members = torch.nonzero(idb == k).flatten()
        assert members.numel() == int(counts[b, k])
        if members.numel() == 0:
            assert torch.equal(C_new[b, k], C_prev[b, k])
            continue
        s = np.zeros(X.shape[-1], np.float64)
        for c0 in range(0, members.numel(), 1 << 19):
            s += X[b, members[c0:c0 + (1 << 19)]].double().sum(0).cpu().numpy()
        ref = s / members.numel()
        got = C_new[b, k].double().cpu().numpy()
        assert np.linalg.norm(got - ref) <= 1e-3 * max(np.linalg.norm(ref), 1e-30), k


@pytest.mark.parametrize("idx", [3, 4, 5])
def test_one_full_iteration(idx, cuda_device):
    d = synth.make_workload(idx, device=cuda_device)
    X, C = d["X"], d["C0"]
    B, N, dd = X.shape
    K = C.shape[1]
    Cx, cn = km.km_prep(C, X.dtype)
    assert km.km_assign_uses_tensor_cores(X, Cx)
    ids, mind, inertia = km.km_assign(X, Cx, cn, want_mind=True, want_inertia=True)
    C_new, counts, _ = km.km_update(X, ids, C)
    torch.cuda.synchronize()
    # assignment: sampled points, each against the full centroid set, exactly
    m = 1024 if idx == 5 else 2048
    rows = _sample_rows(B, N, m, seed=idx)
    near = check_assign(X, C, ids, mind_gpu=mind, rows=rows)
    assert near <= 0.03 * m      # near-ties may differ; they remain a small minority
    # counts: every cluster, from the GPU's own assignment
    ids_h = to_np(ids)
    for b in range(B):
        np.testing.assert_array_equal(to_np(counts[b]), np.bincount(ids_h[b], minlength=K))
    assert int(counts.sum()) == B * N
    # inertia = sum of the reported per-point distances
    np.testing.assert_allclose(to_np(inertia), to_np(mind.double().sum(1)), rtol=1e-6)
    # centroids: sampled clusters plus the largest one, per checked batch
    for b in ([0, B - 1] if B > 1 else [0]):
        cb = to_np(counts[b])
        g = np.random.default_rng(idx + b)
        pick = set(g.choice(K, 24, replace=False).tolist()) | {int(cb.argmax())}
        if (cb == 0).any():
            pick.add(int(np.flatnonzero(cb == 0)[0]))
        _check_centroids(X, ids, C, C_new, counts, sorted(pick), b=b)


def test_full_batch_update_against_oracle(cuda_device):
    """Workload 3 at full N for two batches: the whole update against the oracle."""
    d = synth.make_workload(3, B=2, device=cuda_device)
    X, C = d["X"], d["C0"]
    Cx, cn = km.km_prep(C, X.dtype)
    ids, _, _ = km.km_assign(X, Cx, cn)
    C_new, counts, _ = km.km_update(X, ids, C)
    torch.cuda.synchronize()
    C_ref, cnt_ref, _ = oracle.update(oracle.as_f64(X.cpu()), to_np(ids), oracle.as_f64(C.cpu()))
    np.testing.assert_array_equal(to_np(counts), cnt_ref)
    for b in range(2):
        err = np.linalg.norm(to_np(C_new[b]) - C_ref[b]) / np.linalg.norm(C_ref[b])
        assert err <= 1e-3


def test_rows_workload_full_size(cuda_device):
    """Workload 2 at full size (4096 weighted rows, K=16): the fused per-row fit."""
    d = synth.make_workload(2, device=cuda_device)
    X, w = d["X"], d["w"]
    C = km.km_init_grid1d(X, 16)
    _, ids, ih, ch = km.km_fit(X, C, 30, w=w, want_ids=True, want_inertia=True, want_hist=True)
    torch.cuda.synchronize()
    # sampled rows, every iteration, against the oracle from the same centroids
    rows = np.random.default_rng(2).choice(X.shape[0], 16, replace=False)
    X64 = oracle.as_f64(X[rows].cpu())
    w64 = oracle.as_f64(w[rows].cpu())
    hist = to_np(ch[:, rows]).astype(np.float64)
    for t in range(30):
        ids_t, _, _, inertia = oracle.assign(X64, oracle.round_to_dtype(hist[t], torch.float16), w64)
        np.testing.assert_allclose(to_np(ih[t])[rows], inertia, rtol=1e-4)
        C_ref, _, _ = oracle.update(X64, ids_t, hist[t], w64)
        for j in range(len(rows)):
            assert np.linalg.norm(hist[t + 1][j] - C_ref[j]) <= 1e-3 * np.linalg.norm(C_ref[j])
    check_assign(X[rows], C[rows], ids[rows], w=w[rows])
