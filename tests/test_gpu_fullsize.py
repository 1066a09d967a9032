"""Full-size workloads on the GPU, in the launch configuration the benchmark times.

The oracle cannot evaluate B*N*K*d fp64 assignment work at these sizes in seconds, so the
assignment is checked on a large seeded sample of points (each one against every centroid, by
the oracle). The update is checked for every point: the oracle's update fed the GPU's own
assignment, chunk by chunk for the 8.6 GB workload. The full-size objective is checked against
the oracle's distance of every point to the centroid the kernel chose.
"""
import numpy as np
import pytest
import torch

import exact_lloyd_means_assign_b200 as km
import oracle
import synth
from parity import check_assign, oracle_inertia_of, oracle_update_chunked, to_np

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


# sampled points per workload for the assignment check (the oracle's time grows with K)
ASSIGN_SAMPLE = {3: 65536, 4: 65536, 5: 262144}


@pytest.mark.parametrize("idx", [3, 4, 5])
def test_full_size_iteration_against_oracle(idx, cuda_device):
    """One Lloyd iteration of a full-size workload in the benchmark's launch configuration:
    the assignment on a large seeded sample of points (each against every centroid, by the
    oracle), the update of every point through the oracle (fed the GPU's own assignment: counts
    exact, centroids within 1e-3 relative per problem and per cluster, empty clusters unchanged),
    and the full-size objective against the oracle's distances to the assigned centroids."""
    d = synth.make_workload(idx, device=cuda_device)
    X, C = d["X"], d["C0"]
    B, N, dd = X.shape
    K = C.shape[1]
    Cx, cn = km.km_prep(C, X.dtype)
    assert km.km_assign_uses_tensor_cores(X, Cx)
    ids, mind, inertia = km.km_assign(X, Cx, cn, want_mind=True, want_inertia=True)
    C_new, counts, _ = km.km_update(X, ids, C)
    torch.cuda.synchronize()
    # assignment: a seeded sample, each point against the full centroid set, exactly
    m = ASSIGN_SAMPLE[idx]
    rows = _sample_rows(B, N, m, seed=idx)
    near = check_assign(X, C, ids, mind_gpu=mind, rows=rows)
    print(f"workload {idx}: {m} sampled points, 0 mismatches outside near-ties, {near} near-ties")
    assert near <= 0.03 * m      # near-ties may differ; they remain a small minority
    # update: every point, through the oracle, on the GPU's assignment
    C_ref, cnt_ref = oracle_update_chunked(X, ids, C)
    np.testing.assert_array_equal(to_np(counts), cnt_ref)
    assert int(counts.sum()) == B * N
    Cg = oracle.as_f64(C_new.cpu())
    for b in range(B):
        assert np.linalg.norm(Cg[b] - C_ref[b]) <= 1e-3 * np.linalg.norm(C_ref[b])
    per = np.linalg.norm(Cg - C_ref, axis=-1)
    scale = np.maximum(np.linalg.norm(C_ref, axis=-1), 1e-3 * np.linalg.norm(C_ref, axis=-1).mean())
    worst = np.unravel_index(np.argmax(per / scale), per.shape)
    assert (per <= 1e-3 * scale).all(), f"cluster {worst}: {per[worst] / scale[worst]:.2e}"
    empty = cnt_ref == 0
    np.testing.assert_array_equal(Cg[empty], oracle.as_f64(C.cpu())[empty])
    print(f"workload {idx}: largest cluster {cnt_ref.max()} of {N} points, {int(empty.sum())} empty")
    # objective: the kernel's full-size inertia against the oracle's distances to the clusters
    # the kernel chose (this is the inertia of the assignment being checked)
    ref_in = oracle_inertia_of(X, ids, C, X.dtype)
    np.testing.assert_allclose(to_np(inertia), ref_in, rtol=1e-4, atol=0)
    np.testing.assert_allclose(to_np(inertia), to_np(mind.double().sum(1)), rtol=1e-6)


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
