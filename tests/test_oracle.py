"""Pins for the CPU oracle (no GPU): each check ties the oracle to something other than itself.

- the forum worked example of weight clustering (printed cluster values);
- brute force over every labelling of tiny inputs (global optimum bounds, fixed points,
  contiguity of optimal 1-D clusters);
- an independent numpy evaluation of the full distance matrix (argmin, second best);
- np.average for weighted means, np.bincount for counts, np.linspace for the grid init
  (the routine the LeanQuant code calls);
- scikit-learn's Lloyd KMeans with sample weights;
- closed forms and invariances (K=1, K=N, duplicate centroids, weight scaling,
  permutations, monotone inertia).
"""
import itertools

import numpy as np
import pytest

import oracle
from conftest import load_golden

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _blobs(rng, B, N, K, d, spread=0.15):
    centers = rng.normal(size=(B, K, d)) * 3
    comp = rng.integers(0, K, size=(B, N))
    X = np.take_along_axis(centers, comp[:, :, None].repeat(d, 2), 1) + spread * rng.normal(size=(B, N, d))
    return X


# ---------------------------------------------------------------- worked example

def _worked():
    g = load_golden("worked_example_weight_clustering.txt")
    vals = np.array([float(v) for v in g["values"]])
    return g, vals


def test_worked_example_fp64():
    g, vals = _worked()
    K = int(g["K"][0])
    X = vals[None, :, None]
    C0 = oracle.grid_init(X, K)
    # linspace(-0.6213, 0.8130, 3)
    np.testing.assert_allclose(C0[0, :, 0], [-0.6213, 0.09585, 0.8130], rtol=0, atol=1e-15)
    out = oracle.fit(X, C0, iters=3)
    C = out["C_hist"][1][0, :, 0]
    printed = np.array([float(v) for v in g["centroids"]])
    half_unit = 0.5 * 10.0 ** (-int(g["decimals"][0]))
    # multiset comparison: the page's labels A/B/C are not tied to an init order
    np.testing.assert_allclose(np.sort(C), np.sort(printed), rtol=0, atol=half_unit)
    # the printed index vector of the first ten values: two groups of five, in that order
    lab = out["ids"][0, :10]
    exp = np.array([int(v) for v in g["labels_first10"]])
    assert len(set(lab[exp == 0])) == 1 and len(set(lab[exp == 1])) == 1
    assert lab[0] != lab[5]
    # already a fixed point after the first iteration
    np.testing.assert_array_equal(out["C_hist"][1], out["C_hist"][2])
    np.testing.assert_array_equal(out["C_hist"][2], out["C_hist"][3])
    assert out["inertia_hist"][1, 0] == pytest.approx(2.444e-6, rel=1e-3)


def test_worked_example_fp16_inputs():
    import torch
    g, vals = _worked()
    X16 = torch.tensor(vals, dtype=torch.float16).double().numpy()[None, :, None]
    C0 = oracle.grid_init(X16, 3)
    out = oracle.fit(X16, C0, iters=2, assign_dtype=torch.float16)
    printed = np.array([float(v) for v in g["centroids"]])
    # fp16 spacing near 0.8 is 2^-11; the means of rounded inputs stay within it of the print
    np.testing.assert_allclose(np.sort(out["C_hist"][-1][0, :, 0]), np.sort(printed), atol=2.0 ** -11)


# ---------------------------------------------------------------- independent full-matrix check

@pytest.mark.parametrize("B,N,K,d", [(2, 57, 7, 3), (1, 200, 16, 1), (3, 33, 5, 9)])
def test_assign_matches_full_distance_matrix(B, N, K, d):
    rng = _rng(B * 100 + d)
    X = rng.normal(size=(B, N, d))
    C = rng.normal(size=(B, K, d))
    w = rng.uniform(0.1, 2.0, size=(B, N))
    ids, d1, d2, inertia = oracle.assign(X, C, w)
    D = ((X[:, :, None, :] - C[:, None, :, :]) ** 2).sum(-1)       # [B,N,K]
    np.testing.assert_array_equal(ids, D.argmin(-1))
    Ds = np.sort(D, -1)
    np.testing.assert_allclose(d1, Ds[..., 0], rtol=1e-13, atol=0)
    np.testing.assert_allclose(d2, Ds[..., 1], rtol=1e-13, atol=0)
    np.testing.assert_allclose(inertia, (w * Ds[..., 0]).sum(1), rtol=1e-12)
    # the expanded form through a library matmul agrees away from near-ties
    Dm = (X ** 2).sum(-1)[:, :, None] + (C ** 2).sum(-1)[:, None, :] - 2 * np.einsum("bnd,bkd->bnk", X, C)
    far = ~oracle.near_tie(d1, d2)
    np.testing.assert_array_equal(ids[far], Dm.argmin(-1)[far])


def test_assign_K1_and_second_best_inf():
    X = _rng(1).normal(size=(1, 10, 2))
    C = np.zeros((1, 1, 2))
    ids, d1, d2, _ = oracle.assign(X, C)
    assert (ids == 0).all() and np.isinf(d2).all()
    np.testing.assert_allclose(d1[0], (X[0] ** 2).sum(-1), rtol=1e-14)


def test_duplicate_centroids_lowest_index():
    rng = _rng(2)
    X = rng.normal(size=(1, 300, 3))
    C = rng.normal(size=(1, 6, 3))
    C[0, 5] = C[0, 2]
    ids, d1, d2, _ = oracle.assign(X, C)
    assert not (ids == 5).any()
    assert (ids == 2).any()
    # a point whose nearest location is the duplicated one has d1 == d2 (tie over distinct k)
    assert (d1[ids == 2] == d2[ids == 2]).all()


# ---------------------------------------------------------------- update

def test_update_is_weighted_mean_and_keeps_empty():
    rng = _rng(3)
    B, N, K, d = 2, 120, 9, 4
    X = rng.normal(size=(B, N, d))
    w = rng.uniform(0.01, 3.0, size=(B, N))
    ids = rng.integers(0, K - 2, size=(B, N)).astype(np.int32)     # clusters K-2, K-1 empty
    C_prev = rng.normal(size=(B, K, d))
    C_new, counts, wsum = oracle.update(X, ids, C_prev, w)
    for b in range(B):
        np.testing.assert_array_equal(counts[b], np.bincount(ids[b], minlength=K))
        np.testing.assert_allclose(wsum[b], np.bincount(ids[b], weights=w[b], minlength=K), rtol=1e-13)
        assert counts[b].sum() == N
        for k in range(K):
            m = ids[b] == k
            if m.any():
                np.testing.assert_allclose(C_new[b, k], np.average(X[b, m], axis=0, weights=w[b, m]),
                                           rtol=1e-12, atol=1e-14)
            else:
                np.testing.assert_array_equal(C_new[b, k], C_prev[b, k])


def test_zero_weight_cluster_is_empty():
    X = np.array([[[1.0], [2.0], [10.0]]])
    w = np.array([[1.0, 1.0, 0.0]])
    ids = np.array([[0, 0, 1]], np.int32)
    C_prev = np.array([[[0.0], [7.0]]])
    C_new, counts, wsum = oracle.update(X, ids, C_prev, w)
    assert counts[0, 1] == 1 and wsum[0, 1] == 0.0
    assert C_new[0, 1, 0] == 7.0 and C_new[0, 0, 0] == 1.5


def test_k1_is_weighted_mean():
    rng = _rng(4)
    X = rng.normal(size=(3, 50, 5))
    w = rng.uniform(0.1, 1.0, size=(3, 50))
    out = oracle.fit(X, X[:, :1].copy(), iters=1, w=w)
    for b in range(3):
        np.testing.assert_allclose(out["C_hist"][1][b, 0], np.average(X[b], axis=0, weights=w[b]), rtol=1e-12)


def test_k_equals_n_fixed_point():
    rng = _rng(5)
    X = rng.normal(size=(1, 12, 3))
    out = oracle.fit(X, X.copy(), iters=2)
    np.testing.assert_array_equal(out["ids"][0], np.arange(12))
    np.testing.assert_array_equal(out["C_hist"][-1], X)
    assert out["inertia_hist"].max() == 0.0


def test_two_separated_clusters_1d_exact_means():
    X = np.array([[[-5.0], [-4.0], [-6.0], [3.0], [4.0], [5.0], [7.0]]])
    out = oracle.fit(X, np.array([[[-1.0], [1.0]]]), iters=3)
    np.testing.assert_allclose(out["C_hist"][-1][0, :, 0], [-5.0, 4.75], rtol=1e-15)


# ---------------------------------------------------------------- brute force

def _labelling_inertia(X, lab, K):
    s = 0.0
    for k in range(K):
        m = lab == k
        if m.any():
            s += ((X[m] - X[m].mean(0)) ** 2).sum()
    return s


@pytest.mark.parametrize("d", [1, 2])
def test_brute_force_optimum_bounds_lloyd(d):
    rng = _rng(10 + d)
    N, K = 7, 3
    X = rng.normal(size=(N, d))
    best, best_lab = np.inf, None
    for lab in itertools.product(range(K), repeat=N):
        lab = np.array(lab)
        if len(set(lab)) < K:
            continue
        v = _labelling_inertia(X, lab, K)
        if v < best - 1e-15:
            best, best_lab = v, lab
    # every Lloyd run ends at an inertia no better than the global optimum
    for s in range(20):
        init = X[rng.choice(N, K, replace=False)][None]
        out = oracle.fit(X[None], init, iters=25)
        assert out["final_inertia"][0] >= best - 1e-12
    # the optimum is a Lloyd fixed point of the oracle
    Copt = np.stack([X[best_lab == k].mean(0) for k in range(K)])[None]
    ids, _, _, inertia = oracle.assign(X[None], Copt)
    assert inertia[0] == pytest.approx(best, rel=1e-12)
    np.testing.assert_array_equal(ids[0], best_lab)
    C2, _, _ = oracle.update(X[None], ids, Copt)
    np.testing.assert_allclose(C2, Copt, rtol=1e-14, atol=1e-15)
    if d == 1:
        # optimal 1-D clusters are contiguous in sorted order
        order = np.argsort(X[:, 0])
        runs = best_lab[order]
        assert (np.diff(runs) != 0).sum() == K - 1


def test_brute_force_tiny_assign():
    rng = _rng(20)
    X = rng.normal(size=(1, 6, 2))
    C = rng.normal(size=(1, 3, 2))
    ids, d1, _, _ = oracle.assign(X, C)
    for i in range(6):
        dists = [float(((X[0, i] - C[0, k]) ** 2).sum()) for k in range(3)]
        assert ids[0, i] == min(range(3), key=lambda k: (dists[k], k))
        assert d1[0, i] == pytest.approx(min(dists), rel=1e-15)


# ---------------------------------------------------------------- iteration invariants

@pytest.mark.parametrize("weighted", [False, True])
def test_inertia_never_increases_and_fixed_point_invariants(weighted):
    rng = _rng(30)
    B, N, K, d = 2, 400, 12, 4
    X = _blobs(rng, B, N, 8, d, spread=0.8)
    w = rng.uniform(0.05, 2.0, size=(B, N)) if weighted else None
    C0 = np.stack([X[b, rng.choice(N, K, replace=False)] for b in range(B)])
    out = oracle.fit(X, C0, iters=15, w=w)
    ih = out["inertia_hist"]
    assert (np.diff(ih, axis=0) <= 1e-12 * ih[:-1]).all()
    # each point at its nearest centroid; each nonempty centroid the weighted mean of its members
    C = out["C_hist"][-1]
    ids, d1, d2, _ = oracle.assign(X, C, w)
    D = ((X[:, :, None, :] - C[:, None]) ** 2).sum(-1)
    np.testing.assert_array_equal(ids, D.argmin(-1))
    Cn, counts, _ = oracle.update(X, ids, C, w)
    assert (counts.sum(1) == N).all()


def test_weight_invariances_and_permutations():
    rng = _rng(40)
    B, N, K, d = 1, 150, 6, 3
    X = _blobs(rng, B, N, 6, d, spread=0.5)
    C0 = X[:, rng.choice(N, K, replace=False)]
    base = oracle.fit(X, C0, iters=6)
    const = oracle.fit(X, C0, iters=6, w=np.full((B, N), 0.37))
    scaled_w = rng.uniform(0.1, 1.0, size=(B, N))
    a = oracle.fit(X, C0, iters=6, w=scaled_w)
    s = oracle.fit(X, C0, iters=6, w=3.7 * scaled_w)
    np.testing.assert_allclose(const["C_hist"], base["C_hist"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s["C_hist"], a["C_hist"], rtol=1e-12, atol=1e-13)
    # permuting points leaves the centroids unchanged
    p = rng.permutation(N)
    perm = oracle.fit(X[:, p], C0, iters=6)
    np.testing.assert_allclose(perm["C_hist"], base["C_hist"], rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(perm["ids"][0], base["ids"][0][p])
    # permuting centroids permutes labels
    q = rng.permutation(K)
    ids0, d1, d2, _ = oracle.assign(X, C0)
    ids1, _, _, _ = oracle.assign(X, C0[:, q])
    inv = np.argsort(q)
    assert not oracle.near_tie(d1, d2).all()
    np.testing.assert_array_equal(ids1, inv[ids0])


# ---------------------------------------------------------------- library cross-checks

@pytest.mark.parametrize("iters", [1, 4, 9])
def test_matches_sklearn_lloyd_with_sample_weight(iters):
    sk = pytest.importorskip("sklearn.cluster")
    rng = _rng(50 + iters)
    N, K, d = 300, 5, 3
    X = _blobs(rng, 1, N, K, d, spread=0.7)[0]
    w = rng.uniform(0.1, 2.0, size=N)
    C0 = X[rng.choice(N, K, replace=False)]
    km = sk.KMeans(n_clusters=K, init=C0, n_init=1, algorithm="lloyd", max_iter=iters, tol=0.0)
    km.fit(X, sample_weight=w)
    out = oracle.fit(X[None], C0[None], iters=iters, w=w[None])
    assert (out["counts"] > 0).all(), "sklearn relocates empty clusters; pick a run without them"
    np.testing.assert_allclose(out["C_hist"][-1][0], km.cluster_centers_, rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("K", [1, 2, 3, 8, 16])
def test_grid_init_is_numpy_linspace(K):
    rng = _rng(60 + K)
    X = (rng.standard_t(5, size=(4, 257)) * 0.02).astype(np.float16).astype(np.float64)
    C = oracle.grid_init(X[:, :, None], K)[:, :, 0]
    for b in range(4):
        ref = np.linspace(X[b].min(), X[b].max(), K)
        np.testing.assert_array_equal(C[b], ref)
        assert C[b, 0] == X[b].min()
        if K > 1:
            assert C[b, -1] == X[b].max()


def test_near_tie_rule():
    d1 = np.array([1.0, 1.0, 0.0, 5.0])
    d2 = np.array([1.0005, 1.01, 0.0, 5.0])
    np.testing.assert_array_equal(oracle.near_tie(d1, d2), [True, False, True, True])


def test_round_to_dtype_is_rne():
    import torch
    C = np.array([1.0 + 2.0 ** -11, 1.0 + 3 * 2.0 ** -11], np.float32)   # halfway cases in fp16
    r = oracle.round_to_dtype(C, torch.float16)
    np.testing.assert_array_equal(r, [1.0, 1.0 + 2.0 ** -9])
