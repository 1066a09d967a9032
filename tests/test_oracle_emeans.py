"""Pins for the e-means / splitting oracle (CPU only).

Each test ties the oracle to something other than itself: the Lloyd oracle's C code for the
limits where e-means reduces to a Lloyd step, hand-worked small examples, and invariants of the
moving average and of splitting.
"""
import numpy as np
import pytest

import oracle
from oracle import emeans


def test_alpha_schedule_cosine_endpoints():
    a = emeans.alpha_schedule(100, 0.4)
    assert a[0] == pytest.approx(0.4)
    assert a[50] == pytest.approx(0.4 * 0.55)            # cos(pi/2) = 0: halfway between
    # one step past the end would be 0.1 * alpha0; the last step is just above it
    assert 0.04 < a[-1] < 0.0401
    assert np.all(np.diff(a) < 0)


def test_ema_with_alpha_one_is_the_lloyd_update():
    rng = np.random.default_rng(0)
    X = rng.normal(size=(2, 300, 5))
    C = rng.normal(size=(2, 9, 5))
    C[:, 8] += 50.0                                        # a centroid that gets no point
    w = rng.uniform(0.1, 2.0, size=(2, 300))
    ids, _, _, _ = oracle.assign(X, C, w)
    s, n = emeans.batch_stats(X, ids, 9, w)
    S0 = rng.normal(size=C.shape)
    N0 = rng.uniform(1, 3, size=(2, 9))
    _, _, C1 = emeans.ema_update(S0, N0, C, s, n, 1.0)
    C_ref, counts, wsum = oracle.update(X, ids, C, w)
    np.testing.assert_allclose(n, wsum, rtol=1e-12)
    # the empty cluster: S and N both become 0 -> keeps C
    np.testing.assert_allclose(C1, C_ref, rtol=1e-12, atol=1e-12)


def test_one_full_batch_step_with_alpha_one_is_one_lloyd_iteration():
    rng = np.random.default_rng(1)
    X = rng.normal(size=(1, 400, 4)).astype(np.float32).astype(np.float64)
    C0 = X[:, :7].copy()
    r = emeans.fit(X, C0, batch=400, epochs=1, alpha0=1.0)
    lloyd = oracle.fit(X, C0, 1)["C_hist"][1]
    np.testing.assert_allclose(r["C"], lloyd, rtol=1e-12)
    np.testing.assert_allclose(r["C_epochs"][0], lloyd, rtol=1e-12)


def test_vanishing_step_is_a_lloyd_step_after_the_final_shift():
    # with alpha0 -> 0 the centroids do not move during the epoch, so every batch is labelled
    # against C0 and the empirical mean of the epoch is one Lloyd update of C0
    rng = np.random.default_rng(2)
    X = rng.normal(size=(2, 700, 3))
    C0 = X[:, :5].copy()
    w = rng.uniform(0.5, 1.5, size=(2, 700))
    r = emeans.fit(X, C0, batch=128, epochs=1, alpha0=1e-13, w=w)
    lloyd = oracle.fit(X, C0, 1, w=w)["C_hist"][1]
    np.testing.assert_allclose(r["C"], lloyd, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(r["C_epochs"][0], C0, rtol=1e-9, atol=1e-9)


def test_hand_worked_two_batch_example():
    # 1-D, K = 2, C0 = (0.5, 11), batches (0, 1, 10) and (2, 12, 14), alpha0 = 1, T = 2:
    #   alpha_0 = 1, alpha_1 = 0.1 + 0.9 * (1 + cos(pi/2)) / 2 = 0.55
    #   step 0: labels (0, 0, 1); s = (1, 10), n = (2, 1) -> S = (1, 10), N = (2, 1), C = (0.5, 10)
    #   step 1: labels (0, 1, 1); s = (2, 26), n = (1, 2)
    #           S = 0.45 (1, 10) + 0.55 (2, 26) = (1.55, 18.8); N = (1.45, 1.55)
    #           C = (1.55 / 1.45, 18.8 / 1.55)
    #   final shift: cluster 0 = {0, 1, 2} -> 1, cluster 1 = {10, 12, 14} -> 12
    #   objective at assignment time: (0.25 + 0.25 + 1) + (2.25 + 4 + 16) = 23.75
    X = np.array([0, 1, 10, 2, 12, 14], dtype=np.float64).reshape(1, 6, 1)
    C0 = np.array([0.5, 11.0]).reshape(1, 2, 1)
    r = emeans.fit(X, C0, batch=3, epochs=1, alpha0=1.0)
    np.testing.assert_allclose(r["C_epochs"][0, 0, :, 0], [1.55 / 1.45, 18.8 / 1.55], rtol=1e-12)
    np.testing.assert_allclose(r["C"][0, :, 0], [1.0, 12.0], rtol=1e-12)
    assert r["sse_hist"][0, 0] == pytest.approx(23.75, rel=1e-12)


def test_split_hand_worked_example():
    # sizes (0, 3, 1, 0), u_0 = 0.5, u_3 = 0.9, eps = 0.25, d = 2 (signs +, -):
    #   cluster 0: total 4, target 2, running sums 0, 3 -> donor 1; c1 = (4, 8) gives
    #              c0 = (5, 6), c1 = (3, 10); sizes 1.5 and 1.5
    #   cluster 3: total 4, target 3.6, running sums 1.5, 3, 4 -> donor 2; c2 = (10, -2) gives
    #              c3 = (12.5, -1.5), c2 = (7.5, -2.5); sizes 0.5 and 0.5
    C = np.array([[1.0, 2.0], [4.0, 8.0], [10.0, -2.0], [0.0, 0.0]])
    Cn, sizes, Nn, donors = emeans.split_dead(C, [0, 3, 1, 0], [0.5, 0.0, 0.0, 0.9], 0.25,
                                              Ncnt=[0.2, 2.0, 1.0, 0.0])
    np.testing.assert_array_equal(Cn, [[5, 6], [3, 10], [7.5, -2.5], [12.5, -1.5]])
    np.testing.assert_array_equal(sizes, [1.5, 1.5, 0.5, 0.5])
    np.testing.assert_array_equal(Nn, [1.0, 1.0, 0.5, 0.5])
    np.testing.assert_array_equal(donors, [1, -1, -1, 2])


def test_split_invariants_and_proportional_draws():
    rng = np.random.default_rng(3)
    K, d = 40, 6
    for _ in range(20):
        sizes = rng.integers(0, 5, K).astype(np.float64)
        sizes[rng.random(K) < 0.3] = 0
        if sizes.sum() == 0:
            continue
        C = rng.normal(size=(K, d))
        Ncnt = rng.uniform(0, 3, K)
        u = rng.random(K)
        Cn, sn, Nn, donors = emeans.split_dead(C, sizes, u, 1e-3, Ncnt)
        assert sn.sum() == pytest.approx(sizes.sum())
        # a revived cluster's stale average count is replaced by half of its donor's
        assert Nn.sum() == pytest.approx(Ncnt.sum() - Ncnt[donors >= 0].sum())
        assert np.all(sn > 0)                      # every dead cluster revived
        for i in np.nonzero(donors >= 0)[0]:
            assert sizes[i] == 0 and donors[i] != i
    # draws land in proportion to size: u on a fine grid over one dead cluster
    sizes = np.array([0.0, 1.0, 2.0, 5.0])
    hits = np.zeros(4)
    for u0 in (np.arange(800) + 0.5) / 800:
        _, _, _, dn = emeans.split_dead(np.ones((4, 2)), sizes, [u0, 0, 0, 0], 0.1)
        hits[dn[0]] += 1
    np.testing.assert_array_equal(hits, [0, 100, 200, 500])


def test_dead_cluster_is_revived_between_epochs_only():
    rng = np.random.default_rng(4)
    X = np.concatenate([rng.normal(0, 0.1, (1, 200, 2)), rng.normal(5, 0.1, (1, 200, 2))], axis=1)
    X = X[:, rng.permutation(400)]
    C0 = np.array([[[0.0, 0.0], [5.0, 5.0], [100.0, 100.0]]])   # the third never gets a point
    u = np.full((2, 1, 3), 0.25)
    r = emeans.fit(X, C0, batch=100, epochs=2, alpha0=0.5, split_u=u, eps=0.01)
    assert r["donors"][0, 0, 2] in (0, 1) and (r["donors"][1] == -1).all()
    assert r["sizes_last"][0, 2] > 0           # revived: it owns points in the second epoch
    r0 = emeans.fit(X, C0, batch=100, epochs=2, alpha0=0.5)
    assert r0["sizes_last"][0, 2] == 0
    assert r["sse_hist"][1, 0] < r0["sse_hist"][1, 0]
