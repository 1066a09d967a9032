"""Pins for the 1-D codebook oracle (CPU only): the printed weight-clustering example, brute
force on small inputs, and hand-worked k-means++ draws."""
import numpy as np
import pytest
import torch

from conftest import load_golden
from oracle import codebook1d


def test_encode_reproduces_the_printed_index_vector():
    gold = load_golden("worked_example_weight_clustering.txt")
    vals = np.array([float(v) for v in gold["values"]])[None]
    cents = np.array([float(v) for v in gold["centroids"]])[None]
    codes, _, _ = codebook1d.encode1d(vals, cents)
    assert codes.dtype == np.uint8
    np.testing.assert_array_equal(codes[0, :10], [int(v) for v in gold["labels_first10"]])
    np.testing.assert_array_equal(codes[0, 10:], [2, 2, 2])


@pytest.mark.parametrize("K", [1, 7, 256])
def test_encode_is_brute_force_argmin(K):
    rng = np.random.default_rng(K)
    X = rng.normal(size=(3, 500)).astype(np.float16)
    C = rng.normal(size=(3, K)).astype(np.float32)
    C[:, K // 2] = C[:, 0]                      # a duplicate: the lower index must win
    codes, _, _ = codebook1d.encode1d(X.astype(np.float64), C.astype(np.float64), torch.float16)
    Cr = torch.from_numpy(C).to(torch.float16).double().numpy()
    dist = (X.astype(np.float64)[:, :, None] - Cr[:, None, :]) ** 2
    np.testing.assert_array_equal(codes, np.argmin(dist, axis=2))   # argmin keeps the first


def test_kmeanspp_hand_worked_draws():
    # X = (0, 1, 3), unit weights. Draw 1: u = 0.1, mass (1, 1, 1), target 0.3 -> point 0.
    # Draw 2: D^2 = (0, 1, 9), total 10, u = 0.5 -> target 5, running (0, 1, 10) -> point 2.
    # Draw 3: D^2 = (0, 1, 0), only point 1 has mass -> point 1.
    C, chosen = codebook1d.kmeanspp1d(np.array([[0.0, 1.0, 3.0]]), 3, np.array([[0.1, 0.5, 0.7]]))
    np.testing.assert_array_equal(chosen, [[0, 2, 1]])
    np.testing.assert_array_equal(C, [[0.0, 3.0, 1.0]])
    # a fourth centre finds no mass left: point 0
    C, chosen = codebook1d.kmeanspp1d(np.array([[0.0, 1.0, 3.0]]), 4,
                                      np.array([[0.1, 0.5, 0.7, 0.9]]))
    np.testing.assert_array_equal(chosen, [[0, 2, 1, 0]])


def test_kmeanspp_draw_frequencies_are_weight_times_d2():
    X = np.array([[0.0, 1.0, 2.0, 4.0]])
    w = np.array([[1.0, 3.0, 1.0, 0.5]])
    first = np.zeros(4)
    second = np.zeros(4)
    grid = (np.arange(1300) + 0.5) / 1300
    for g in grid:
        _, ch = codebook1d.kmeanspp1d(X, 1, np.array([[g]]), w)
        first[ch[0, 0]] += 1
        _, ch = codebook1d.kmeanspp1d(X, 2, np.array([[0.0, g]]), w)   # first centre = point 0
        second[ch[0, 1]] += 1
    # first: proportional to w = (1, 3, 1, 0.5) / 5.5; second: w * D^2 = (0, 3, 4, 8) / 15
    np.testing.assert_allclose(first / 1300, np.array([1, 3, 1, 0.5]) / 5.5, atol=1.5 / 1300)
    np.testing.assert_allclose(second / 1300, np.array([0, 3, 4, 8]) / 15, atol=1.5 / 1300)
