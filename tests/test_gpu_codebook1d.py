"""1-D codebook encoding and k-means++ seeding on the GPU against the CPU oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import exact_lloyd_means_assign_b200 as km
import oracle
from conftest import load_golden
from oracle import codebook1d
from parity import to_np

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    torch.cuda.set_device(cuda_device)
    yield
    assert km.km_device_error() == 0


def test_encode_printed_example(cuda_device):
    gold = load_golden("worked_example_weight_clustering.txt")
    vals = torch.tensor([[float(v) for v in gold["values"]]], dtype=torch.float32, device=cuda_device)
    cents = torch.tensor([[float(v) for v in gold["centroids"]]], dtype=torch.float32, device=cuda_device)
    codes = km.km_encode1d(vals, cents)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(codes)[0, :10], [int(v) for v in gold["labels_first10"]])
    np.testing.assert_array_equal(to_np(codes)[0, 10:], [2, 2, 2])


@pytest.mark.parametrize("dt,B,N,K", [("f16", 7, 5000, 16), ("bf16", 3, 4099, 256), ("f32", 2, 777, 1),
                                      ("f16", 2, 70000, 200)])
def test_encode_matches_oracle(dt, B, N, K, cuda_device):
    g = torch.Generator().manual_seed(N + K)
    X = (torch.randn((B, N), generator=g) * 0.03).to(DT[dt])
    C = torch.randn((B, K), generator=g) * 0.03
    if K > 2:
        C[:, K - 1] = C[:, 1]           # duplicates: the lower index wins
        C[:, 2] = C[:, 1]
    codes = km.km_encode1d(X.to(cuda_device), C.to(cuda_device))
    torch.cuda.synchronize()
    ref, d1, d2 = codebook1d.encode1d(oracle.as_f64(X), oracle.as_f64(C), DT[dt])
    got = to_np(codes)
    bad = (got != ref) & ~oracle.near_tie(d1, d2)
    assert not bad.any(), int(bad.sum())
    if K > 2:
        assert not np.isin(got, [2, K - 1]).any()


@pytest.mark.parametrize("dt,B,N,K,weighted", [("f16", 5, 3000, 16, True), ("bf16", 2, 8192, 64, False),
                                               ("f32", 3, 100, 100, True), ("f32", 1, 50, 60, False)])
def test_kmeanspp_matches_oracle(dt, B, N, K, weighted, cuda_device):
    g = torch.Generator().manual_seed(3 * N + K)
    X = (torch.randn((B, N), generator=g) * 0.02).to(DT[dt])
    w = (torch.randn((B, N), generator=g) ** 2 + 1e-3) if weighted else None
    u = torch.rand((B, K), generator=g)
    C, chosen = km.km_init_kmeanspp1d(X.to(cuda_device), K, u.to(cuda_device),
                                      w=None if w is None else w.to(cuda_device), want_chosen=True)
    torch.cuda.synchronize()
    Cr, ch = codebook1d.kmeanspp1d(oracle.as_f64(X), K, oracle.as_f64(u),
                                   None if w is None else oracle.as_f64(w))
    np.testing.assert_array_equal(to_np(chosen), ch)
    np.testing.assert_array_equal(to_np(C)[:, :, 0].astype(np.float64), Cr)
