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


def _fp32_decision(X, C, dtype):
    """The encoding's decision taken in its own precision: x and the centroids rounded to the
    values' dtype, (x - c)^2 in fp32, the first (lowest-index) minimum."""
    x = X.to(dtype).float().numpy()
    c = C.to(dtype).float().numpy()
    dd = x[:, :, None] - c[:, None, :]
    dd = dd * dd
    return np.argmin(dd, axis=2)


@pytest.mark.parametrize("dt", ["f16", "bf16", "f32"])
@pytest.mark.parametrize("K", [1, 2, 3, 8, 15, 16, 17, 31, 64, 129, 256])
@pytest.mark.parametrize("N,offset", [(4096, 0), (1000, 0), (4096, 1)])
def test_encode_fp32_decision_exact(dt, K, N, offset, cuda_device):
    # every search depth, the vector form (N a multiple of 16, aligned rows) and the strided one
    # (ragged N, or rows starting one element past a 16-byte boundary); values on centroids, on
    # midpoints, far outside the codebook (ties among several rounded distances) and duplicates
    g = torch.Generator().manual_seed(K * 7 + N + offset)
    B = 3
    C = torch.randn((B, K), generator=g) * 0.05
    if K > 3:
        C[:, 3] = C[:, 0]
        C[:, K - 1] = C[:, 1]
    Cr = C.to(DT[dt]).float()
    X = torch.randn((B, N + offset), generator=g) * 0.06
    n_on = min(N // 8, 64)
    pick = torch.randint(0, K, (B, n_on), generator=g)
    X[:, offset:offset + n_on] = torch.gather(Cr, 1, pick)
    if K > 1:
        srt = torch.sort(Cr, dim=1).values
        mids = (srt[:, :-1] + srt[:, 1:]) / 2
        m = min(N // 8, mids.shape[1])
        X[:, offset + n_on:offset + n_on + m] = mids[:, :m]
    inf = float("inf")
    X[:, offset + N - 8:offset + N] = torch.tensor([6e4, -6e4, 1e5, -1e5, inf, -inf, 0.0, -0.0])
    Xd = X.to(DT[dt]).to(cuda_device)[:, offset:]
    ref = _fp32_decision(X[:, offset:], C, DT[dt])
    for b in range(B):
        row = Xd[b:b + 1]
        if offset:
            # a view one element into a row: the data pointer sits off the 16-byte grid
            buf = torch.empty(N + 8, dtype=DT[dt], device=cuda_device)
            buf[1:N + 1] = row[0]
            row = buf[1:N + 1].view(1, N)
        codes = km.km_encode1d(row, C[b:b + 1].to(cuda_device))
        torch.cuda.synchronize()
        got = to_np(codes)[0].astype(np.int64)
        np.testing.assert_array_equal(got, ref[b], err_msg=f"row {b}")
