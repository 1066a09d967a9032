"""The single-launch fit for small problems against the oracle, iteration by iteration.

Lloyd's iteration as the pages state it (technologypulse.uk Flash-KMeans article, the assignment
and update of "Bottleneck 1" and "Bottleneck 2"): every point to its nearest centroid (lowest
index on ties), every centroid to the weighted mean of its members, an empty cluster keeping its
previous centroid. The data are well separated clusters, so no point is a near tie and the labels
of every iteration are unique; the check is then exact on labels and within the stated
tolerances on centroids (1e-3 relative) and inertia (1e-4 relative).
"""
import numpy as np
import pytest
import torch

import exact_lloyd_means_assign_b200 as km
import oracle

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def _separated(B, N, K, d, seed, far=0):
    """Tight clusters around well separated centres; the initial centroids are noisy copies of
    the centres, and the last `far` of them sit far away, so they stay empty."""
    g = torch.Generator().manual_seed(seed)
    mu = torch.randn((B, K, d), generator=g) * 4.0
    lab = torch.randint(0, K - far, (B, N), generator=g)
    X = torch.gather(mu, 1, lab[..., None].expand(B, N, d)) + 0.05 * torch.randn((B, N, d), generator=g)
    C0 = mu + 0.2 * torch.randn((B, K, d), generator=g)
    if far:
        C0[:, K - far:] = 1e3
    return X, C0


@pytest.mark.parametrize("dt,B,N,K,d,weighted,far", [
    ("f32", 1, 4096, 32, 16, False, 0),     # config 1's shape
    ("f16", 2, 3000, 40, 24, True, 3),      # 17..32 coordinates; empty clusters
    ("bf16", 3, 700, 17, 64, True, 0),      # 33..64 coordinates, ragged last CTA
    ("f32", 2, 1000, 64, 2, True, 5),
    ("f32", 4, 200, 8, 3, False, 0),        # one CTA per problem
    ("f32", 1, 9000, 32, 16, False, 0),     # 141 CTAs
    ("bf16", 2, 5000, 20, 40, True, 2),
])
def test_small_fit_matches_oracle(dt, B, N, K, d, weighted, far, cuda_device):
    dtype = DT[dt]
    X, C0 = _separated(B, N, K, d, seed=B * 100 + K + d, far=far)
    X = X.to(dtype)
    w = (torch.rand((B, N), generator=torch.Generator().manual_seed(7)) + 0.1) if weighted else None
    iters = 6
    Xd, Cd = X.to(cuda_device), C0.clone().to(cuda_device)
    wd = None if w is None else w.to(cuda_device)
    _, ids, ih, ch = km.km_fit(Xd, Cd, iters, w=wd, want_ids=True, want_inertia=True, want_hist=True)
    torch.cuda.synchronize()
    assert km.km_device_error() == 0
    ref = oracle.fit(oracle.as_f64(X), oracle.as_f64(C0), iters, w=None if w is None else oracle.as_f64(w),
                     assign_dtype=dtype)
    hist = ch.cpu().numpy().astype(np.float64)
    X64 = oracle.as_f64(X)
    for t in range(iters + 1):
        err = np.linalg.norm(hist[t] - ref["C_hist"][t]) / np.linalg.norm(ref["C_hist"][t])
        assert err <= 1e-3, (t, err)
        if t < iters:
            _, d1, d2, _ = oracle.assign(X64, oracle.round_to_dtype(ref["C_hist"][t], dtype))
            assert not oracle.near_tie(d1, d2).any()
    np.testing.assert_allclose(ih.cpu().numpy(), ref["inertia_hist"], rtol=1e-4)
    np.testing.assert_array_equal(ids.cpu().numpy(), ref["ids"])
    if far:   # the far centroids never gain a member and keep their place
        np.testing.assert_array_equal(hist[iters][:, K - far:], 1e3)


def test_small_fit_barrier_timeout_and_the_next_fit_is_clean(cuda_device):
    X, C0 = _separated(1, 4096, 32, 16, seed=3)
    Xd = X.to(cuda_device)
    assert km.km_device_error() == 0
    old = km.km_debug_wait_limit(20_000_000)          # 20 ms
    try:
        km.km_debug_inject(2)
        km.km_fit(Xd, C0.clone().to(cuda_device), 4)
        code = km.km_device_error()                    # synchronises
    finally:
        km.km_debug_inject(0)
        km.km_debug_wait_limit(old)
    assert code & 1, "the skipped arrival must make the barrier waits run out"
    Cd = C0.clone().to(cuda_device)
    km.km_fit(Xd, Cd, 4)
    torch.cuda.synchronize()
    assert km.km_device_error() == 0
    ref = oracle.fit(oracle.as_f64(X), oracle.as_f64(C0), 4, assign_dtype=torch.float32)
    err = np.linalg.norm(Cd.cpu().numpy() - ref["C_hist"][4]) / np.linalg.norm(ref["C_hist"][4])
    assert err <= 1e-3
