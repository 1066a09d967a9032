"""e-means and dead-cluster splitting on the GPU against the CPU oracle (needs a B200).

The data are blobs far apart with one starting centroid per blob, so every assignment the run
makes is unambiguous and the GPU run must follow the oracle's trajectory step for step; the
remaining difference is fp32 (GPU state) against fp64 (oracle) arithmetic.
"""
import numpy as np
import pytest
import torch

import exact_lloyd_means_assign_b200 as km
import oracle
from oracle import emeans as em_oracle
from parity import to_np

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    torch.cuda.set_device(cuda_device)
    yield
    assert km.km_device_error() == 0


def blobs(B, N, K, d, seed, spread=3.0, sigma=0.2):
    g = torch.Generator().manual_seed(seed)
    mu = torch.randn((B, K, d), generator=g) * spread
    comp = torch.randint(0, K, (B, N), generator=g)
    X = torch.gather(mu, 1, comp[..., None].expand(B, N, d)) + sigma * torch.randn((B, N, d), generator=g)
    C0 = mu + 0.05 * torch.randn((B, K, d), generator=g)
    return X, C0


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30)


def _check_sse(got, ref, X):
    """Objective per epoch: 1e-4 relative, or the rounding scale of the expanded distance
    ||x||^2 - 2 x.c + ||c||^2 evaluated with fp32 accumulation, about 1e-6 (||x||^2 + ||c||^2)
    per point; it dominates when the points sit far from the origin relative to their spread."""
    scale = 2.0 * (oracle.as_f64(X) ** 2).sum(axis=(1, 2))
    assert np.all(np.abs(got - ref) <= 1e-4 * np.abs(ref) + 1e-6 * scale[None, :]), (got, ref)


@pytest.mark.parametrize("dt,B,N,K,d,batch,epochs,alpha0,weighted", [
    ("f16", 2, 3000, 12, 64, 700, 3, 0.3, False),    # tensor-core assignment, ragged last batch
    ("f32", 1, 2500, 9, 16, 512, 2, 0.5, True),      # exact fp32 assignment, weighted
    ("bf16", 1, 2000, 20, 128, 2000, 2, 0.8, False),  # one mini-batch per epoch
    # one launch sequence per mini-batch for all problems (fused moving-average update)
    ("f16", 3, 5000, 40, 128, 1024, 3, 0.4, True),
    ("f32", 2, 2500, 9, 32, 512, 2, 0.5, True),      # exact fp32 assignment of a strided view
    ("f16", 4, 1500, 70, 256, 600, 2, 0.6, False),
])
def test_emeans_matches_oracle(dt, B, N, K, d, batch, epochs, alpha0, weighted, cuda_device):
    X, C0 = blobs(B, N, K, d, seed=N + K)
    X = X.to(DT[dt])
    w = torch.rand((B, N), generator=torch.Generator().manual_seed(7)) + 0.1 if weighted else None
    C = C0.to(cuda_device)
    _, sse = km.km_emeans_fit(X.to(cuda_device), C, batch, epochs, alpha0,
                              w=None if w is None else w.to(cuda_device), want_sse=True)
    torch.cuda.synchronize()
    ref = em_oracle.fit(oracle.as_f64(X), oracle.as_f64(C0), batch, epochs, alpha0,
                        w=None if w is None else oracle.as_f64(w), assign_dtype=DT[dt])
    for b in range(B):
        assert _rel(to_np(C)[b], ref["C"][b]) <= 1e-4, b
    _check_sse(to_np(sse), ref["sse_hist"], X)


@pytest.mark.parametrize("d", [32, 64])
def test_emeans_zero_epochs_and_alpha_one_full_batch(d, cuda_device):
    X, C0 = blobs(1, 1000, 6, d, seed=3)
    X = X.to(torch.float16).to(cuda_device)
    C = C0.to(cuda_device)
    km.km_emeans_fit(X, C, 100, 0, 0.5)
    torch.cuda.synchronize()
    assert torch.equal(C.cpu(), C0)
    # one epoch, one full batch, alpha 1: one Lloyd iteration
    C = C0.to(cuda_device)
    km.km_emeans_fit(X, C, 1000, 1, 1.0)
    C_l = C0.to(cuda_device)
    km.km_fit(X, C_l, 1)
    torch.cuda.synchronize()
    assert _rel(to_np(C), to_np(C_l)) <= 1e-6


@pytest.mark.parametrize("K,d", [(300, 24), (2500, 7)])
def test_split_dead_matches_oracle(K, d, cuda_device):
    rng = np.random.default_rng(K)
    B = 3
    C = rng.normal(size=(B, K, d)).astype(np.float32)
    sizes = rng.integers(1, 9, size=(B, K)).astype(np.float32)
    sizes[rng.random((B, K)) < 0.2] = 0
    Nc = rng.uniform(0.5, 3, size=(B, K)).astype(np.float32)
    # targets u * total land on m + 0.3, never on a running sum (those stay dyadic rationals)
    total = sizes.sum(1, keepdims=True)
    u = ((rng.integers(0, total.astype(np.int64)[:, 0][:, None], size=(B, K)) + 0.3) / total)
    u = u.astype(np.float32)
    eps = 0.01
    Cg = torch.from_numpy(C).to(cuda_device)
    sg = torch.from_numpy(sizes).to(cuda_device)
    Ng = torch.from_numpy(Nc).to(cuda_device)
    Sg = torch.zeros((B, K, d), device=cuda_device)
    donors = km.km_split_dead(Cg, sg, torch.from_numpy(u).to(cuda_device), eps, Nc=Ng, S=Sg,
                              want_donors=True)
    torch.cuda.synchronize()
    for b in range(B):
        Cr, sr, Nr, dr = em_oracle.split_dead(C[b], sizes[b], u[b].astype(np.float64), np.float32(eps),
                                              Nc[b])
        np.testing.assert_array_equal(to_np(donors)[b], dr)
        np.testing.assert_array_equal(to_np(sg)[b], sr)
        np.testing.assert_allclose(to_np(Cg)[b], Cr, rtol=2e-7, atol=1e-7)
        np.testing.assert_allclose(to_np(Ng)[b], Nr, rtol=1e-7)
        rev = dr >= 0
        np.testing.assert_allclose(to_np(Sg)[b][rev], (Cr * Nr[:, None])[rev], rtol=1e-6, atol=1e-7)


@pytest.mark.parametrize("d", [32, 64])
def test_emeans_split_revives_a_dead_centroid(d, cuda_device):
    # blob 1 is two sub-blobs at mu1 (1 +/- 0.3 s_k); centroid 3 starts far away and gets no
    # point in the first epoch; its uniform picks blob 1 as donor, and the split with eps = 0.3
    # puts the two halves on the sub-blob centres, so the second epoch separates them cleanly
    eps = 0.3
    g = torch.Generator().manual_seed(11)
    mu = torch.randn((3, d), generator=g) * 3
    sgn = torch.tensor([1.0 if k % 2 == 0 else -1.0 for k in range(d)])
    centres = torch.stack([mu[0], mu[1] * (1 + eps * sgn), mu[1] * (1 - eps * sgn), mu[2]])
    comp = torch.randint(0, 4, (1, 2400), generator=g)
    X = (centres[comp] + 0.1 * torch.randn((1, 2400, d), generator=g)).to(torch.float16)
    C0 = torch.stack([mu[0], mu[1], mu[2], torch.full((d,), 60.0)])[None]
    sizes0 = em_oracle.fit(oracle.as_f64(X), oracle.as_f64(C0), 400, 1, 0.5,
                           assign_dtype=torch.float16)["sizes_last"][0]
    assert sizes0[3] == 0 and sizes0[1] > 0
    u = np.zeros((2, 1, 4), np.float32)
    u[0, 0, 3] = (sizes0[0] + 0.5 * sizes0[1] + 0.3) / sizes0.sum()
    C = C0.to(cuda_device)
    _, sse = km.km_emeans_fit(X.to(cuda_device), C, 400, 2, 0.5,
                              split_u=torch.from_numpy(u).to(cuda_device), split_eps=eps, want_sse=True)
    torch.cuda.synchronize()
    ref = em_oracle.fit(oracle.as_f64(X), oracle.as_f64(C0), 400, 2, 0.5, split_u=u.astype(np.float64),
                        eps=eps, assign_dtype=torch.float16)
    assert ref["donors"][0, 0, 3] == 1 and ref["sizes_last"][0, 3] > 0
    assert _rel(to_np(C)[0], ref["C"][0]) <= 1e-4
    _check_sse(to_np(sse), ref["sse_hist"], X)
    # the revived centroid sits on one of the sub-blob centres
    got = to_np(C)[0]
    dists = [np.linalg.norm(got[3] - centres[i].numpy()) for i in (1, 2)]
    assert min(dists) < 0.1
