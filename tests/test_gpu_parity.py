"""CUDA path vs the CPU oracle, element by element, through the C ABI (needs a B200).

Sizes are chosen so the oracle finishes in seconds while the kernels still see several tiles
and ragged tails (N not a multiple of 128, K not a multiple of the centroid tile, d not a
multiple of 64). Full-size workloads are in test_gpu_fullsize.py.
"""
import numpy as np
import pytest
import torch

import exact_lloyd_means_assign_b200 as km
import oracle
import synth
from parity import check_assign, check_update, mixture, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_device):
    torch.cuda.set_device(cuda_device)
    yield
    assert km.km_device_error() == 0


DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


# ------------------------------------------------------------------ prep / grid init

@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
def test_prep_rounds_and_norms(dt, cuda_device):
    dtype = DT[dt]
    C = torch.randn((3, 50, 40), device=cuda_device) * 3
    Cx, cn = km.km_prep(C, dtype)
    torch.cuda.synchronize()
    assert torch.equal(Cx, C.to(dtype))
    ref = (Cx.double() ** 2).sum(-1)
    torch.testing.assert_close(cn.double(), ref, rtol=2e-6, atol=0)


@pytest.mark.parametrize("dt", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("K", [1, 2, 8, 16, 33])
def test_grid_init_matches_oracle(dt, K, cuda_device):
    g = torch.Generator().manual_seed(K)
    X = (torch.randn((37, 1001, 1), generator=g) * 0.02).to(DT[dt])
    C = km.km_init_grid1d(X.to(cuda_device), K)
    ref = oracle.grid_init(X, K).astype(np.float32)
    np.testing.assert_array_equal(to_np(C), ref)


# ------------------------------------------------------------------ assignment

TC_CASES = [
    ("f16", 2, 3000, 300, 128),
    ("bf16", 2, 3000, 300, 128),
    ("f16", 1, 1000, 1024, 128),
    ("f16", 3, 777, 64, 64),
    ("f16", 2, 500, 100, 96),
    ("f16", 1, 640, 200, 16),
    ("f16", 1, 300, 37, 200),
    ("bf16", 1, 300, 513, 256),
    ("f16", 2, 2100, 700, 128),     # three 256-wide centroid tiles: an odd count per item
    ("f16", 1, 129, 1, 128),
    ("f16", 2, 100, 300, 24),
    ("bf16", 5, 1, 7, 8),
    ("bf16", 1, 600, 40000, 64),     # 157 centroid tiles streamed through the ring
]
SIMT_CASES = [
    ("f32", 1, 4096, 32, 16),
    ("f16", 2, 1000, 50, 12),
    ("f32", 1, 500, 70, 130),
    ("bf16", 1, 300, 40, 1),
    ("f16", 1, 200, 20, 264),
]


@pytest.mark.parametrize("dt,B,N,K,d", TC_CASES + SIMT_CASES)
@pytest.mark.parametrize("weighted", [False, True])
def test_assign_matches_oracle(dt, B, N, K, d, weighted, cuda_device):
    dtype = DT[dt]
    X, C = mixture(B, N, d, K, dtype, cuda_device, seed=B * 1000 + N + K + d)
    w = (torch.rand((B, N), device=cuda_device) + 0.1) if weighted else None
    Cx, cn = km.km_prep(C, dtype)
    assert km.km_assign_uses_tensor_cores(X, Cx) == ((dt, B, N, K, d) in TC_CASES)
    ids, mind, inertia = km.km_assign(X, Cx, cn, w=w, want_mind=True, want_inertia=True)
    torch.cuda.synchronize()
    near = check_assign(X, C, ids, w=w, mind_gpu=mind, inertia_gpu=inertia)
    # near-ties (allowed to differ) depend on the data only; they stay a small minority here
    assert near <= max(2, B * N // 20)
    # without cn the kernel computes the norms itself; without mind/inertia it skips ||x||^2
    ids2, _, _ = km.km_assign(X, Cx)
    torch.cuda.synchronize()
    check_assign(X, C, ids2)


@pytest.mark.parametrize("dt,B,N,K,d", [("f16", 2, 3000, 300, 128), ("bf16", 3, 777, 64, 64),
                                         ("f32", 1, 4096, 32, 16), ("f16", 1, 129, 1, 128),
                                         ("f16", 2, 1000, 50, 12), ("f16", 1, 5000, 2, 128)])
def test_assign_counts_and_the_update_that_reuses_them(dt, B, N, K, d, cuda_device):
    """km_assign's per-cluster counts equal a histogram of its ids (exact), and the update fed
    those counts (counts_ready) gives the same centroids as the one that counts for itself."""
    dtype = DT[dt]
    X, C = mixture(B, N, d, K, dtype, cuda_device, seed=31 + N + K)
    Cx, cn = km.km_prep(C, dtype)
    counts = torch.full((B, K), -7, dtype=torch.int32, device=cuda_device)   # overwritten
    ids, _, _ = km.km_assign(X, Cx, cn, counts=counts)
    torch.cuda.synchronize()
    g = to_np(ids)
    for b in range(B):
        np.testing.assert_array_equal(to_np(counts[b]), np.bincount(g[b], minlength=K))
    Cx1, cn1, Cx2, cn2 = (torch.empty_like(t) for t in (Cx, cn, Cx, cn))
    C1, c1, _ = km.km_update_next(X, ids, C, Cx1, cn1)
    C2, c2, _ = km.km_update_next(X, ids, C, Cx2, cn2, counts=counts.clone(), counts_ready=True)
    torch.cuda.synchronize()
    assert torch.equal(c1, counts) and torch.equal(c2, counts)
    torch.testing.assert_close(C2, C1, rtol=1e-5, atol=1e-6)
    check_update(X, ids, C, C2, c2)


def test_tensor_core_distance_precision_bound(cuda_device):
    """Centroids almost on top of their points: the reported distance comes from the expanded
    form ||x||^2 + ||c||^2 - 2<x,c> in fp32, so its absolute error is bounded by a small multiple
    of 2^-24 (||x||^2 + ||c||^2), not by a fraction of the (tiny) distance itself. The
    assignment itself stays exact away from near-ties."""
    X, C = mixture(2, 2000, 128, 300, torch.float16, cuda_device, seed=11, c_noise=0.01)
    Cx, cn = km.km_prep(C, torch.float16)
    ids, mind, _ = km.km_assign(X, Cx, cn, want_mind=True)
    torch.cuda.synchronize()
    check_assign(X, C, ids, mind_gpu=mind)     # mind checked against 1e-5 * (||x||^2 + ||c||^2)


@pytest.mark.parametrize("dt,d", [("f16", 128), ("bf16", 64), ("f32", 16), ("f16", 12)])
def test_duplicate_centroids_go_to_lowest_index(dt, d, cuda_device):
    dtype = DT[dt]
    X, C = mixture(1, 2000, d, 300, dtype, cuda_device, seed=5)
    C[0, 290] = C[0, 3]      # duplicates in different centroid tiles
    C[0, 150] = C[0, 3]
    Cx, cn = km.km_prep(C, dtype)
    ids, _, _ = km.km_assign(X, Cx, cn)
    torch.cuda.synchronize()
    g = to_np(ids)
    assert not (g == 290).any() and not (g == 150).any()
    ids_ref, d1, d2, _ = oracle.assign(oracle.as_f64(X.cpu()), oracle.round_to_dtype(C.cpu(), dtype))
    np.testing.assert_array_equal(g[ids_ref == 3], 3)


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_duplicates_in_later_tiles_and_earlier_column_quarters(dt, cuda_device):
    """K = 1024 in 256-column tiles: each copy below sits in a later tile than its original and
    in a column quarter that the per-row merge visits first (or in another half of the split
    tile), so the lowest index must win on the (value, index) order, not on the visiting order."""
    dtype = DT[dt]
    X, C = mixture(1, 4000, 128, 1024, dtype, cuda_device, seed=11)
    g = torch.Generator().manual_seed(12)
    pairs = [(100, 300), (140, 260), (70, 600), (200, 1000), (5, 900)]
    rows = []
    for lo, hi in pairs:
        C[0, hi] = C[0, lo]
        near = C[0, lo].cpu() + 0.01 * torch.randn((100, 128), generator=g)
        rows.append(near)
    X[0, :500] = torch.cat(rows).to(dtype).to(cuda_device)
    Cx, cn = km.km_prep(C, dtype)
    ids, _, _ = km.km_assign(X, Cx, cn)
    torch.cuda.synchronize()
    got = to_np(ids)[0]
    ids_ref, _, _, _ = oracle.assign(oracle.as_f64(X.cpu()), oracle.round_to_dtype(C.cpu(), dtype))
    ref = ids_ref[0]
    for lo, hi in pairs:
        assert not (got == hi).any()
        np.testing.assert_array_equal(got[ref == lo], lo)
    assert sum((ref == lo).sum() for lo, _ in pairs) >= 400


@pytest.mark.parametrize("dt,d,K", [("f16", 128, 300), ("bf16", 128, 300), ("f16", 64, 100),
                                     ("f16", 256, 60), ("bf16", 8, 300), ("f32", 16, 300)])
def test_points_on_duplicate_centroids_take_lowest_index(dt, d, K, cuda_device):
    """Points placed exactly on a centroid that occurs several times: every copy is at distance 0,
    so the tie rule alone decides, and it must give the lowest index. The copies sit in the same
    column group of one tile, in other column groups and in other tiles. (The oracle's near-tie
    exemption covers d2 = 0, so this is asserted directly, not through check_assign.)"""
    dtype = DT[dt]
    X, C = mixture(1, 3000, d, K, dtype, cuda_device, seed=17)
    C = C.to(dtype).float()                  # representable, so a point can equal its centroid
    groups = {3: [4, 40 % K, 130 % K, (K - 10)], (K // 3): [K // 3 + 1, K // 3 + 20]}
    for lo, dups in groups.items():
        for k in dups:
            if k != lo:
                C[0, k] = C[0, lo]
    g = torch.Generator().manual_seed(23)
    pos = torch.randperm(3000, generator=g)[:600].to(cuda_device)
    owner = torch.tensor(list(groups), device=cuda_device)[torch.arange(600, device=cuda_device) % 2]
    X[0, pos] = C[0, owner].to(dtype)
    Cx, cn = km.km_prep(C, dtype)
    ids, mind, _ = km.km_assign(X, Cx, cn, want_mind=True)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_np(ids[0, pos]), to_np(owner))
    # the same bound as every other distance check: 1e-5 (||x||^2 + ||c||^2), here 2e-5 ||x||^2
    xn = (X[0, pos].float() ** 2).sum(-1)
    assert bool((mind[0, pos] <= 2e-5 * xn + 1e-30).all())
    # the labels-only form takes the same decisions
    ids2, _, _ = km.km_assign(X, Cx, cn)
    torch.cuda.synchronize()
    assert torch.equal(ids2, ids)


def test_all_points_identical(cuda_device):
    X = torch.full((1, 700, 128), 0.5, dtype=torch.float16, device=cuda_device)
    C = torch.randn((1, 300, 128), device=cuda_device)
    C[0, 123] = 0.5
    Cx, cn = km.km_prep(C, torch.float16)
    ids, mind, _ = km.km_assign(X, Cx, cn, want_mind=True)
    torch.cuda.synchronize()
    assert (ids == 123).all()
    assert float(mind.max()) < 1e-2


# ------------------------------------------------------------------ update

UPD_CASES = [
    ("f16", 2, 3000, 300, 128),
    ("bf16", 1, 5000, 64, 64),
    ("f32", 1, 4096, 32, 16),
    ("f16", 3, 1000, 50, 12),
    ("f16", 1, 800, 20, 300),
    ("f32", 2, 600, 17, 1),
    ("f16", 1, 100, 400, 128),       # K > N: empty clusters keep their centroid
    ("f16", 1, 20000, 3, 32),        # few huge segments spanning many warps
    # the fused reduce-and-divide form (rows of 128, 256, 512 bytes)
    ("f16", 1, 200000, 3, 128),      # three segments, each split over many ranges
    ("f32", 2, 3000, 100, 64),
    ("f32", 1, 5000, 40, 128),
    ("f16", 1, 3000, 70, 256),
    ("bf16", 3, 2000, 1, 128),       # K = 1: one segment per problem
    ("f32", 1, 1000, 10, 32),
    ("bf16", 40, 700, 30, 64),       # more problems than ranges per problem
    ("f16", 1, 30000, 20000, 128),   # K above the 16384 shared-memory bins: the two-launch sort
    ("f16", 2, 20000, 4096, 128),    # the largest K whose scatter tiles are sorted in shared memory
    ("bf16", 1, 20000, 4097, 64),    # one above: labels ranked straight into perm
    ("f16", 1, 40000, 16384, 128),   # the largest K whose counts are scanned in shared memory
    ("f16", 1, 40000, 16385, 64),    # one above: the separate scan launch
]


@pytest.mark.parametrize("dt,B,N,K,d", UPD_CASES)
@pytest.mark.parametrize("weighted", [False, True])
def test_update_matches_oracle(dt, B, N, K, d, weighted, cuda_device):
    dtype = DT[dt]
    X, C = mixture(B, N, d, K, dtype, cuda_device, seed=N + K)
    w = (torch.rand((B, N), device=cuda_device) * 2 + 0.01) if weighted else None
    Cx, cn = km.km_prep(C, dtype)
    ids, _, _ = km.km_assign(X, Cx, cn)
    C_new, counts, wsum = km.km_update(X, ids, C, w=w, want_wsum=True)
    torch.cuda.synchronize()
    check_update(X, ids, C, C_new, counts, w=w, wsum_gpu=wsum)
    # partial + finalize is the same computation split in two
    sums, ws2, c2 = km.km_update_partial(X, ids, K, w=w)
    C2, Cx2, cn2 = km.km_finalize(sums, c2, C, wsum=ws2, cx_dtype=dtype)
    torch.cuda.synchronize()
    assert torch.equal(c2, counts)
    torch.testing.assert_close(C2, C_new, rtol=1e-5, atol=1e-6)
    assert torch.equal(Cx2, C2.to(dtype))


@pytest.mark.parametrize("dt,B,N,K,d", [("f16", 2, 3000, 300, 128), ("bf16", 1, 50000, 5, 64),
                                         ("f32", 1, 4000, 33, 16), ("f16", 1, 100, 400, 128)])
@pytest.mark.parametrize("weighted", [False, True])
def test_update_next_writes_the_next_assignment_inputs(dt, B, N, K, d, weighted, cuda_device):
    """km_update_next = km_update plus the rounded centroids and their norms in one pass."""
    dtype = DT[dt]
    X, C = mixture(B, N, d, K, dtype, cuda_device, seed=7 + N)
    w = (torch.rand((B, N), device=cuda_device) * 2 + 0.01) if weighted else None
    Cx, cn = km.km_prep(C, dtype)
    ids, _, _ = km.km_assign(X, Cx, cn)
    C_ref, counts_ref, wsum_ref = km.km_update(X, ids, C, w=w, want_wsum=True)
    Cx2 = torch.empty_like(Cx)
    cn2 = torch.empty_like(cn)
    C_new, counts, wsum = km.km_update_next(X, ids, C, Cx2, cn2, w=w, want_wsum=True)
    torch.cuda.synchronize()
    check_update(X, ids, C, C_new, counts, w=w, wsum_gpu=wsum)
    assert torch.equal(counts, counts_ref)
    torch.testing.assert_close(C_new, C_ref, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(wsum, wsum_ref, rtol=1e-5, atol=1e-6)
    assert torch.equal(Cx2, C_new.to(dtype))
    torch.testing.assert_close(cn2.double(), (Cx2.double() ** 2).sum(-1), rtol=2e-6, atol=0)
    # in place (C_new aliases C_prev), as a fit runs it
    C_in = C.clone()
    km.km_update_next(X, ids, C_in, Cx2, cn2, w=w, C_new=C_in)
    torch.cuda.synchronize()
    torch.testing.assert_close(C_in, C_ref, rtol=1e-5, atol=1e-6)


def test_update_in_place_and_random_ids(cuda_device):
    g = torch.Generator().manual_seed(3)
    X = torch.randn((2, 10000, 64), generator=g).half().to(cuda_device)
    ids = torch.randint(0, 50, (2, 10000), generator=g).int().to(cuda_device)
    ids[0, :9000] = 7                                   # one hot cluster
    C = torch.randn((2, 60, 64), generator=g).to(cuda_device)   # clusters 50..59 empty
    C_prev = C.clone()
    _, counts, _ = km.km_update(X, ids, C, C_new=C)      # in place
    torch.cuda.synchronize()
    check_update(X, ids, C_prev, C, counts)


# ------------------------------------------------------------------ fits

@pytest.mark.parametrize("K", [16, 8])
def test_fit1d_weighted_rows_per_iteration(K, cuda_device):
    d = synth.make_workload(2, B=48, N=4096, device="cpu")
    X, w = d["X"].to(cuda_device), d["w"].to(cuda_device)
    C = km.km_init_grid1d(X, K)
    C0 = C.clone()
    iters = 30
    _, ids, ih, ch = km.km_fit(X, C, iters, w=w, want_ids=True, want_inertia=True, want_hist=True)
    torch.cuda.synchronize()
    assert torch.equal(ch[0], C0) and torch.equal(ch[-1], C)
    X64, w64 = oracle.as_f64(X.cpu()), oracle.as_f64(w.cpu())
    hist = to_np(ch).astype(np.float64)
    for t in range(iters):
        Ct = hist[t]
        ids_t, d1, d2, inertia = oracle.assign(X64, oracle.round_to_dtype(Ct, torch.float16), w64)
        np.testing.assert_allclose(to_np(ih[t]), inertia, rtol=1e-4)
        C_ref, _, _ = oracle.update(X64, ids_t, Ct, w64)
        for b in range(C_ref.shape[0]):
            err = np.linalg.norm(hist[t + 1][b] - C_ref[b]) / np.linalg.norm(C_ref[b])
            assert err <= 1e-3, (t, b, err)
    check_assign(X, C, ids)


@pytest.mark.parametrize("dt,N,K,weighted", [
    ("f32", 3000, 32, True),    # warp-per-row form at its largest K; ragged radix segments
    ("bf16", 1000, 5, False),
    ("f16", 8192, 1, True),     # the largest row; one cluster
    ("f16", 700, 48, True),     # K > 32: the fused one-CTA-per-row form
    ("f16", 2000, 20, True),    # 12 unused centroid registers of the 32-wide form
    ("bf16", 1500, 12, False),  # 4 unused of the 16-wide form
])
def test_fit1d_shapes_per_iteration(dt, N, K, weighted, cuda_device):
    g = torch.Generator().manual_seed(N + K)
    B = 6
    X = (torch.randn((B, N, 1), generator=g) * 0.05).to(DT[dt])
    X[:, : N // 10] = X[:, N // 10: 2 * (N // 10)]          # repeated values (ties in the sort)
    w = torch.rand((B, N), generator=g) + 0.01 if weighted else None
    Xd = X.to(cuda_device)
    wd = None if w is None else w.to(cuda_device)
    C = km.km_init_grid1d(Xd, K)
    iters = 6
    _, ids, ih, ch = km.km_fit(Xd, C, iters, w=wd, want_ids=True, want_inertia=True, want_hist=True)
    torch.cuda.synchronize()
    X64 = oracle.as_f64(X)
    w64 = None if w is None else oracle.as_f64(w)
    hist = to_np(ch).astype(np.float64)
    for t in range(iters):
        ids_t, d1, d2, inertia = oracle.assign(X64, oracle.round_to_dtype(hist[t], DT[dt]), w64)
        np.testing.assert_allclose(to_np(ih[t]), inertia, rtol=1e-4)
        C_ref, _, _ = oracle.update(X64, ids_t, hist[t], w64)
        for b in range(B):
            err = np.linalg.norm(hist[t + 1][b] - C_ref[b]) / max(np.linalg.norm(C_ref[b]), 1e-30)
            assert err <= 1e-3, (t, b, err)
    check_assign(Xd, C, ids, w=wd)


def test_fit1d_unweighted_fp32_and_worked_example(cuda_device):
    from conftest import load_golden
    gold = load_golden("worked_example_weight_clustering.txt")
    vals = torch.tensor([float(v) for v in gold["values"]], dtype=torch.float32)
    X = vals.reshape(1, -1, 1).to(cuda_device)
    C = km.km_init_grid1d(X, 3)
    _, ids, ih, _ = km.km_fit(X, C, 3, want_ids=True, want_inertia=True)
    torch.cuda.synchronize()
    got = np.sort(to_np(C)[0, :, 0])
    printed = np.sort([float(v) for v in gold["centroids"]])
    np.testing.assert_allclose(got, printed, atol=0.5e-4)
    lab = to_np(ids)[0]
    assert len(set(lab[:5])) == 1 and len(set(lab[5:10])) == 1 and lab[0] != lab[5]
    assert to_np(ih)[1, 0] == pytest.approx(2.444e-6, rel=1e-2)


@pytest.mark.parametrize("case", ["config1", "config3_small", "d1_generic"])
def test_fit_generic_per_iteration(case, cuda_device):
    if case == "config1":
        d = synth.make_workload(1, device="cpu")
        X, C, w = d["X"], d["C0"], None
        iters = d["iters"]
    elif case == "config3_small":
        d = synth.make_workload(3, B=2, N=8192, K=256, device="cpu")
        X, C, w = d["X"], d["C0"], None
        iters = 3
    else:   # d = 1 with N beyond the fused per-row kernel: the generic chain
        d = synth.make_workload(2, B=3, N=9000, device="cpu")
        X, w = d["X"], d["w"]
        C = torch.from_numpy(oracle.grid_init(X, 16).astype(np.float32))
        iters = 5
    X, C = X.to(cuda_device), C.to(cuda_device)
    w = None if w is None else w.to(cuda_device)
    dtype = X.dtype
    _, ids, ih, ch = km.km_fit(X, C, iters, w=w, want_ids=True, want_inertia=True, want_hist=True)
    torch.cuda.synchronize()
    X64 = oracle.as_f64(X.cpu())
    w64 = None if w is None else oracle.as_f64(w.cpu())
    hist = to_np(ch).astype(np.float64)
    for t in range(iters):
        ids_t, d1, d2, inertia = oracle.assign(X64, oracle.round_to_dtype(hist[t], dtype), w64)
        np.testing.assert_allclose(to_np(ih[t]), inertia, rtol=1e-4)
        # Iteration t's assignment, recomputed from the same centroids (the kernels are
        # deterministic): equal to the oracle's except at near ties, where either answer is
        # correct. The update is then checked against the oracle update of that assignment,
        # since a single near-tie point moves two centroids of a small cluster visibly.
        Ct = ch[t].contiguous()
        Cx, cn = km.km_prep(Ct, dtype)
        ids_g, _, _ = km.km_assign(X, Cx, cn, w=w)
        torch.cuda.synchronize()
        g = to_np(ids_g)
        near = oracle.near_tie(d1, d2)
        assert not ((g != ids_t) & ~near).any(), t
        assert near.mean() <= 0.03, (t, near.mean())
        C_ref, _, _ = oracle.update(X64, g.astype(np.int32), hist[t], w64)
        for b in range(C_ref.shape[0]):
            err = np.linalg.norm(hist[t + 1][b] - C_ref[b]) / np.linalg.norm(C_ref[b])
            assert err <= 1e-3, (t, b, err)
    check_assign(X, C, ids)


def test_fit_host_matches_device(cuda_device):
    d = synth.make_workload(3, B=2, N=5000, K=200, device="cpu")
    X, C0 = d["X"], d["C0"]
    Xh = X.pin_memory()
    Ch = C0.clone().pin_memory()
    idsh = torch.empty((2, 5000), dtype=torch.int32).pin_memory()
    inh = torch.empty((4, 2), dtype=torch.float64).pin_memory()
    km.km_fit_host(Xh, Ch, 4, ids_host=idsh, inertia_host=inh)
    Cd = C0.to(cuda_device)
    _, ids, ih, _ = km.km_fit(X.to(cuda_device), Cd, 4, want_ids=True, want_inertia=True)
    torch.cuda.synchronize()
    torch.testing.assert_close(Ch, Cd.cpu(), rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(inh.numpy(), to_np(ih), rtol=1e-9)
    assert (idsh.numpy() != to_np(ids)).mean() < 1e-3


@pytest.mark.parametrize("dtype,N,weighted", [(torch.float16, 262144, False),
                                               (torch.bfloat16, 270001, True)])
def test_fit_host_single_iteration_streamed(dtype, N, weighted, cuda_device):
    # X of 64 MiB or more, one iteration, no labels: km_fit_host streams X in 16 chunks (the last
    # one ragged for N = 270001); the result matches the resident fit up to summation order
    B, K, d = 1, 1024, 128
    g = torch.Generator().manual_seed(11)
    X = (torch.randn(B, N, d, generator=g) * 2).to(dtype)
    C0 = X[:, torch.randperm(N, generator=g)[:K]].float().contiguous()
    w = torch.rand(B, N, generator=g) + 0.5 if weighted else None
    Xh, Ch = X.pin_memory(), C0.clone().pin_memory()
    wh = w.pin_memory() if weighted else None
    inh = torch.empty((1, B), dtype=torch.float64).pin_memory()
    km.km_fit_host(Xh, Ch, 1, w_host=wh, inertia_host=inh)
    Cd = C0.to(cuda_device)
    _, _, ih, _ = km.km_fit(X.to(cuda_device), Cd, 1, w=w.to(cuda_device) if weighted else None,
                            want_inertia=True)
    torch.cuda.synchronize()
    torch.testing.assert_close(Ch, Cd.cpu(), rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(inh.numpy(), to_np(ih), rtol=1e-9)


STREAM_CASES = {
    # (dtype, B, N, K, d, chunk, weighted): ragged last chunk, several tiles per chunk
    "f16_tc": (torch.float16, 2, 5000, 300, 128, 1536, False),
    "f32_exact_weighted": (torch.float32, 3, 3000, 64, 32, 700, True),
    "bf16_one_chunk": (torch.bfloat16, 1, 2500, 130, 64, 4096, True),
}


@pytest.mark.parametrize("case", list(STREAM_CASES))
def test_fit_stream_per_iteration(case, cuda_device):
    dtype, B, N, K, d, chunk, weighted = STREAM_CASES[case]
    X, C = mixture(B, N, d, K, dtype, "cpu", seed=11)
    g = torch.Generator().manual_seed(5)
    w = torch.rand((B, N), generator=g) * 2 + 0.05 if weighted else None
    Xh = X.pin_memory()
    wh = None if w is None else w.pin_memory()
    Xd = X.to(cuda_device)
    wd = None if w is None else w.to(cuda_device)
    X64 = oracle.as_f64(X)
    w64 = None if w is None else oracle.as_f64(w)
    Cd = C.to(cuda_device)
    for t in range(3):
        C_prev = Cd.clone()
        _, ih = km.km_fit_stream(Xh, Cd, 1, chunk, w_host=wh, want_inertia=True)
        torch.cuda.synchronize()
        Cp = to_np(C_prev).astype(np.float64)
        ids_t, d1, d2, inertia = oracle.assign(X64, oracle.round_to_dtype(Cp, dtype), w64)
        np.testing.assert_allclose(to_np(ih[0]), inertia, rtol=1e-4)
        # the same assignment on the resident points (deterministic kernels): oracle ids
        # except at near ties; the update of that assignment is the oracle's
        Cx, cn = km.km_prep(C_prev, dtype)
        ids_g, _, _ = km.km_assign(Xd, Cx, cn, w=wd)
        torch.cuda.synchronize()
        ig = to_np(ids_g)
        assert not ((ig != ids_t) & ~oracle.near_tie(d1, d2)).any(), t
        C_ref, _, _ = oracle.update(X64, ig.astype(np.int32), Cp, w64)
        Cn = to_np(Cd).astype(np.float64)
        for b in range(B):
            err = np.linalg.norm(Cn[b] - C_ref[b]) / np.linalg.norm(C_ref[b])
            assert err <= 1e-3, (t, b, err)


def test_fit_stream_matches_resident_fit(cuda_device):
    d = synth.make_workload(3, B=2, N=6000, K=256, device="cpu")
    X, C0 = d["X"], d["C0"]
    Cs = C0.to(cuda_device)
    _, ih_s = km.km_fit_stream(X.pin_memory(), Cs, 4, 1000, want_inertia=True)
    Cr = C0.to(cuda_device)
    _, _, ih_r, _ = km.km_fit(X.to(cuda_device), Cr, 4, want_inertia=True)
    torch.cuda.synchronize()
    # only the order of the fp32 accumulation differs (per chunk, then across chunks)
    torch.testing.assert_close(Cs, Cr, rtol=1e-4, atol=1e-5)
    np.testing.assert_allclose(to_np(ih_s), to_np(ih_r), rtol=1e-5)
    # zero iterations leave C untouched
    C_keep = Cs.clone()
    km.km_fit_stream(X.pin_memory(), Cs, 0, 1000)
    torch.cuda.synchronize()
    assert torch.equal(Cs, C_keep)


def test_fit_k_greater_than_n_keeps_empty(cuda_device):
    X, C = mixture(1, 50, 32, 80, torch.float16, cuda_device, seed=9)
    C0 = C.clone()
    _, ids, _, ch = km.km_fit(X, C, 2, want_ids=True, want_hist=True)
    torch.cuda.synchronize()
    assert len(set(to_np(ids)[0].tolist())) <= 50
    # a centroid that never received a point in either iteration equals its start
    ids0, _, _, _ = oracle.assign(oracle.as_f64(X.cpu()), oracle.round_to_dtype(C0.cpu(), torch.float16))
    never = np.setdiff1d(np.arange(80), np.unique(ids0[0]))
    ids1, _, _, _ = oracle.assign(oracle.as_f64(X.cpu()), oracle.round_to_dtype(ch[1].cpu(), torch.float16))
    never = np.setdiff1d(never, np.unique(ids1[0]))
    np.testing.assert_array_equal(to_np(C)[0, never], to_np(C0)[0, never])


@pytest.mark.parametrize("d", [32, 64])   # 64-byte rows: the sums-array update; 128: the fused one
def test_more_problems_than_the_grid_y_limit(d, cuda_device):
    # 65600 problems: the launches that put problems on the grid's y axis (65535 at most) run
    # in slices; every problem must come out as if it were alone
    B, N, K = 65600, 32, 4
    X, C = mixture(B, N, d, K, torch.float16, cuda_device, seed=5)
    Cx, cn = km.km_prep(C, torch.float16)
    ids, _, _ = km.km_assign(X, Cx, cn)
    C_new, counts, _ = km.km_update(X, ids, C)
    torch.cuda.synchronize()
    check_assign(X, C, ids)
    check_update(X, ids, C, C_new, counts)
    # 1-D encoding of as many rows
    vals = X[:, :, 0].contiguous()
    cents = C[:, :, 0].contiguous()
    codes = km.km_encode1d(vals, cents)
    torch.cuda.synchronize()
    from oracle import codebook1d
    ref, d1, d2 = codebook1d.encode1d(oracle.as_f64(vals.cpu()), oracle.as_f64(cents.cpu()), torch.float16)
    assert not ((to_np(codes) != ref) & ~oracle.near_tie(d1, d2)).any()
