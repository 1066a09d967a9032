"""The seeded input generators (CPU): deterministic, shaped and distributed as each workload's
recipe states, and free of any k-means arithmetic."""
import numpy as np
import pytest
import torch

import synth


@pytest.mark.parametrize("idx,kw", [(1, {}), (2, {"B": 6, "N": 500}), (3, {"B": 2, "N": 2000}),
                                    (4, {"N": 3000, "K": 64}), (5, {"N": 5000, "K": 32})])
def test_workloads_are_deterministic_and_shaped(idx, kw):
    a = synth.make_workload(idx, **kw)
    b = synth.make_workload(idx, **kw)
    wl = synth.WORKLOADS[idx]
    assert a["X"].dtype == wl.dtype and a["X"].shape == (a["B"], a["N"], wl.d)
    assert torch.equal(a["X"], b["X"])
    if wl.weighted:
        assert a["w"].shape == (a["B"], a["N"]) and torch.equal(a["w"], b["w"])
        assert float(a["w"].min()) > 0
    else:
        assert a["w"] is None
    if wl.init == "grid":
        assert a["C0"] is None
    else:
        assert a["C0"].dtype == torch.float32 and a["C0"].shape == (a["B"], a["K"], wl.d)
        assert torch.equal(a["C0"], b["C0"])
    c = synth.make_workload(idx, seed=99, **kw)
    assert not torch.equal(a["X"], c["X"])


def test_more_centroids_than_points_is_refused():
    with pytest.raises(ValueError):
        synth.make_workload(3, B=1, N=100, K=200)


def test_initial_centroids_are_distinct_points():
    d = synth.make_workload(3, B=2, N=2000, K=50)
    X, C0 = d["X"].float(), d["C0"]
    for b in range(2):
        rows = {tuple(r) for r in X[b].numpy().tolist()}
        assert all(tuple(c) in rows for c in C0[b].numpy().tolist())
        assert len({tuple(c) for c in C0[b].numpy().tolist()}) == 50


def test_rows_workload_distribution():
    d = synth.make_workload(2, B=64, N=4096)
    x = d["X"].float().numpy().ravel()
    # Student-t(5) x 0.02: symmetric, heavier tails than a normal of the same scale
    assert abs(np.median(x)) < 2e-3
    q99 = np.quantile(np.abs(x), 0.99)
    assert 0.02 * 3.0 < q99 < 0.02 * 5.5       # t(5): |x| 99th percentile is 4.03 scales
    w = d["w"].numpy().ravel()
    assert w.min() >= 1e-3 and abs(w.mean() - (1.0 + 1e-3)) < 0.05   # N(0,1)^2 + 1e-3
