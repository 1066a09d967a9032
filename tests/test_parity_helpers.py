"""The full-size parity checks regroup the oracle's work into chunks (the 8.6 GB workload does
not fit the host as fp64 at once). These CPU tests pin that regrouping to the oracle called once
on the whole set: the chunked update must give the same counts and the same means, and the
per-cluster objective must equal the oracle's own inertia when the assignment is the oracle's.
"""
import numpy as np
import torch

import oracle
from parity import oracle_inertia_of, oracle_update_chunked


def _problem(seed=0):
    g = torch.Generator().manual_seed(seed)
    B, N, K, d = 2, 3001, 37, 24
    X = (torch.randn((B, N, d), generator=g) + 3 * torch.randint(0, 4, (B, N, 1), generator=g)).half()
    C = torch.randn((B, K, d), generator=g) * 3
    C[:, 5] = 1e3                   # nobody's nearest: an empty cluster
    return X, C


def test_chunked_update_equals_one_oracle_call():
    X, C = _problem()
    ids, _, _, _ = oracle.assign(oracle.as_f64(X), oracle.round_to_dtype(C, torch.float16))
    ids_t = torch.from_numpy(ids)
    C_ref, cnt_ref, _ = oracle.update(oracle.as_f64(X), ids, oracle.as_f64(C))
    for chunk in (1000, 3001, 1 << 21):
        C_ch, cnt = oracle_update_chunked(X, ids_t, C, chunk=chunk)
        np.testing.assert_array_equal(cnt, cnt_ref)
        np.testing.assert_allclose(C_ch, C_ref, rtol=1e-12, atol=1e-12)
    assert (cnt_ref[:, 5] == 0).all()
    np.testing.assert_array_equal(C_ch[:, 5], oracle.as_f64(C)[:, 5])


def test_inertia_of_an_assignment_equals_the_oracles_objective():
    X, C = _problem(1)
    Cr = oracle.round_to_dtype(C, torch.float16)
    ids, _, _, inertia = oracle.assign(oracle.as_f64(X), Cr)
    for chunk in (777, 1 << 21):
        got = oracle_inertia_of(X, torch.from_numpy(ids), C, torch.float16, chunk=chunk)
        np.testing.assert_allclose(got, inertia, rtol=1e-12)
    # a worse assignment (everyone to cluster 0) has a larger objective
    worse = oracle_inertia_of(X, torch.zeros_like(torch.from_numpy(ids)), C, torch.float16)
    assert (worse > inertia).all()
