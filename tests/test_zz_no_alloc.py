"""km_update_noalloc: the update for callers that cannot allocate device memory.

Some callers must not call cudaMalloc/cudaFree where they run the update (those calls can
synchronise the device and stall other streams, and some embeddings give the library no
allocator), so they cannot provide a workspace. This entry point keeps its scratch in a fixed
32 MiB array inside the library instead. The test calls it through the C ABI twice in a row and
compares each result with km_update's (which takes a caller workspace) on the same inputs.
This file is collected last so a failure here never hides the other tests.
"""
import ctypes

import pytest
import torch

import exact_lloyd_means_assign_b200 as km
from parity import mixture

pytestmark = pytest.mark.gpu

KM_ERR_WORKSPACE = 3


def _call_noalloc(X, ids, C_prev, w, C_new, counts, wsum):
    B, N, d = X.shape
    K = C_prev.shape[1]
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return km._load().km_update_noalloc(
        P(X), km._dt(X.dtype), P(ids), P(w), B, N, K, d, P(C_prev), P(C_new), P(counts), P(wsum),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_update_matches_workspace_update_twice(cuda_device):
    torch.cuda.set_device(cuda_device)
    cases = [(torch.float16, 2, 3000, 300, 128, True), (torch.float32, 3, 1000, 50, 12, False)]
    for i, (dtype, B, N, K, d, weighted) in enumerate(cases):
        X, C = mixture(B, N, d, K, dtype, cuda_device, seed=100 + i)
        w = (torch.rand((B, N), device=cuda_device) + 0.05) if weighted else None
        Cx, cn = km.km_prep(C, dtype)
        ids, _, _ = km.km_assign(X, Cx, cn)
        C_ref, counts_ref, wsum_ref = km.km_update(X, ids, C, w=w, want_wsum=True)
        # outputs are the caller's; they exist before the call is measured
        C_new = torch.empty_like(C)
        counts = torch.empty((B, K), dtype=torch.int32, device=cuda_device)
        wsum = torch.empty((B, K), dtype=torch.float32, device=cuda_device)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info(cuda_device)[0]
        st = _call_noalloc(X, ids, C, w, C_new, counts, wsum)
        torch.cuda.synchronize()
        free_after = torch.cuda.mem_get_info(cuda_device)[0]
        assert st == 0, km.km_status_string(st)
        # the call itself took no device memory
        assert free_after == free_before
        assert torch.equal(counts, counts_ref)
        torch.testing.assert_close(C_new, C_ref, rtol=1e-5, atol=1e-6)
        torch.testing.assert_close(wsum, wsum_ref, rtol=1e-5, atol=1e-6)
    assert km.km_device_error() == 0


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_device):
    lib = km._load()
    need = lib.km_noalloc_scratch_needed(1, 1 << 24, 4096, 128)
    assert need > 32 * 1024 * 1024
    fake = ctypes.c_void_p(0x10000)      # never touched: the size check fails first
    st = lib.km_update_noalloc(fake, 1, fake, None, 1, 1 << 24, 4096, 128, fake, fake, fake, None,
                               ctypes.c_void_p(0))
    assert st == KM_ERR_WORKSPACE
