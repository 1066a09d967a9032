"""The failure path of the bounded waits, on the GPU, without a fault.

Every wait inside the kernels gives up after a limit, records bit 0 in the device error word and
lets its kernel leave cleanly. Here the limit is cut to 20 ms and a test-only switch makes the
tensor-core assignment withhold one point tile, so a wait must run out: the call returns, the
error word reports the timeout, and the next normal assignment (which allocates the same tensor
memory) runs and matches the oracle, i.e. the aborted kernel drained its copies and MMAs and
freed tensor memory. The switch and the limit are restored whatever happens.
"""
import time

import pytest
import torch

import exact_lloyd_means_assign_b200 as km
from parity import check_assign, mixture

pytestmark = pytest.mark.gpu


def test_withheld_tile_times_out_and_the_next_call_is_clean(cuda_device):
    torch.cuda.set_device(cuda_device)
    X, C = mixture(2, 3000, 128, 300, torch.float16, cuda_device, seed=41)
    Cx, cn = km.km_prep(C, torch.float16)
    assert km.km_assign_uses_tensor_cores(X, Cx)
    assert km.km_device_error() == 0
    old = km.km_debug_wait_limit(20_000_000)          # 20 ms
    try:
        km.km_debug_inject(1)
        t = time.perf_counter()
        km.km_assign(X, Cx, cn)
        code = km.km_device_error()                    # synchronises
        elapsed = time.perf_counter() - t
    finally:
        km.km_debug_inject(0)
        km.km_debug_wait_limit(old)
    assert code & 1, "the withheld tile must make a wait run out"
    assert elapsed < 5.0
    # the context stays usable and tensor memory was released: a normal call matches the oracle
    ids, mind, inertia = km.km_assign(X, Cx, cn, want_mind=True, want_inertia=True)
    torch.cuda.synchronize()
    check_assign(X, C, ids, mind_gpu=mind, inertia_gpu=inertia)
    assert km.km_device_error() == 0
    assert km.km_debug_wait_limit(old) == old
