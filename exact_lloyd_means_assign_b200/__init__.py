"""exact_lloyd_means_assign_b200: exact Lloyd k-means on NVIDIA B200 (sm_100a).

A thin ctypes binding over ``libkmeans_b200.so`` (C ABI in ``include/kmeans_b200.h``). The
functions keep the C names; they only marshal torch tensors (device memory, streams) into
pointers and sizes, allocate outputs and the workspace with torch, and raise ``KMError`` on a
non-OK status. Every step of the computation runs in the library's CUDA kernels; there is no
CPU or PyTorch fallback, and the module refuses to load without the built library.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "KMError", "KM_OP_ASSIGN", "KM_OP_UPDATE", "KM_OP_FIT", "KM_OP_FIT_HOST", "lib_path",
    "km_abi_version", "km_status_string", "km_workspace_size", "km_prep", "km_assign",
    "km_update", "km_update_next", "km_update_partial", "km_finalize", "km_init_grid1d", "km_fit",
    "km_fit_host",
    "km_device_error", "km_assign_uses_tensor_cores", "workspace",
]

KM_OP_ASSIGN, KM_OP_UPDATE, KM_OP_FIT, KM_OP_FIT_HOST = 0, 1, 2, 3
_DTYPES = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libkmeans_b200.so")
_lib = None


class KMError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: {km_status_string(status)} ({status})")


def lib_path():
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(
            f"{_LIB_PATH} is missing: build it with `python -m exact_lloyd_means_assign_b200.build` "
            "(or __graft_entry__.build()); there is no fallback implementation")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I64, I, SZ, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
    sig = {
        "km_status_string": ([I], ctypes.c_char_p),
        "km_abi_version": ([], I),
        "km_workspace_size": ([I, I64, I64, I64, I64, I, I, I], SZ),
        "km_prep": ([P, I, I64, I64, I64, P, P, P], I),
        "km_assign": ([P, I, P, P, P, I64, I64, I64, I64, P, P, P, P, P, SZ, P], I),
        "km_update": ([P, I, P, P, I64, I64, I64, I64, P, P, P, P, P, SZ, P], I),
        "km_update_next": ([P, I, P, P, I64, I64, I64, I64, P, P, P, P, P, I, P, P, SZ, P], I),
        "km_update_partial": ([P, I, P, P, I64, I64, I64, I64, P, P, P, P, SZ, P], I),
        "km_finalize": ([P, P, P, P, I64, I64, I64, P, I, P, P, P], I),
        "km_init_grid1d": ([P, I, I64, I64, I64, P, P], I),
        "km_fit": ([P, I, P, I64, I64, I64, I64, P, I, P, P, P, P, SZ, P], I),
        "km_fit_host": ([P, I, P, I64, I64, I64, I64, P, I, P, P, P, SZ, P], I),
        "km_device_error": ([P, ctypes.POINTER(I)], I),
        "km_debug_wait_limit": ([ctypes.c_ulonglong, ctypes.POINTER(ctypes.c_ulonglong)], I),
        "km_debug_inject": ([I], I),
        "km_assign_uses_tensor_cores": ([I, I64, P, P], I),
        "km_update_noalloc": ([P, I, P, P, I64, I64, I64, I64, P, P, P, P, P], I),
        "km_noalloc_scratch_needed": ([I64, I64, I64, I64], SZ),
        "km_stream_workspace_size": ([I64, I64, I64, I, I, I64], SZ),
        "km_emeans_workspace_size": ([I64, I64, I64, I, I, I64], SZ),
        "km_emeans_fit": ([P, I, P, I64, I64, I64, I64, P, I64, I, F, P, F, P, P, SZ, P], I),
        "km_split_dead": ([P, P, P, F, I64, I64, I64, P, P, P, P], I),
        "km_encode1d": ([P, I, I64, I64, P, I64, P, P], I),
        "km_init_kmeanspp1d": ([P, I, P, I64, I64, I64, P, P, P, P], I),
        "km_fit_stream": ([P, I, P, I64, I64, I64, I64, P, I, I64, P, P, SZ, P], I),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    _lib = lib
    return lib


def km_status_string(status):
    return _load().km_status_string(int(status)).decode()


def km_abi_version():
    return int(_load().km_abi_version())


def _check(fn, status):
    if status != 0:
        raise KMError(fn, status)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dt(dtype):
    if dtype not in _DTYPES:
        raise ValueError(f"unsupported dtype {dtype}")
    return _DTYPES[dtype]


def _need(t, name, dtype=None, shape=None, device=None):
    if t is None:
        return
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}")


def km_workspace_size(op, B, N, K, d, dtype, weighted=False, iters=0):
    return int(_load().km_workspace_size(op, B, N, K, d, _dt(dtype), int(bool(weighted)), iters))


def workspace(op, B, N, K, d, dtype, device, weighted=False, iters=0):
    """A device buffer large enough for ``op`` (torch allocations are 512-byte aligned)."""
    n = km_workspace_size(op, B, N, K, d, dtype, weighted, iters)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def km_prep(C, dtype, Cx=None, cn=None, stream=None):
    """Cx = C rounded to ``dtype``, cn = ||Cx||^2. C: [B,K,d] fp32 (device)."""
    B, K, d = C.shape
    _need(C, "C", torch.float32)
    Cx = torch.empty((B, K, d), dtype=dtype, device=C.device) if Cx is None else Cx
    cn = torch.empty((B, K), dtype=torch.float32, device=C.device) if cn is None else cn
    _need(Cx, "Cx", dtype, (B, K, d), C.device)
    _need(cn, "cn", torch.float32, (B, K), C.device)
    _check("km_prep", _load().km_prep(_p(C), _dt(dtype), B, K, d, _p(Cx), _p(cn), _s(stream)))
    return Cx, cn


def km_assign(X, Cx, cn=None, w=None, ids=None, mind=None, inertia=None, want_mind=False,
              want_inertia=False, counts=None, ws=None, stream=None):
    """Assignment stage. X: [B,N,d], Cx: [B,K,d] same dtype. Returns (ids, mind, inertia).
    `counts` ([B,K] int32, optional) receives the number of points assigned to each cluster."""
    B, N, d = X.shape
    K = Cx.shape[1]
    dev = X.device
    _need(X, "X")
    _need(Cx, "Cx", X.dtype, (B, K, d), dev)
    _need(cn, "cn", torch.float32, (B, K), dev)
    _need(w, "w", torch.float32, (B, N), dev)
    ids = torch.empty((B, N), dtype=torch.int32, device=dev) if ids is None else ids
    if want_mind and mind is None:
        mind = torch.empty((B, N), dtype=torch.float32, device=dev)
    if want_inertia and inertia is None:
        inertia = torch.empty((B,), dtype=torch.float64, device=dev)
    _need(ids, "ids", torch.int32, (B, N), dev)
    _need(counts, "counts", torch.int32, (B, K), dev)
    if ws is None:
        ws = workspace(KM_OP_ASSIGN, B, N, K, d, X.dtype, dev)
    _check("km_assign", _load().km_assign(
        _p(X), _dt(X.dtype), _p(Cx), _p(cn), _p(w), B, N, K, d, _p(ids), _p(mind), _p(inertia),
        _p(counts), _p(ws), ws.numel(), _s(stream)))
    return ids, mind, inertia


def km_update(X, ids, C_prev, w=None, C_new=None, counts=None, wsum=None, want_wsum=False,
              ws=None, stream=None):
    """Update stage. Returns (C_new, counts, wsum)."""
    B, N, d = X.shape
    K = C_prev.shape[1]
    dev = X.device
    _need(X, "X")
    _need(ids, "ids", torch.int32, (B, N), dev)
    _need(C_prev, "C_prev", torch.float32, (B, K, d), dev)
    _need(w, "w", torch.float32, (B, N), dev)
    C_new = torch.empty_like(C_prev) if C_new is None else C_new
    counts = torch.empty((B, K), dtype=torch.int32, device=dev) if counts is None else counts
    if want_wsum and wsum is None:
        wsum = torch.empty((B, K), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(KM_OP_UPDATE, B, N, K, d, X.dtype, dev)
    _check("km_update", _load().km_update(
        _p(X), _dt(X.dtype), _p(ids), _p(w), B, N, K, d, _p(C_prev), _p(C_new), _p(counts),
        _p(wsum), _p(ws), ws.numel(), _s(stream)))
    return C_new, counts, wsum


def km_update_next(X, ids, C_prev, Cx, cn, w=None, C_new=None, counts=None, wsum=None,
                   want_wsum=False, counts_ready=False, ws=None, stream=None):
    """Update stage that also writes the next assignment's inputs: Cx (C_new rounded to X's
    dtype) and cn = ||Cx||^2, both given by the caller. With counts_ready the given `counts`
    already hold the histogram of ids (km_assign(counts=...)). Returns (C_new, counts, wsum)."""
    B, N, d = X.shape
    K = C_prev.shape[1]
    dev = X.device
    _need(X, "X")
    _need(ids, "ids", torch.int32, (B, N), dev)
    _need(C_prev, "C_prev", torch.float32, (B, K, d), dev)
    _need(Cx, "Cx", X.dtype, (B, K, d), dev)
    _need(cn, "cn", torch.float32, (B, K), dev)
    _need(w, "w", torch.float32, (B, N), dev)
    C_new = torch.empty_like(C_prev) if C_new is None else C_new
    if counts_ready and counts is None:
        raise ValueError("counts_ready needs the counts")
    counts = torch.empty((B, K), dtype=torch.int32, device=dev) if counts is None else counts
    if want_wsum and wsum is None:
        wsum = torch.empty((B, K), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(KM_OP_UPDATE, B, N, K, d, X.dtype, dev)
    _check("km_update_next", _load().km_update_next(
        _p(X), _dt(X.dtype), _p(ids), _p(w), B, N, K, d, _p(C_prev), _p(C_new), _p(Cx), _p(cn),
        _p(counts), int(bool(counts_ready)), _p(wsum), _p(ws), ws.numel(), _s(stream)))
    return C_new, counts, wsum


def km_update_partial(X, ids, K, w=None, sums=None, wsum=None, counts=None, ws=None, stream=None):
    """Per-device partial sums of the update. Returns (sums, wsum, counts)."""
    B, N, d = X.shape
    dev = X.device
    _need(ids, "ids", torch.int32, (B, N), dev)
    sums = torch.empty((B, K, d), dtype=torch.float32, device=dev) if sums is None else sums
    counts = torch.empty((B, K), dtype=torch.int32, device=dev) if counts is None else counts
    if w is not None and wsum is None:
        wsum = torch.empty((B, K), dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(KM_OP_UPDATE, B, N, K, d, X.dtype, dev)
    _check("km_update_partial", _load().km_update_partial(
        _p(X), _dt(X.dtype), _p(ids), _p(w), B, N, K, d, _p(sums), _p(wsum), _p(counts), _p(ws),
        ws.numel(), _s(stream)))
    return sums, wsum, counts


def km_finalize(sums, counts, C_prev, wsum=None, C_new=None, cx_dtype=None, Cx=None, cn=None,
                stream=None):
    """Divide (empty clusters keep C_prev); with cx_dtype (or Cx/cn given) also the rounded
    centroids and their squared norms for the next assignment. Returns (C_new, Cx, cn)."""
    B, K, d = sums.shape
    dev = sums.device
    C_new = torch.empty_like(C_prev) if C_new is None else C_new
    if Cx is not None:
        cx_dtype = Cx.dtype
    if cx_dtype is not None:
        Cx = torch.empty((B, K, d), dtype=cx_dtype, device=dev) if Cx is None else Cx
        cn = torch.empty((B, K), dtype=torch.float32, device=dev) if cn is None else cn
        _need(Cx, "Cx", cx_dtype, (B, K, d), dev)
        _need(cn, "cn", torch.float32, (B, K), dev)
    _check("km_finalize", _load().km_finalize(
        _p(sums), _p(wsum), _p(counts), _p(C_prev), B, K, d, _p(C_new),
        _dt(cx_dtype or torch.float32), _p(Cx), _p(cn), _s(stream)))
    return C_new, Cx, cn


def km_init_grid1d(X, K, C=None, stream=None):
    """linspace(min, max, K) per row of X[B,N,1] (or X[B,N]). Returns C[B,K,1] fp32."""
    B, N = X.shape[0], X.shape[1]
    _need(X, "X")
    C = torch.empty((B, K, 1), dtype=torch.float32, device=X.device) if C is None else C
    _check("km_init_grid1d", _load().km_init_grid1d(_p(X), _dt(X.dtype), B, N, K, _p(C), _s(stream)))
    return C


def km_fit(X, C, iters, w=None, want_ids=False, want_inertia=False, want_hist=False, ws=None,
           stream=None):
    """``iters`` Lloyd iterations; C [B,K,d] fp32 is updated in place.

    Returns (C, ids or None, inertia_hist [iters,B] or None, C_hist [iters+1,B,K,d] or None).
    """
    B, N, d = X.shape
    K = C.shape[1]
    dev = X.device
    _need(X, "X")
    _need(C, "C", torch.float32, (B, K, d), dev)
    _need(w, "w", torch.float32, (B, N), dev)
    ids = torch.empty((B, N), dtype=torch.int32, device=dev) if want_ids else None
    ih = torch.empty((iters, B), dtype=torch.float64, device=dev) if want_inertia and iters else None
    ch = torch.empty((iters + 1, B, K, d), dtype=torch.float32, device=dev) if want_hist else None
    if ws is None:
        ws = workspace(KM_OP_FIT, B, N, K, d, X.dtype, dev, w is not None, iters)
    _check("km_fit", _load().km_fit(
        _p(X), _dt(X.dtype), _p(w), B, N, K, d, _p(C), iters, _p(ids), _p(ih), _p(ch), _p(ws),
        ws.numel(), _s(stream)))
    return C, ids, ih, ch


def km_fit_host(X_host, C_host, iters, w_host=None, ids_host=None, inertia_host=None, ws=None,
                device=None, stream=None):
    """km_fit on host tensors (pinned for full bandwidth); synchronous. C_host is updated."""
    B, N, d = X_host.shape
    K = C_host.shape[1]
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    for t, n in ((X_host, "X_host"), (C_host, "C_host"), (w_host, "w_host"), (ids_host, "ids_host"),
                 (inertia_host, "inertia_host")):
        if t is not None and (t.device.type != "cpu" or not t.is_contiguous()):
            raise ValueError(f"{n} must be a contiguous host tensor")
    if ws is None:
        ws = workspace(KM_OP_FIT_HOST, B, N, K, d, X_host.dtype, dev, w_host is not None, iters)
    _check("km_fit_host", _load().km_fit_host(
        _p(X_host), _dt(X_host.dtype), _p(w_host), B, N, K, d, _p(C_host), iters, _p(ids_host),
        _p(inertia_host), _p(ws), ws.numel(), _s(stream)))
    return C_host


def km_fit_stream(X_host, C, iters, chunk, w_host=None, want_inertia=False, ws=None, stream=None):
    """Out-of-core fit: X_host [B,N,d] (host, pinned for overlap) streamed in chunks of `chunk`
    points per batch element every iteration; C [B,K,d] fp32 on the device, updated in place.
    Returns (C, inertia_hist [iters,B] fp64 on the device, or None). Asynchronous on `stream`."""
    B, N, d = X_host.shape
    K = C.shape[1]
    dev = C.device
    for t, n in ((X_host, "X_host"), (w_host, "w_host")):
        if t is not None and (t.device.type != "cpu" or not t.is_contiguous()):
            raise ValueError(f"{n} must be a contiguous host tensor")
    _need(C, "C", torch.float32, (B, K, d))
    inertia = torch.empty((iters, B), dtype=torch.float64, device=dev) if want_inertia and iters else None
    if ws is None:
        n = _load().km_stream_workspace_size(B, K, d, _dt(X_host.dtype), int(w_host is not None),
                                             min(chunk, N))
        ws = torch.empty(max(int(n), 1), dtype=torch.uint8, device=dev)
    _check("km_fit_stream", _load().km_fit_stream(
        _p(X_host), _dt(X_host.dtype), _p(w_host), B, N, K, d, _p(C), iters, chunk, _p(inertia),
        _p(ws), ws.numel(), _s(stream)))
    return C, inertia


def km_emeans_fit(X, C, batch, epochs, alpha0, w=None, split_u=None, split_eps=1.0 / 1024,
                  want_sse=False, ws=None, stream=None):
    """e-means run on device tensors: X [B,N,d], C [B,K,d] fp32 updated in place; split_u
    [epochs,B,K] fp32 uniforms or None. Returns (C, sse_hist [epochs,B] fp64 or None)."""
    B, N, d = X.shape
    K = C.shape[1]
    dev = X.device
    _need(X, "X")
    _need(C, "C", torch.float32, (B, K, d), dev)
    _need(w, "w", torch.float32, (B, N), dev)
    _need(split_u, "split_u", torch.float32, (epochs, B, K), dev)
    sse = torch.empty((epochs, B), dtype=torch.float64, device=dev) if want_sse and epochs else None
    if ws is None:
        n = _load().km_emeans_workspace_size(B, K, d, _dt(X.dtype), int(w is not None), min(batch, N))
        ws = torch.empty(max(int(n), 1), dtype=torch.uint8, device=dev)
    _check("km_emeans_fit", _load().km_emeans_fit(
        _p(X), _dt(X.dtype), _p(w), B, N, K, d, _p(C), batch, epochs, float(alpha0), _p(split_u),
        float(split_eps), _p(sse), _p(ws), ws.numel(), _s(stream)))
    return C, sse


def km_split_dead(C, sizes, u, eps=1.0 / 1024, Nc=None, S=None, want_donors=False, stream=None):
    """Revive clusters with sizes == 0 by proportional splitting (in place on C, sizes, Nc, S).
    C [B,K,d], sizes/u/Nc [B,K], S [B,K,d] fp32 device tensors. Returns donors [B,K] or None."""
    B, K, d = C.shape
    dev = C.device
    _need(C, "C", torch.float32, None, dev)
    _need(sizes, "sizes", torch.float32, (B, K), dev)
    _need(u, "u", torch.float32, (B, K), dev)
    _need(Nc, "Nc", torch.float32, (B, K), dev)
    _need(S, "S", torch.float32, (B, K, d), dev)
    donors = torch.empty((B, K), dtype=torch.int32, device=dev) if want_donors else None
    _check("km_split_dead", _load().km_split_dead(
        _p(C), _p(sizes), _p(u), float(eps), B, K, d, _p(Nc), _p(S), _p(donors), _s(stream)))
    return donors


def km_encode1d(X, C, codes=None, stream=None):
    """uint8 index of the nearest codebook value: X [B,N] (or [B,N,1]), C [B,K] (or [B,K,1])
    fp32 with K <= 256. Returns codes [B,N] uint8."""
    B, N = X.shape[0], X.shape[1]
    K = C.shape[1]
    _need(X, "X")
    _need(C, "C", torch.float32, None, X.device)
    codes = torch.empty((B, N), dtype=torch.uint8, device=X.device) if codes is None else codes
    _need(codes, "codes", torch.uint8, (B, N), X.device)
    _check("km_encode1d", _load().km_encode1d(_p(X), _dt(X.dtype), B, N, _p(C), K, _p(codes), _s(stream)))
    return codes


def km_init_kmeanspp1d(X, K, u, w=None, want_chosen=False, stream=None):
    """k-means++ seeds per row: X [B,N] (or [B,N,1]), u [B,K] fp32 uniforms, w [B,N] or None.
    Returns (C [B,K,1] fp32, chosen [B,K] int32 or None)."""
    B, N = X.shape[0], X.shape[1]
    _need(X, "X")
    _need(u, "u", torch.float32, (B, K), X.device)
    _need(w, "w", torch.float32, (B, N), X.device)
    C = torch.empty((B, K, 1), dtype=torch.float32, device=X.device)
    chosen = torch.empty((B, K), dtype=torch.int32, device=X.device) if want_chosen else None
    _check("km_init_kmeanspp1d", _load().km_init_kmeanspp1d(
        _p(X), _dt(X.dtype), _p(w), B, N, K, _p(u), _p(C), _p(chosen), _s(stream)))
    return C, chosen


def km_assign_uses_tensor_cores(X, Cx):
    """True when km_assign(X, Cx, ...) runs on the tensor cores."""
    return bool(_load().km_assign_uses_tensor_cores(_dt(X.dtype), X.shape[-1], _p(X), _p(Cx)))


def km_device_error(stream=None):
    """Synchronise and read/clear the device error word; returns the code (0 = none)."""
    code = ctypes.c_int(0)
    st = _load().km_device_error(_s(stream), ctypes.byref(code))
    if st not in (0, 5):
        raise KMError("km_device_error", st)
    return code.value


def km_debug_wait_limit(limit_ns):
    """Test hook: set the bound of every in-kernel wait (ns); returns the previous bound."""
    old = ctypes.c_ulonglong(0)
    _check("km_debug_wait_limit", _load().km_debug_wait_limit(int(limit_ns), ctypes.byref(old)))
    return old.value


def km_debug_inject(mode):
    """Test hook: 1 = the next tensor-core assignments withhold one point tile (waits run out);
    0 = off (the default)."""
    _check("km_debug_inject", _load().km_debug_inject(int(mode)))
