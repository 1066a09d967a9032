"""CPU oracle for exact Lloyd k-means: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg import this package. The product path (``exact_lloyd_means_assign_b200``)
never imports it and shares no code with it.

The arithmetic lives in ``kmeans_oracle.c`` (plain C, fp64, OpenMP over
points). This wrapper only marshals arrays and composes the two stages into a
multi-iteration fit. Sources for each definition are cited in the C file:
Lloyd's two stages (technologypulse.uk Flash-KMeans article, "same maths, new
dataflow"), sum/count centroids (steinslab e-means daily), per-point
sample weights and the linspace grid init (LeanQuant issue "1D k-means").

Precision reading: the assignment stage compares distances to the centroids
rounded to the points' storage dtype (fp16/bf16 inputs are multiplied against
fp16/bf16 centroids on the GPU), so ``fit`` rounds C to ``assign_dtype`` before
each assignment; the arithmetic itself is fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kmeans_oracle.c")
_LIB = os.path.join(_HERE, "libkmeans_oracle.so")
_lib = None

NEAR_TIE_REL = 1e-3


def build(force=False):
    """Compile the C oracle into ``libkmeans_oracle.so`` next to this file."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
           "-o", _LIB + ".tmp", _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int64
        lib.kmo_assign.argtypes = [P, P, P, I, I, I, I, P, P, P, P]
        lib.kmo_assign.restype = None
        lib.kmo_update.argtypes = [P, P, P, P, I, I, I, I, P, P, P]
        lib.kmo_update.restype = None
        lib.kmo_grid_init.argtypes = [P, I, I, I, P]
        lib.kmo_grid_init.restype = None
        lib.kmo_threads.argtypes = []
        lib.kmo_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def threads():
    """OpenMP threads the oracle uses."""
    return int(_load().kmo_threads())


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def as_f64(a):
    """Exact upcast to a contiguous fp64 numpy array (torch tensors included)."""
    if a is None:
        return None
    try:
        import torch
        if isinstance(a, torch.Tensor):
            a = a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def round_to_dtype(C, dtype):
    """Values of C rounded (round-to-nearest-even) to ``dtype``, returned as fp64.

    ``dtype`` is a torch dtype (float16, bfloat16, float32) or None (no rounding).
    C is taken as fp32 first when it is not already fp32, matching the fp32
    master centroids that are cast for the assignment.
    """
    if dtype is None:
        return as_f64(C)
    import torch
    t = C if isinstance(C, torch.Tensor) else torch.from_numpy(np.asarray(C))
    t = t.detach().to("cpu")
    if t.dtype != torch.float32:
        t = t.to(torch.float32)
    return t.to(dtype).to(torch.float64).numpy()


def assign(X, C, w=None):
    """Assignment stage on fp64 inputs: returns (ids int32, d1, d2, inertia)."""
    X, C, w = as_f64(X), as_f64(C), as_f64(w)
    B, N, d = X.shape
    K = C.shape[1]
    assert C.shape == (B, K, d)
    ids = np.empty((B, N), np.int32)
    d1 = np.empty((B, N), np.float64)
    d2 = np.empty((B, N), np.float64)
    inertia = np.empty((B,), np.float64)
    if w is not None:
        assert w.shape == (B, N)
    _load().kmo_assign(_ptr(X), _ptr(C), _ptr(w), B, N, K, d, _ptr(ids), _ptr(d1), _ptr(d2),
                       _ptr(inertia))
    return ids, d1, d2, inertia


def update(X, ids, C_prev, w=None):
    """Update stage fed a given assignment: returns (C_new, counts int64, wsum)."""
    X, C_prev, w = as_f64(X), as_f64(C_prev), as_f64(w)
    ids = np.ascontiguousarray(np.asarray(ids, dtype=np.int32))
    B, N, d = X.shape
    K = C_prev.shape[1]
    assert ids.shape == (B, N) and C_prev.shape == (B, K, d)
    if ids.size and (ids.min() < 0 or ids.max() >= K):
        raise ValueError("ids out of range")
    C_new = np.empty((B, K, d), np.float64)
    counts = np.empty((B, K), np.int64)
    wsum = np.empty((B, K), np.float64)
    _load().kmo_update(_ptr(X), _ptr(ids), _ptr(w), _ptr(C_prev), B, N, K, d, _ptr(C_new),
                       _ptr(counts), _ptr(wsum))
    return C_new, counts, wsum


def grid_init(X, K):
    """linspace(row min, row max, K) per batch for d = 1 inputs X[B,N,1] or X[B,N]."""
    X = as_f64(X)
    if X.ndim == 3:
        assert X.shape[2] == 1
        X = np.ascontiguousarray(X[:, :, 0])
    B, N = X.shape
    C = np.empty((B, K), np.float64)
    _load().kmo_grid_init(_ptr(X), B, N, K, _ptr(C))
    return C[:, :, None]


def fit(X, C0, iters, w=None, assign_dtype=None):
    """``iters`` Lloyd iterations from C0, then one final assignment.

    Before each assignment C is rounded to ``assign_dtype`` (see module doc).
    Returns dict(C_hist [iters+1,B,K,d], inertia_hist [iters,B], ids (final
    assignment against the last centroids), counts of the last update).
    """
    X = as_f64(X)
    w = as_f64(w)
    C = as_f64(C0)
    hist = [C.copy()]
    inertias = []
    counts = None
    for _ in range(iters):
        ids, _, _, inertia = assign(X, round_to_dtype(C, assign_dtype), w)
        C, counts, _ = update(X, ids, C, w)
        hist.append(C.copy())
        inertias.append(inertia)
    ids, _, _, final_inertia = assign(X, round_to_dtype(C, assign_dtype), w)
    return {"C_hist": np.stack(hist), "inertia_hist": np.array(inertias).reshape(iters, -1),
            "ids": ids, "counts": counts, "final_inertia": final_inertia}


def near_tie(d1, d2, rel=NEAR_TIE_REL):
    """Points whose best and second-best distances differ by less than ``rel`` (relative to d2).

    Such points may legitimately be assigned differently by a kernel that
    rounds differently; everything else must match bit for bit.
    """
    d1 = np.asarray(d1)
    d2 = np.asarray(d2)
    return (d2 - d1 < rel * d2) | (d2 == 0)
