"""C-ABI checks that need no GPU: the library builds/loads, exports every symbol the header
declares, sizes its workspaces consistently and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest
import torch

import exact_lloyd_means_assign_b200 as km
from exact_lloyd_means_assign_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return km._load()


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(km_[a-z0-9_]+)\s*\(",
                                src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ["km_assign", "km_update", "km_update_partial", "km_finalize", "km_fit", "km_fit_host",
              "km_init_grid1d", "km_prep", "km_workspace_size", "km_status_string",
              "km_device_error", "km_abi_version"]:
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in _declared_functions():
        assert hasattr(lib, n), n
    # exported with C linkage (no mangling)
    out = os.popen(f"nm -D --defined-only {km.lib_path()}").read()
    for n in _declared_functions():
        assert re.search(rf"\bT {n}$", out, flags=re.M), n


def test_every_declared_symbol_has_a_typed_binding(lib):
    # the binding sets argtypes/restype for each entry point it marshals; every one the header
    # declares must be covered, with as many arguments as the header's parameter list
    hdr = open(os.path.join(ROOT, "include", "kmeans_b200.h")).read()
    hdr = re.sub(r"/\*.*?\*/", "", hdr, flags=re.S)
    for n in _declared_functions():
        fn = getattr(lib, n)
        assert fn.argtypes is not None, n
        m = re.search(rf"\b{n}\s*\(([^)]*)\)", hdr)
        params = [p for p in m.group(1).split(",") if p.strip() and p.strip() != "void"]
        assert len(fn.argtypes) == len(params), (n, len(fn.argtypes), len(params))


def test_status_strings_and_version(lib):
    assert km.km_abi_version() == 2
    assert km.km_status_string(0) == "KM_OK"
    assert km.km_status_string(3) == "KM_ERR_WORKSPACE"
    assert km.km_status_string(99) == "KM_ERR_UNKNOWN"


def test_workspace_sizes(lib):
    f16, f32 = torch.float16, torch.float32
    # the exact-fp32 CUDA-core assignment needs no workspace; the tensor-core one needs one
    # 16-value bf16 augmentation row per (padded) centroid: B * ceil(K/bn)*bn * 32 bytes
    assert km.km_workspace_size(km.KM_OP_ASSIGN, 2, 100, 32, 16, f32) == 0
    assert km.km_workspace_size(km.KM_OP_ASSIGN, 2, 100, 300, 128, f16) == 2 * 512 * 32
    assert km.km_workspace_size(km.KM_OP_ASSIGN, 1, 100, 50, 128, f16) == 64 * 32
    up = km.km_workspace_size(km.KM_OP_UPDATE, 32, 65536, 1024, 128, f16)
    assert up >= 32 * 65536 * 4 + 32 * 1024 * 128 * 4
    fit = km.km_workspace_size(km.KM_OP_FIT, 32, 65536, 1024, 128, f16)
    assert fit > up
    host = km.km_workspace_size(km.KM_OP_FIT_HOST, 32, 65536, 1024, 128, f16, True, 10)
    assert host >= fit + 32 * 65536 * 128 * 2 + 32 * 65536 * 4
    for bad in [(0, 1, 1, 1), (1, 0, 1, 1), (1, 1, 0, 1), (1, 1, 1, 0), (1, 1 << 31, 1, 1)]:
        assert km.km_workspace_size(km.KM_OP_UPDATE, *bad, f16) == 0
    # streamed fit: scratch grows with the chunk, not with N; two chunk buffers of points
    s1 = lib.km_stream_workspace_size(32, 1024, 128, 1, 0, 4096)
    s2 = lib.km_stream_workspace_size(32, 1024, 128, 1, 0, 8192)
    assert 2 * 32 * 4096 * 128 * 2 <= s1 and s2 - s1 >= 2 * 32 * 4096 * 128 * 2
    assert lib.km_stream_workspace_size(32, 1024, 128, 1, 1, 4096) >= s1 + 2 * 32 * 4096 * 4
    assert lib.km_stream_workspace_size(32, 1024, 128, 1, 0, 0) == 0
    # e-means: state (S, epoch sums, batch sums) is 3 * B*K*d fp32, plus one batch's scratch
    e1 = lib.km_emeans_workspace_size(1, 65536, 128, 1, 0, 1 << 16)
    assert e1 >= 3 * 65536 * 128 * 4 + (1 << 16) * 8
    assert lib.km_emeans_workspace_size(1, 65536, 128, 1, 0, 0) == 0
    for op in range(4):
        assert km.km_workspace_size(op, 3, 1000, 17, 24, f16, True, 5) % 256 == 0


def _raw(lib):
    P = ctypes.c_void_p
    fake = P(0x10000)        # never dereferenced: validation fails first
    return P, fake


def test_argument_errors_return_before_any_launch(lib):
    P, fake = _raw(lib)
    null = None
    st = P(0)
    # km_assign: null X / Cx / ids
    assert lib.km_assign(null, 1, fake, null, null, 1, 10, 4, 8, fake, null, null, null, null, 0, st) == 1
    assert lib.km_assign(fake, 1, null, null, null, 1, 10, 4, 8, fake, null, null, null, null, 0, st) == 1
    assert lib.km_assign(fake, 1, fake, null, null, 1, 10, 4, 8, null, null, null, null, null, 0, st) == 1
    # bad dtype, bad sizes
    assert lib.km_assign(fake, 7, fake, null, null, 1, 10, 4, 8, fake, null, null, null, null, 0, st) == 1
    assert lib.km_assign(fake, 1, fake, null, null, 0, 10, 4, 8, fake, null, null, null, null, 0, st) == 1
    assert lib.km_assign(fake, 1, fake, null, null, 1, 1 << 31, 4, 8, fake, null, null, null, null, 0, st) == 1
    # misaligned fp16 pointer
    assert lib.km_assign(P(0x10001), 1, fake, null, null, 1, 10, 4, 8, fake, null, null, null, null, 0, st) == 1
    # tensor-core shape without a workspace
    assert lib.km_assign(fake, 1, fake, null, null, 1, 10, 4, 128, fake, null, null, null, null, 0, st) == 3
    # km_update: workspace too small
    assert lib.km_update(fake, 1, fake, null, 1, 10, 4, 8, fake, fake, fake, null, fake, 16, st) == 3
    # km_update_partial: weights without wsum
    assert lib.km_update_partial(fake, 1, fake, fake, 1, 10, 4, 8, fake, null, fake, fake, 1 << 20, st) == 1
    # km_fit: negative iterations, and a generic shape without workspace
    assert lib.km_fit(fake, 1, null, 1, 10, 4, 8, fake, -1, null, null, null, null, 0, st) == 1
    assert lib.km_fit(fake, 1, null, 1, 10, 4, 8, fake, 3, null, null, null, null, 0, st) == 3
    # km_fit_host: null host pointers
    assert lib.km_fit_host(null, 1, null, 1, 10, 4, 8, fake, 3, null, null, fake, 1 << 30, st) == 1
    # km_fit_stream: null host X, chunk < 1, and a workspace smaller than the chunked scratch
    assert lib.km_fit_stream(null, 1, null, 1, 10, 4, 8, fake, 3, 4, null, fake, 1 << 30, st) == 1
    assert lib.km_fit_stream(fake, 1, null, 1, 10, 4, 8, fake, 3, 0, null, fake, 1 << 30, st) == 1
    assert lib.km_fit_stream(fake, 1, null, 1, 10, 4, 8, fake, 3, 4, null, fake, 16, st) == 3
    # km_emeans_fit: batch < 1, alpha0 outside (0, 1], workspace too small
    f = ctypes.c_float
    assert lib.km_emeans_fit(fake, 1, null, 1, 10, 4, 8, fake, 0, 2, f(0.5), null, f(0.01), null,
                             fake, 1 << 30, st) == 1
    assert lib.km_emeans_fit(fake, 1, null, 1, 10, 4, 8, fake, 5, 2, f(1.5), null, f(0.01), null,
                             fake, 1 << 30, st) == 1
    assert lib.km_emeans_fit(fake, 1, null, 1, 10, 4, 8, fake, 5, 2, f(0.5), null, f(0.01), null,
                             fake, 16, st) == 3
    # km_split_dead: null sizes, eps outside [0, 1)
    assert lib.km_split_dead(fake, null, fake, f(0.1), 1, 4, 8, null, null, null, st) == 1
    assert lib.km_split_dead(fake, fake, fake, f(1.0), 1, 4, 8, null, null, null, st) == 1
    # km_encode1d: K above 256; km_init_kmeanspp1d: rows longer than 8192 are not provided
    assert lib.km_encode1d(fake, 1, 1, 10, fake, 257, fake, st) == 1
    assert lib.km_init_kmeanspp1d(fake, 1, null, 1, 9000, 4, fake, fake, null, st) == 2
    assert lib.km_init_kmeanspp1d(fake, 1, null, 1, 100, 4, null, fake, null, st) == 1
    # km_init_grid1d: d is implied 1, K must be >= 1
    assert lib.km_init_grid1d(fake, 1, 1, 10, 0, fake, st) == 1
    # km_prep: nothing to write
    assert lib.km_prep(fake, 1, 1, 4, 8, null, null, st) == 1
    code = ctypes.c_int(7)
    assert lib.km_device_error(st, None) == 1
