"""Host-side checks of libtitansmem's C ABI. No GPU is touched: every call here
either is host-only or returns before its first CUDA call."""
import ctypes
import os
import re

import pytest

from test_trained_neural_b200 import _native as N

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "titansmem.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.findall(r"TM_API\s+[\w\s\*]+?\b(tm_\w+)\s*\(", src)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("tm_create", "tm_run", "tm_destroy", "tm_workspace_size", "tm_status_string",
                     "tm_sync", "tm_param_count"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = N.load()
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(declared_functions()) <= set(N.SIGNATURES), "binding misses a declared function"


def create(L=2, d=64, e=4):
    lib = N.load()
    h = ctypes.c_void_p()
    rc = lib.tm_create(L, d, e, N.TM_ACT_SILU, ctypes.byref(h))
    return rc, h


@pytest.mark.parametrize("L,d,e,ok", [(1, 64, 1, True), (2, 384, 4, True), (4, 128, 2, True),
                                      (0, 64, 4, False), (5, 64, 4, False), (2, 6, 4, False),
                                      (2, 0, 4, False), (2, 64, 0, False), (2, 1024, 8, False),
                                      (1, 64, 0, True)])
def test_create_validates(L, d, e, ok):
    rc, h = create(L, d, e)
    assert (rc == N.TM_OK) == ok, rc
    if ok:
        N.load().tm_destroy(h)
    else:
        assert rc == N.TM_ERR_INVALID_ARG and not h.value


def test_create_null_out_and_bad_activation():
    lib = N.load()
    assert lib.tm_create(2, 64, 4, 0, None) == N.TM_ERR_INVALID_ARG
    h = ctypes.c_void_p()
    assert lib.tm_create(2, 64, 4, 7, ctypes.byref(h)) == N.TM_ERR_INVALID_ARG


@pytest.mark.parametrize("L,d,e,P", [(1, 64, 1, 4096), (2, 384, 4, 1179648), (2, 64, 4, 32768),
                                     (2, 128, 4, 131072), (4, 128, 2, 196608)])
def test_param_count(L, d, e, P):
    rc, h = create(L, d, e)
    assert rc == N.TM_OK
    assert N.load().tm_param_count(h) == P
    N.load().tm_destroy(h)
    assert N.load().tm_param_count(None) == 0


def test_workspace_and_shape_validation():
    lib = N.load()
    _, h = create(2, 64, 4)
    out = ctypes.c_size_t()
    assert lib.tm_workspace_size(h, 4, 8, 8192, 64, N.TM_BF16, ctypes.byref(out)) == N.TM_OK
    assert out.value >= 256 and out.value % 4 == 0
    for B, H, T, C in [(0, 1, 64, 64), (1, 0, 64, 64), (1, 1, 0, 64), (1, 1, 512, 512), (1, 1, 64, 0)]:
        assert lib.tm_workspace_size(h, B, H, T, C, N.TM_BF16, ctypes.byref(out)) == N.TM_ERR_INVALID_ARG
    # a shorter last chunk (C does not divide T, or T < C) is accepted
    for T in (100, 32):
        assert lib.tm_workspace_size(h, 1, 1, T, 64, N.TM_BF16, ctypes.byref(out)) == N.TM_OK
    assert lib.tm_workspace_size(h, 1, 1, 64, 64, 9, ctypes.byref(out)) == N.TM_ERR_INVALID_ARG
    assert lib.tm_workspace_size(None, 1, 1, 64, 64, N.TM_BF16, ctypes.byref(out)) == N.TM_ERR_INVALID_ARG
    lib.tm_destroy(h)


def test_path_selection_and_query():
    lib = N.load()
    _, h = create(1, 64, 1)
    p = ctypes.c_int()
    assert lib.tm_query_path(h, 1, 1, 256, 16, N.TM_F32, ctypes.byref(p)) == N.TM_OK
    assert p.value == N.TM_PATH_SIMT
    assert lib.tm_set_path(h, 9) == N.TM_ERR_INVALID_ARG
    assert lib.tm_set_path(h, N.TM_PATH_TC_GLOBAL) == N.TM_OK
    assert lib.tm_set_path(h, N.TM_PATH_TC_PHASED) == N.TM_OK
    assert lib.tm_query_path(h, 1, 1, 256, 64, N.TM_BF16, ctypes.byref(p)) == N.TM_OK
    assert p.value == N.TM_PATH_TC_PHASED
    assert lib.tm_set_path(h, N.TM_PATH_SIMT) == N.TM_OK
    assert lib.tm_query_path(h, 1, 1, 256, 16, N.TM_BF16, ctypes.byref(p)) == N.TM_OK
    assert p.value == N.TM_PATH_SIMT
    lib.tm_destroy(h)


def test_launch_count():
    """Launches per tm_run: one persistent kernel, or for the layered paths
    per group of streams an init and a coefficient kernel plus, per chunk,
    the fused forward/backward (or 2L - 1 phase launches) and one update;
    the tensor-core paths add one launch that converts keys and queries to
    fp16."""
    import os
    lib = N.load()
    _, h = create(2, 64, 4)
    n = ctypes.c_longlong()
    assert lib.tm_launch_count(h, 1, 2, 256, 64, N.TM_F32, ctypes.byref(n)) == N.TM_OK
    assert n.value == 1
    assert lib.tm_launch_count(h, 1, 2, 256, 64, N.TM_BF16, None) == N.TM_ERR_INVALID_ARG
    groups = int(os.environ.get("TM_TCL_GROUPS", "0"))
    for path, per_chunk in ((N.TM_PATH_TC_LAYERED, 2), (N.TM_PATH_TC_PHASED, 2 * 2)):
        assert lib.tm_set_path(h, path) == N.TM_OK
        for B, H in ((1, 2), (2, 4), (3, 3)):
            S = B * H
            g = max(1, min(groups or min(S // 8, 8), S))
            assert lib.tm_launch_count(h, B, H, 256, 64, N.TM_BF16, ctypes.byref(n)) == N.TM_OK
            assert n.value == 1 + g * (2 + per_chunk * 4), (path, B, H, n.value)
    lib.tm_destroy(h)


def _run(lib, h, ptrs, B=1, H=1, T=64, C=16, dt=N.TM_F32, ws_bytes=1 << 30):
    args = [ctypes.c_void_p(x) for x in ptrs]
    return lib.tm_run(h, B, H, T, C, dt, *args[:11], args[11], ws_bytes, None)


def test_run_rejects_bad_arguments_before_any_launch():
    lib = N.load()
    _, h = create(1, 64, 1)
    # distinct fake, never-dereferenced addresses, 256-byte aligned, far apart
    base = [0x10_0000_0000 + i * 0x1_0000_0000 for i in range(12)]
    bad_null = list(base)
    bad_null[3] = 0
    assert _run(lib, h, bad_null) == N.TM_ERR_INVALID_ARG
    bad_align = list(base)
    bad_align[0] += 8
    assert _run(lib, h, bad_align) == N.TM_ERR_INVALID_ARG
    bad_ws_align = list(base)
    bad_ws_align[11] += 16
    assert _run(lib, h, bad_ws_align) == N.TM_ERR_INVALID_ARG
    assert _run(lib, h, base, T=0, C=16) == N.TM_ERR_INVALID_ARG
    assert _run(lib, h, base, C=0) == N.TM_ERR_INVALID_ARG
    # y overlapping k
    ov = list(base)
    ov[8] = ov[0] + 256
    assert _run(lib, h, ov) == N.TM_ERR_INVALID_ARG
    # W_end partially overlapping W0 (exact equality would be allowed)
    ov = list(base)
    ov[9] = ov[6] + 256
    assert _run(lib, h, ov) == N.TM_ERR_INVALID_ARG
    # W_end overlapping S_end
    ov = list(base)
    ov[10] = ov[9]
    assert _run(lib, h, ov) == N.TM_ERR_INVALID_ARG
    # workspace too small
    assert _run(lib, h, base, ws_bytes=64) == N.TM_ERR_OOM
    assert lib.tm_run(None, 1, 1, 64, 16, 0, *([None] * 12), 0, None) == N.TM_ERR_INVALID_ARG
    lib.tm_destroy(h)


def test_status_strings():
    for code in range(7):
        s = N.status_string(code)
        assert isinstance(s, str) and s
    assert N.status_string(99) == "unknown status"
    assert N.load().tm_version() >= 100
