"""Host-side checks of the C-ABI library that need no GPU: it builds for sm_100a, loads, and
exports every function include/splat.h declares. No compute call is made here."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "splat.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(splat_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib_path():
    from gaussian_splatting_raster_b200 import build
    return build()


def test_header_lists_the_binding_exports():
    import gaussian_splatting_raster_b200 as P
    assert _declared() == sorted(P.EXPORTS)


def test_library_loads_and_exports_every_declared_symbol(lib_path):
    lib = ctypes.CDLL(lib_path)
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r" T (splat_\w+)", out))
    assert exported == set(_declared())


def test_binding_loads_without_a_device(lib_path):
    import gaussian_splatting_raster_b200 as P
    L = P.load_library()
    assert L.splat_last_error(None) == b"no workspace"
    assert L.splat_launch_count(None) == 0


def test_built_for_sm100a_only(lib_path):
    import importlib
    B = importlib.import_module("gaussian_splatting_raster_b200.build")
    flags = " ".join(B.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert "-fmad=false" in flags and "-use_fast_math" not in flags


def test_missing_library_fails_loudly(tmp_path):
    import gaussian_splatting_raster_b200 as P
    with pytest.raises(OSError):
        P.load_library(str(tmp_path / "nope.so"))


# entry points whose first argument is the workspace handle (or, for splat_ws_create, the place
# to store it): a NULL there is an argument error reported before any device work
_HANDLE_CALLS = [
    "splat_ws_create", "splat_project", "splat_bin_sort", "splat_render", "splat_score_replay",
    "splat_render_score", "splat_score_partials", "splat_backward", "splat_render_features", "splat_scatter",
    "splat_attribution", "splat_copy_projection", "splat_copy_tile_lists", "splat_copy_last",
    "splat_copy_accumulators", "splat_pair_count", "splat_check_status", "splat_set_deterministic",
    "splat_profile_enable", "splat_profile_read",
]


def _zero_args(fn):
    args = []
    for t in fn.argtypes:
        if t in (ctypes.c_int, ctypes.c_longlong):
            args.append(0)
        elif t is ctypes.c_float:
            args.append(ctypes.c_float(0.0))
        else:  # pointers and handles
            args.append(None)
    return args


def test_null_handle_is_an_argument_error(lib_path):
    import gaussian_splatting_raster_b200 as P
    L = P.load_library()
    assert set(_HANDLE_CALLS) <= set(P.EXPORTS)
    for name in _HANDLE_CALLS:
        fn = getattr(L, name)
        assert fn(*_zero_args(fn)) == -1, name  # SPLAT_ERR_INVALID_ARG
    L.splat_ws_destroy(None)  # a no-op


def test_kernel_group_names_and_build_flavour(lib_path):
    import gaussian_splatting_raster_b200 as P
    L = P.load_library()
    names = [L.splat_kernel_name(i).decode() for i in range(P.KERNEL_GROUPS)]
    assert len(set(names)) == P.KERNEL_GROUPS and "?" not in names
    assert {"project", "render", "replay", "finalize", "backward"} <= set(names)
    assert L.splat_kernel_name(-1) == b"?" and L.splat_kernel_name(P.KERNEL_GROUPS) == b"?"
    assert L.splat_checked_build() == 0  # the release library


def test_argument_errors_come_before_any_device_work(lib_path):
    """The refusals include/splat.h documents as taken before any work: they return their codes
    here, where there is no device (a call that reached CUDA would fail with SPLAT_ERR_CUDA or
    SPLAT_ERR_OOM instead)."""
    import gaussian_splatting_raster_b200 as P
    L = P.load_library()
    INVALID, CAPACITY, OK = -1, -2, 0
    h = ctypes.c_void_p()
    for args in ((-1, 1, 8, 8, 0), (1, 0, 8, 8, 0), (1, 1025, 8, 8, 0), (1, 1, 0, 8, 0),
                 (1, 1, 8, 0, 0), (1, 1, 8, 8, -1), (1, 1, 8, 8, 4)):
        assert L.splat_ws_create(ctypes.byref(h), *args) == INVALID, args
        assert h.value is None  # *ws is set to NULL on failure
    assert L.splat_ws_create(None, 1, 1, 8, 8, 0) == INVALID
    fin = L.splat_finalize_partials
    some = ctypes.c_void_p(4096)  # never dereferenced: every call below returns first
    for G, deg, lam in ((-1, 0, 1.0), (4, -1, 1.0), (4, 4, 1.0), (4, 0, -1.0),
                        (4, 0, float("nan")), (4, 0, float("inf"))):
        assert fin(some, G, deg, ctypes.c_float(lam), some, None) == INVALID, (G, deg, lam)
    assert fin(None, 4, 0, ctypes.c_float(1.0), some, None) == INVALID
    assert fin(ctypes.c_void_p(4098), 4, 0, ctypes.c_float(1.0), some, None) == INVALID  # align
    assert fin(None, 0, 3, ctypes.c_float(1.0), None, None) == OK  # nothing to do
    srt = L.splat_sort_depths_noalloc
    srt.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    srt.restype = ctypes.c_int
    assert srt(some, -1, some, None) == INVALID
    assert srt(None, 5, some, None) == INVALID and srt(some, 5, None, None) == INVALID
    assert srt(some, 262144 + 1, some, None) == CAPACITY  # SPLAT_NOALLOC_MAX_N + 1
    assert srt(None, 0, None, None) == OK
