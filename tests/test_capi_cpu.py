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
