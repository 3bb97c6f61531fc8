"""The allocation-free depth ordering entry point, through the C ABI.

Callers that cannot allocate device memory (allocator hooks, fixed buffers handed to a plugin)
get the binning's contributor order from splat_sort_depths_noalloc, whose scratch is a fixed
device array inside the library. Its order must equal the per-tile order the regular binning
entry point produces, on two calls in a row (the second call reuses the array the first left
behind). This file is collected last on purpose.
"""
import ctypes
import math

import numpy as np
import pytest

from synth import scenes

pytestmark = pytest.mark.gpu


def _lib():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for the gpu tests")
    import gaussian_splatting_raster_b200 as P
    P.build()
    L = P.load_library()
    L.splat_sort_depths_noalloc.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
                                            ctypes.c_void_p]
    L.splat_sort_depths_noalloc.restype = ctypes.c_int
    return L


def _one_tile_lists(seed, G):
    """All Gaussians of a 16x16 single-tile view, binned by the regular entry points."""
    import torch
    from gaussian_splatting_raster_b200 import runner
    sc = scenes.tiny_scene(seed, G, 16, 16, V=1, deg=0, depth_range=(1.0, 40.0),
                           log_scale_mean=math.log(0.05))
    ds = runner.to_device(sc)
    ws = runner.workspace_for(ds)
    out = runner.alloc_outputs(ds)
    n = runner.render(ws, ds, out)[0]
    rec = torch.empty((1, sc.G, 16), dtype=torch.float32, device="cuda")
    rect = torch.empty((1, sc.G, 4), dtype=torch.int32, device="cuda")
    ws.copy_projection(rec, rect)
    off = torch.empty((1, 2), dtype=torch.int64, device="cuda")
    ids = torch.empty((max(n, 1),), dtype=torch.int32, device="cuda")
    ws.copy_tile_lists(off, ids)
    torch.cuda.synchronize()
    ws.close()
    return rec[0, :, 12].clone(), ids[:n].clone()  # camera depth z per Gaussian, the tile list


@pytest.mark.parametrize("G", [3000, 20000])
def test_noalloc_order_equals_binning_order_twice(G):
    import torch
    L = _lib()
    depth, tile_list = _one_tile_lists(17 + G, G)
    members = torch.sort(tile_list).values  # the listed Gaussians in index order
    d = depth[members.long()].contiguous()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        order = torch.full((d.numel(),), -1, dtype=torch.int32, device="cuda")
        rc = L.splat_sort_depths_noalloc(ctypes.c_void_p(d.data_ptr()), d.numel(),
                                         ctypes.c_void_p(order.data_ptr()), stream)
        assert rc == 0
        torch.cuda.synchronize()
        got = members[order.long()]
        assert torch.equal(got, tile_list), f"call {call}: order differs from the tile list"


def test_noalloc_rejects_oversize_and_null():
    import torch
    L = _lib()
    cap = 262144  # SPLAT_NOALLOC_MAX_N
    d = torch.zeros(1, device="cuda")
    o = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert L.splat_sort_depths_noalloc(ctypes.c_void_p(d.data_ptr()), cap + 1,
                                       ctypes.c_void_p(o.data_ptr()), None) == -2
    assert L.splat_sort_depths_noalloc(None, 5, ctypes.c_void_p(o.data_ptr()), None) == -1
    assert L.splat_sort_depths_noalloc(None, 0, None, None) == 0
    # a full-capacity call still orders correctly (negative values and index ties included)
    rng = np.random.default_rng(5)
    x = rng.integers(-50, 50, cap).astype(np.float32) * np.float32(0.25)
    dx = torch.from_numpy(x).cuda()
    ox = torch.empty(cap, dtype=torch.int32, device="cuda")
    assert L.splat_sort_depths_noalloc(ctypes.c_void_p(dx.data_ptr()), cap,
                                       ctypes.c_void_p(ox.data_ptr()), None) == 0
    torch.cuda.synchronize()
    assert (ox.cpu().numpy() == np.argsort(x, kind="stable")).all()
