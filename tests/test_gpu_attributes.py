"""Attribute render, map scatter and scalar attribution on the GPU (through the C ABI) against
the oracle (fp32 decisions). The attribute render takes the render's fp32 weights in the same
order as the oracle's fp32 mode, so it must agree bit for bit; the scatters add fp32 products in
fp64 in another order: 1e-5 relative per Gaussian (floor 1e-6 x the largest row) for non-negative
maps, 1e-5 of the scatter of |m| for signed ones."""
import numpy as np
import pytest

from oracle import oracle as O
from synth import scenes

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for the gpu tests")
    from gaussian_splatting_raster_b200 import build, load_library
    build()
    load_library()


def _gpu(sc, obs, feats=None, pixel_map=None):
    import torch
    from gaussian_splatting_raster_b200 import runner

    ds = runner.to_device(sc)
    ws = runner.workspace_for(ds)
    out = runner.alloc_outputs(ds)
    runner.render(ws, ds, out)
    res = {}
    if feats is not None:
        f = torch.as_tensor(feats).cuda()
        F = torch.full((sc.V, sc.H, sc.W, feats.shape[1]), float("nan"), device="cuda")
        ws.render_features(f, F)
        res["F"] = F
    if pixel_map is not None:
        m = torch.as_tensor(pixel_map).cuda()
        S = torch.full((sc.G, pixel_map.shape[3]), float("nan"), device="cuda")
        ws.scatter(m, S)
        res["S"] = S
    if obs is not None:
        A = torch.full((sc.G, 3), float("nan"), device="cuda")
        ws.attribution(torch.as_tensor(obs).cuda(), A)
        res["A"] = A
    res["img"] = out.img
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in res.items()}
    ws.close()
    return res


def _rows_close(g, o, rtol=1e-5):
    scale = np.abs(o).max(initial=0.0)
    err = np.abs(g.astype(np.float64) - o).max(axis=1) / np.maximum(np.abs(o).max(axis=1),
                                                                      1e-6 * scale)
    assert err.max(initial=0) <= rtol, (err.max(), err.argmax())


def _oracle(sc):
    p = O.project(sc, "f")
    L = O.bin_lists(p, sc.H, sc.W)
    r = O.render(p, L, sc.H, sc.W, sc.bg, "f")
    return p, L, r


@pytest.mark.parametrize("C", [1, 3, 9, 20])
def test_attribute_render_bitwise(C):
    sc = scenes.make(2)
    rng = np.random.default_rng(C)
    f = rng.normal(size=(sc.G, C)).astype(np.float32)
    g = _gpu(sc, None, feats=f)
    p, L, r = _oracle(sc)
    F = O.render_features(p, L, r, f, sc.H, sc.W, "f")
    assert np.isfinite(g["F"]).all()
    assert np.array_equal(g["F"].astype(np.float64), F)


@pytest.mark.parametrize("C", [1, 2, 5, 9, 17])
def test_scatter_matches_oracle_and_is_the_adjoint(C):
    sc = scenes.tiny_scene(60 + C, 400, 45, 77, V=2, deg=1)
    rng = np.random.default_rng(C)
    m = rng.normal(size=(sc.V, sc.H, sc.W, C)).astype(np.float32)
    f = rng.normal(size=(sc.G, C)).astype(np.float32)
    g = _gpu(sc, None, feats=f, pixel_map=m)
    p, L, r = _oracle(sc)
    S = O.scatter(p, L, r, m, sc.H, sc.W, "f")
    # a signed map's sum can be far smaller than its terms; the fp32 products and the warp's fp32
    # partial sums round relative to the terms, so the bar is relative to the scatter of |m|
    S_abs = O.scatter(p, L, r, np.abs(m), sc.H, sc.W, "f")
    err = np.abs(g["S"].astype(np.float64) - S) / np.maximum(S_abs, 1e-30)
    assert err.max(initial=0) <= 1e-5, (err.max(), np.unravel_index(err.argmax(), err.shape))
    lhs = float((m.astype(np.float64) * g["F"]).sum())
    rhs = float((g["S"].astype(np.float64) * f).sum())
    assert abs(lhs - rhs) <= 1e-5 * float(np.abs(m * g["F"]).sum())


def test_attribution_matches_oracle():
    sc = scenes.make(2)
    obs = O.observe(sc, "f")
    g = _gpu(sc, obs)
    p, L, r = _oracle(sc)
    A = O.attribution(p, L, r, obs, sc.H, sc.W, "f")
    _rows_close(g["A"][:, :2], A[:, :2])
    seen = A[:, 0] > 1e-3  # the per-coverage error of barely seen Gaussians is a tiny quotient
    np.testing.assert_allclose(g["A"][seen, 2], A[seen, 2], rtol=1e-5)


def test_full_size_sampled():
    """ReSplat-scale scene: the attribute render on sampled tiles (bitwise) and the scatter of
    sampled Gaussians (the oracle covers every tile they touch)."""
    sc = scenes.make(3)
    rng = np.random.default_rng(5)
    f = rng.uniform(0, 1, (sc.G, 9)).astype(np.float32)
    obs = scenes.smooth_observation(17, sc.V, sc.H, sc.W)
    g = _gpu(sc, obs, feats=f)
    p = O.project(sc, "f")
    L = O.bin_lists(p, sc.H, sc.W)
    TX, TY = O.n_tiles(sc.H, sc.W)
    gs = rng.choice(np.nonzero(p["valid"].any(0))[0], size=24, replace=False)
    sel = set()
    for v in range(sc.V):
        for gg in gs:
            if p["valid"][v, gg]:
                x0, y0, x1, y1 = p["rect"][v, gg]
                sel.update((v, ty * TX + tx) for ty in range(y0, y1) for tx in range(x0, x1))
    sel = np.array(sorted(sel), np.int32)
    r = O.render(p, L, sc.H, sc.W, sc.bg, "f", sel=sel)
    F = O.render_features(p, L, r, f, sc.H, sc.W, "f", sel=sel)
    mask = np.zeros((sc.V, sc.H, sc.W), bool)
    for v, t in sel:
        tx, ty = t % TX, t // TX
        mask[v, ty * 16:(ty + 1) * 16, tx * 16:(tx + 1) * 16] = True
    assert np.array_equal(g["F"][mask].astype(np.float64), F[mask])
    A = O.attribution(p, L, r, obs, sc.H, sc.W, "f", sel=sel)
    _rows_close(g["A"][gs, :2], A[gs, :2])


def test_call_errors():
    import torch
    from gaussian_splatting_raster_b200 import SplatError, runner

    sc = scenes.tiny_scene(3, 64, 32, 32, V=1, deg=1)
    ds = runner.to_device(sc)
    ws = runner.workspace_for(ds)
    ws.project(ds.means, ds.log_scales, ds.quats, ds.opac, ds.sh, ds.viewmats, ds.intrin,
               ds.H, ds.W)
    ws.bin_sort()
    f = torch.zeros((64, 4), device="cuda")
    F = torch.zeros((1, 32, 32, 4), device="cuda")
    with pytest.raises(SplatError) as e:  # not rendered yet
        ws.render_features(f, F)
    assert e.value.code == -3
    out = runner.alloc_outputs(ds)
    ws.render(ds.bg, out.img, out.T, out.n_contrib)
    with pytest.raises(SplatError) as e:  # too many channels
        ws.render_features(torch.zeros((64, 65), device="cuda"),
                           torch.zeros((1, 32, 32, 65), device="cuda"))
    assert e.value.code == -1
    ws.close()


def test_all_culled_and_empty():
    """Nothing composited: attributes render 0 and scatter 0; G = 0 works."""
    sc = scenes.tiny_scene(3, 5, 20, 24, V=2)
    sc.means[:, 2] = -1.0
    m = np.ones((2, 20, 24, 2), np.float32)
    g = _gpu(sc, np.zeros((2, 20, 24, 3), np.float32), feats=np.ones((5, 3), np.float32),
             pixel_map=m)
    assert (g["F"] == 0).all() and (g["S"] == 0).all() and (g["A"][:, :2] == 0).all()
    sc0 = scenes.tiny_scene(3, 1, 20, 24, V=1)
    for name in ("means", "log_scales", "quats", "opac", "sh"):
        setattr(sc0, name, getattr(sc0, name)[:0])
    g0 = _gpu(sc0, np.zeros((1, 20, 24, 3), np.float32), feats=np.zeros((0, 4), np.float32),
              pixel_map=np.ones((1, 20, 24, 4), np.float32))
    assert (g0["F"] == 0).all() and g0["S"].shape == (0, 4) and g0["A"].shape == (0, 3)
