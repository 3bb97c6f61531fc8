"""Pins of the oracle's attribute render, map scatter and scalar attribution (multi-channel /
scalar-attribute compositing of "ReCoSplat" 2.1 and "ATSplat"; alphaT and PRIMU-style
error/coverage of "Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting",
"Novelty Boundary"; the mask-channel gain scatter of "L2D2-GS").

* with the colours of a degree-0 scene as the attributes, the attribute render equals the colour
  render without its background term, bit for bit in fp32 and fp64;
* an attribute of ones renders the coverage 1 - T_final;
* a single Gaussian renders alpha f (closed form);
* the scatter is the adjoint of the render: <m, R f> = <R^T m, f>;
* the scatter of ones equals the replay's support sums, and the attribution columns equal
  scatters of ones and of the residual norm computed here.
"""
import numpy as np
import pytest

from oracle import oracle as O
from synth import scenes


def _setup(sc, mode):
    p = O.project(sc, mode)
    L = O.bin_lists(p, sc.H, sc.W)
    r = O.render(p, L, sc.H, sc.W, sc.bg, mode)
    return p, L, r


@pytest.mark.parametrize("mode", ["f", "d"])
def test_colour_attributes_reproduce_the_render(mode):
    sc = scenes.tiny_scene(11, 300, 40, 56, V=2, deg=0, opac_mean=1.0)
    sc.bg = np.zeros(3, np.float32)
    p, L, r = _setup(sc, mode)
    col = p["rec"][0, :, 7:10]  # degree 0: the colour is the same in every view
    assert np.array_equal(col, p["rec"][1, :, 7:10])
    F = O.render_features(p, L, r, col.astype(np.float32), sc.H, sc.W, mode)
    if mode == "f":  # the same fp32 operations in the same order
        assert np.array_equal(F, r["img"])
    else:  # the attributes are the fp64 colours rounded to fp32
        np.testing.assert_allclose(F, r["img"], rtol=0, atol=1e-7)


@pytest.mark.parametrize("mode,tol", [("f", 2e-6), ("d", 1e-12)])
def test_ones_render_the_coverage(mode, tol):
    sc = scenes.make(2)
    p, L, r = _setup(sc, mode)
    F = O.render_features(p, L, r, np.ones((sc.G, 1), np.float32), sc.H, sc.W, mode)
    np.testing.assert_allclose(F[..., 0], 1.0 - r["T"], atol=tol)


def test_single_gaussian_closed_form():
    sc = scenes.tiny_scene(3, 1, 32, 32, V=1, deg=0, opac_mean=0.5, opac_sigma=0.0)
    p, L, r = _setup(sc, "d")
    f = np.array([[0.25, -1.5, 3.0]], np.float32)
    F = O.render_features(p, L, r, f, sc.H, sc.W, "d")
    tr = [O.trace(p, L, sc.H, sc.W, sc.bg, 0, i, j, "d") for j in range(32) for i in range(32)]
    alpha = np.array([t[0, 1] if len(t) else 0.0 for t in tr]).reshape(32, 32)
    assert (alpha > 0).sum() > 20
    np.testing.assert_allclose(F[0], alpha[..., None] * f.astype(np.float64), rtol=1e-14, atol=0)


@pytest.mark.parametrize("mode,tol", [("f", 1e-6), ("d", 1e-12)])
def test_scatter_is_the_adjoint_of_the_render(mode, tol):
    sc = scenes.make(2)
    p, L, r = _setup(sc, mode)
    rng = np.random.default_rng(4)
    C = 5
    f = rng.normal(size=(sc.G, C)).astype(np.float32)
    m = rng.normal(size=(sc.V, sc.H, sc.W, C)).astype(np.float32)
    F = O.render_features(p, L, r, f, sc.H, sc.W, mode)
    S = O.scatter(p, L, r, m, sc.H, sc.W, mode)
    lhs = float((m.astype(np.float64) * F).sum())
    rhs = float((S * f.astype(np.float64)).sum())
    # relative to the sum of the terms' magnitudes (fp32 mode rounds every composited F)
    mag = float(np.abs(m.astype(np.float64) * F).sum())
    assert abs(lhs - rhs) <= tol * mag


def test_scatter_of_ones_is_the_support_and_attribution_columns():
    sc = scenes.make(2)
    obs = O.observe(sc, "d")
    o = O.run(sc, obs, "d")
    r = dict(img=o["img"], last=o["last"])
    ones = np.ones((sc.V, sc.H, sc.W, 1), np.float32)
    S = O.scatter(o["proj"], o["lists"], r, ones, sc.H, sc.W, "d")[:, 0]
    np.testing.assert_allclose(S, o["acc"][..., 0].sum(0), rtol=1e-12, atol=1e-15)
    A = O.attribution(o["proj"], o["lists"], r, obs, sc.H, sc.W, "d")
    np.testing.assert_allclose(A[:, 0], S, rtol=1e-12, atol=1e-15)
    rn = np.linalg.norm(o["img"] - obs.astype(np.float64), axis=-1)
    E = O.scatter(o["proj"], o["lists"], r, rn[..., None].astype(np.float32), sc.H, sc.W, "d")
    np.testing.assert_allclose(A[:, 1], E[:, 0], rtol=1e-6, atol=1e-12)
    np.testing.assert_allclose(A[:, 2], A[:, 1] / (A[:, 0] + 1e-6), rtol=1e-12)
    assert (A[:, 1] <= A[:, 0] * rn.max() * (1 + 1e-9)).all()  # a weighted mean of |r|
