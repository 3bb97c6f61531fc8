"""Renderer backward on the GPU (splat_backward through the C ABI) against the oracle's
(fp32 decisions): the raw, detached, support-normalised and parameter-scale-normalised gradients
per Gaussian and parameter block within 1e-4 relative L2 (floor 1e-3 x the block's median norm).
"""
import numpy as np
import pytest

from oracle import oracle as O
from synth import scenes
from tests import parity_util as PU
from tests.test_oracle_backward import _clamp_scene

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for the gpu tests")
    from gaussian_splatting_raster_b200 import build, load_library
    build()
    load_library()


def _support(o):
    """q_g = 1e-6 + sum over visible views of (1e-6 + q_gv), from the oracle's sums."""
    return 1e-6 + ((1e-6 + o["accb"][..., 0]) * o["proj"]["valid"]).sum(0)


def _compare_variants(g, o, q, which=None, exclude=None):
    worst = {}
    for k in PU.GRAD_VARIANTS:
        if k == "support":
            # raw / q_g: compared after undoing the oracle's q_g, since dividing by the small
            # support of a barely visible Gaussian magnifies the absolute rounding of its raw
            # gradient (an ill-conditioned quotient, not a property of either implementation)
            worst[k] = PU.compare_grads(g[k] * q[:, None], o["raw"], which, exclude)
            np.testing.assert_allclose(o[k] * q[:, None], o["raw"], rtol=1e-12, atol=0)
        else:
            worst[k] = PU.compare_grads(g[k], o[k], which, exclude)
    assert (g["detached"][:, 3:10] == 0).all()
    return worst


def _check(sc, obs):
    g = PU.gpu_backward(sc, obs)
    o = O.run_backward(sc, obs, "f")
    near = PU.compare_projection(sc, g, o["proj"])
    np.testing.assert_allclose(g["img"], o["img"], atol=PU.COLOUR_ATOL)
    return _compare_variants(g, o, _support(o), exclude=near)


@pytest.mark.parametrize("cfg", [1, 2])
def test_backward_small_configs(cfg):
    sc = scenes.make(cfg)
    _check(sc, O.observe(sc, "f"))


@pytest.mark.parametrize("deg", [0, 2, 3])
def test_backward_sh_degrees_ragged_image(deg):
    sc = scenes.tiny_scene(50 + deg, 300, 37, 70, V=3, deg=deg)
    obs = np.random.default_rng(deg).uniform(0, 1, (3, 37, 70, 3)).astype(np.float32)
    _check(sc, obs)


def test_backward_with_clamps_active():
    sc = _clamp_scene()
    obs = np.random.default_rng(41).uniform(0.2, 0.8, (sc.V, sc.H, sc.W, 3)).astype(np.float32)
    _check(sc, obs)


def test_backward_full_size_sampled():
    """ReSplat-scale scene: gradients of sampled Gaussians (the oracle runs the backward over
    every tile those Gaussians touch)."""
    sc = scenes.make(3)
    obs = scenes.smooth_observation(91, sc.V, sc.H, sc.W)
    g = PU.gpu_backward(sc, obs)
    p = O.project(sc, "f")
    near = PU.compare_projection(sc, g, p)
    L = O.bin_lists(p, sc.H, sc.W)
    rng = np.random.default_rng(3)
    TX, TY = O.n_tiles(sc.H, sc.W)
    cand = np.nonzero(p["valid"].any(0) & ~near)[0]
    gs = rng.choice(cand, size=24, replace=False)
    sel = set()
    for v in range(sc.V):
        for gg in gs:
            if p["valid"][v, gg]:
                x0, y0, x1, y1 = p["rect"][v, gg]
                sel.update((v, ty * TX + tx) for ty in range(y0, y1) for tx in range(x0, x1))
    sel = np.array(sorted(sel), np.int32)
    r = O.render(p, L, sc.H, sc.W, sc.bg, "f", sel=sel)
    accb = O.backward(p, L, r, obs, sc.bg, sc.H, sc.W, "f", sel=sel)
    o = dict(proj=p, accb=accb, **O.gradients(p, accb, sc, "f"))
    _compare_variants(g, o, _support(o), which=gs)


def test_backward_leaves_the_replay_intact():
    """splat_backward between render and score replay changes neither the tokens nor itself. Run
    in deterministic mode, where the sums do not depend on the order of the additions, so the
    repeated calls must give the same bits."""
    import torch
    from gaussian_splatting_raster_b200 import grad_dim, runner, token_dim

    sc = scenes.make(2)
    obs = O.observe(sc, "f")
    ds = runner.to_device(sc)
    obs_t = torch.as_tensor(obs).cuda()
    ws = runner.workspace_for(ds)
    ws.deterministic(True)
    out = runner.alloc_outputs(ds)
    K = grad_dim(ds.deg)
    g1 = torch.empty((ds.G, K), device="cuda")
    g2 = torch.empty((ds.G, K), device="cuda")
    runner.render_and_backward(ws, ds, obs_t, out, {"raw": g1})
    ws.score_replay(obs_t, out.tokens)
    z1 = out.tokens.clone()
    ws.backward(obs_t, ds.log_scales, ds.quats, ds.sh, raw=g2)
    ws.score_replay(obs_t, out.tokens)
    torch.cuda.synchronize()
    assert torch.equal(z1, out.tokens) and torch.equal(g1, g2)
    ws.close()


def test_backward_call_errors():
    import torch
    from gaussian_splatting_raster_b200 import SplatError, runner

    sc = scenes.tiny_scene(3, 64, 32, 32, V=1, deg=1)
    ds = runner.to_device(sc)
    ws = runner.workspace_for(ds)
    ws.project(ds.means, ds.log_scales, ds.quats, ds.opac, ds.sh, ds.viewmats, ds.intrin,
               ds.H, ds.W)
    obs = torch.zeros((1, 32, 32, 3), device="cuda")
    g = torch.zeros((64, 23), device="cuda")
    with pytest.raises(SplatError) as e:  # not rendered yet
        ws.backward(obs, ds.log_scales, ds.quats, ds.sh, raw=g)
    assert e.value.code == -3
    ws.bin_sort()
    out = runner.alloc_outputs(ds)
    ws.render(ds.bg, out.img, out.T, out.n_contrib)
    with pytest.raises(SplatError) as e:  # no output requested
        ws.backward(obs, ds.log_scales, ds.quats, ds.sh)
    assert e.value.code == -1
    ws.close()


def test_backward_all_culled_and_empty():
    """Every Gaussian behind the cameras: zero gradients; G = 0: empty outputs, no error."""
    sc = scenes.tiny_scene(3, 5, 20, 24, V=2)
    sc.means[:, 2] = -1.0
    obs = np.random.default_rng(1).uniform(0, 1, (2, 20, 24, 3)).astype(np.float32)
    g = PU.gpu_backward(sc, obs)
    for k in PU.GRAD_VARIANTS:
        assert (g[k] == 0).all()
    sc0 = scenes.tiny_scene(3, 1, 20, 24, V=1)
    for name in ("means", "log_scales", "quats", "opac", "sh"):
        setattr(sc0, name, getattr(sc0, name)[:0])
    g0 = PU.gpu_backward(sc0, np.zeros((1, 20, 24, 3), np.float32))
    assert g0["raw"].shape == (0, 23)
