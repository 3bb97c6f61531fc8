"""The bounds-checked build (libsplat_checked.so, -DSPLAT_CHECKED): every index the kernels take
from data is checked; the small parity cases run through it with no failed check and the same
results as the oracle (race/overrun detection where compute-sanitizer is not available)."""
import numpy as np
import pytest

from oracle import oracle as O
from synth import scenes
from tests import parity_util as PU

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def checked():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for the gpu tests")
    from gaussian_splatting_raster_b200 import LIB_CHECKED, build, load_library
    build(checked=True)
    L = load_library(LIB_CHECKED)
    assert L.splat_checked_build() == 1
    return L


@pytest.mark.parametrize("which", ["two_plane", "three_layer", "tiny_deg3_ragged", "resplat"])
def test_checked_build_runs_clean(checked, which):
    import torch
    from gaussian_splatting_raster_b200 import grad_dim, runner

    sc = {"two_plane": lambda: scenes.make(1), "three_layer": lambda: scenes.make(2),
          "tiny_deg3_ragged": lambda: scenes.tiny_scene(5, 300, 37, 70, V=3, deg=3),
          "resplat": lambda: scenes.make(3)}[which]()
    obs = (O.observe(sc, "f") if which != "resplat"
           else scenes.smooth_observation(3, sc.V, sc.H, sc.W))
    ds = runner.to_device(sc)
    ws = runner.workspace_for(ds, lib=checked)
    out = runner.alloc_outputs(ds)
    obs_t = torch.as_tensor(np.ascontiguousarray(obs, np.float32)).cuda()
    runner.render_and_score(ws, ds, obs_t, out)
    g = torch.empty((ds.G, grad_dim(ds.deg)), device="cuda")
    ws.backward(obs_t, ds.log_scales, ds.quats, ds.sh, raw=g)
    F = torch.empty((ds.V, ds.H, ds.W, 3), device="cuda")
    ws.render_features(torch.ones((ds.G, 3), device="cuda"), F)
    A = torch.empty((ds.G, 3), device="cuda")
    ws.attribution(obs_t, A)
    ws.check_status()  # raises SplatError(BOUNDS) when any check failed
    torch.cuda.synchronize()
    if which != "resplat":  # full comparison on the small cases
        o = O.run(sc, obs, "f")
        np.testing.assert_allclose(out.img.cpu().numpy(), o["img"], atol=PU.COLOUR_ATOL)
        PU.compare_tokens(out.tokens.cpu().numpy(), o["tokens"])
        np.testing.assert_allclose(F.cpu().numpy()[..., 0], 1.0 - o["T"], atol=2e-6)
    ws.close()
