"""Deterministic accumulation (splat_set_deterministic): fixed-point integer atomics make the
replay's and the backward's per-(view, Gaussian) sums independent of the order of the adds, so two
runs give the same bits; the results still meet the oracle's bars and agree with the default
(floating-point reduction) mode to rounding."""
import numpy as np
import pytest

from oracle import oracle as O
from synth import scenes
from tests import parity_util as PU

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for the gpu tests")
    from gaussian_splatting_raster_b200 import build, load_library
    build()
    load_library()


def _runs(sc, obs, det, n=2):
    import torch
    from gaussian_splatting_raster_b200 import grad_dim, runner

    ds = runner.to_device(sc)
    obs_t = torch.as_tensor(np.ascontiguousarray(obs, np.float32)).cuda()
    ws = runner.workspace_for(ds)
    ws.deterministic(det)
    out = runner.alloc_outputs(ds)
    res = []
    for _ in range(n):
        runner.render_and_score(ws, ds, obs_t, out)
        g = torch.empty((ds.G, grad_dim(ds.deg)), device="cuda")
        ws.backward(obs_t, ds.log_scales, ds.quats, ds.sh, raw=g)
        torch.cuda.synchronize()
        res.append((out.tokens.clone(), g))
    ws.close()
    return res


@pytest.mark.parametrize("cfg", [2, 3])
def test_two_runs_give_the_same_bits(cfg):
    import torch
    sc = scenes.make(cfg)
    obs = O.observe(sc, "f") if cfg == 2 else scenes.smooth_observation(5, sc.V, sc.H, sc.W)
    (z1, g1), (z2, g2) = _runs(sc, obs, True)
    assert torch.equal(z1, z2) and torch.equal(g1, g2)
    # agrees with the default floating-point reductions to rounding
    (z3, g3), = _runs(sc, obs, False, n=1)
    za, zb = z1.cpu().numpy().astype(np.float64), z3.cpu().numpy().astype(np.float64)
    assert PU.token_errors(za, zb).max() <= 1e-5
    PU.compare_grads(g1.cpu().numpy(), g3.cpu().numpy().astype(np.float64), rtol=1e-5,
                     block_rtol=1e-4)


def test_deterministic_mode_meets_the_oracle_bars():
    sc = scenes.make(2)
    obs = O.observe(sc, "f")
    (z, g), = _runs(sc, obs, True, n=1)
    o = O.run(sc, obs, "f")
    PU.compare_tokens(z.cpu().numpy(), o["tokens"])
    ob = O.run_backward(sc, obs, "f")
    PU.compare_grads(g.cpu().numpy(), ob["raw"])
