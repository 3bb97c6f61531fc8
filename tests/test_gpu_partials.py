"""View-split scoring on the GPU: per-Gaussian partial sums (splat_score_partials) and tokens
from summed partials (splat_finalize_partials) against the oracle's partials and tokens.

Bars: partial rows within 1e-4 relative L2 per Gaussian (floor 1e-3 x median row norm), tokens
as in the fused path (1e-4 relative L2 per Gaussian).
"""
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


def _view_subset(ds, lo, hi):
    import dataclasses
    return dataclasses.replace(ds, viewmats=ds.viewmats[lo:hi].contiguous(),
                               intrin=ds.intrin[lo:hi].contiguous())


def _gpu_partials(ds, obs_t, lo, hi):
    """Render views [lo, hi) of the device scene and return their partials [G, 11 + 3d]."""
    import torch
    from gaussian_splatting_raster_b200 import partials_dim, runner

    local = _view_subset(ds, lo, hi)
    ws = runner.workspace_for(local)
    out = runner.alloc_outputs(local)
    runner.render(ws, local, out)
    P = torch.full((ds.G, partials_dim(ds.deg)), float("nan"), dtype=torch.float32,
                   device="cuda")
    ws.score_partials(obs_t[lo:hi].contiguous(), P)
    torch.cuda.synchronize()
    ws.close()
    return P


def _finalize(P, deg, lam):
    import torch
    from gaussian_splatting_raster_b200 import finalize_partials, token_dim
    z = torch.empty((P.shape[0], token_dim(deg)), dtype=torch.float32, device="cuda")
    finalize_partials(P.contiguous(), deg, z, lam)
    torch.cuda.synchronize()
    return z.cpu().numpy()


def _oracle_partials(sc, obs, views):
    o = O.run(sc, obs, "f")
    return O.partials(o["proj"], o["acc"], sc, views), o


@pytest.mark.parametrize("cfg,deg", [(2, None), (None, 0), (None, 3)])
def test_partials_all_views_match_oracle_and_fused_tokens(cfg, deg):
    import torch
    from gaussian_splatting_raster_b200 import runner

    sc = scenes.make(cfg) if cfg else scenes.tiny_scene(5 + deg, 300, 40, 72, V=3, deg=deg)
    obs = O.observe(sc, "f")
    lam = 0.7
    ds = runner.to_device(sc)
    obs_t = torch.as_tensor(np.ascontiguousarray(obs, np.float32)).cuda()
    P = _gpu_partials(ds, obs_t, 0, sc.V)
    Po, o = _oracle_partials(sc, obs, None)
    assert np.isfinite(P.cpu().numpy()).all(), "a partial row was left unwritten"
    PU.compare_tokens(P.cpu().numpy(), Po)
    z = _finalize(P, sc.sh_degree, lam)
    zo = O.finalize(o["proj"], o["acc"], sc, lam)
    PU.compare_tokens(z, zo)
    g = PU.gpu_run(sc, obs, lam)  # the fused score replay on the same inputs
    PU.compare_tokens(z, g["tokens"].astype(np.float64))


@pytest.mark.parametrize("split", [(0, 1, 4), (0, 3, 4)])
def test_two_view_blocks_sum_to_all_views(split):
    """Two disjoint view blocks, rendered by separate workspaces; their partials summed on the
    device give the tokens of all views (the single-process stand-in for the reduce-scatter)."""
    import torch
    from gaussian_splatting_raster_b200 import runner

    sc = scenes.make(2)
    obs = O.observe(sc, "f")
    ds = runner.to_device(sc)
    obs_t = torch.as_tensor(np.ascontiguousarray(obs, np.float32)).cuda()
    a, b, c = split
    P1 = _gpu_partials(ds, obs_t, a, b)
    P2 = _gpu_partials(ds, obs_t, b, c)
    P1o, o = _oracle_partials(sc, obs, range(a, b))
    PU.compare_tokens(P1.cpu().numpy(), P1o)
    z = _finalize(P1 + P2, sc.sh_degree, 1.3)
    PU.compare_tokens(z, O.finalize(o["proj"], o["acc"], sc, 1.3))


def test_sharded_tokens_single_rank_nccl():
    """The sharding module's own path (reduce-scatter over a one-rank NCCL group)."""
    import socket

    import torch
    import torch.distributed as dist
    from gaussian_splatting_raster_b200 import runner, sharding

    sc = scenes.make(2)
    obs = O.observe(sc, "f")
    ds = runner.to_device(sc)
    obs_t = torch.as_tensor(np.ascontiguousarray(obs, np.float32)).cuda()
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, device_id=torch.device("cuda:0"))
    try:
        ws = runner.workspace_for(ds)
        z, (lo, hi), out, n = sharding.sharded_tokens(ws, ds, obs_t, 0.9)
        torch.cuda.synchronize()
        ws.close()
    finally:
        dist.destroy_process_group()
    assert (lo, hi) == (0, sc.G) and len(n) == sc.V
    o = O.run(sc, obs, "f", lam=0.9)
    PU.compare_tokens(z.cpu().numpy(), o["tokens"])
    PU.compare_render({"img": out.img.cpu().numpy(), "T": out.T.cpu().numpy(),
                       "n_contrib": out.n_contrib.cpu().numpy(), "last": o["last"]}, o)


def test_partials_reject_bad_shapes():
    import torch
    from gaussian_splatting_raster_b200 import SplatError, finalize_partials, runner

    sc = scenes.tiny_scene(3, 64, 32, 32, V=1, deg=1)
    ds = runner.to_device(sc)
    ws = runner.workspace_for(ds)
    ws.project(ds.means, ds.log_scales, ds.quats, ds.opac, ds.sh, ds.viewmats, ds.intrin,
               ds.H, ds.W)
    with pytest.raises(SplatError) as e:  # projected, but neither binned nor rendered
        ws.score_partials(torch.zeros((1, 32, 32, 3), device="cuda"),
                          torch.zeros((64, 23), device="cuda"))
    assert e.value.code == -3
    ws.close()
    with pytest.raises((SplatError, ValueError)):  # wrong row width
        finalize_partials(torch.zeros((64, 22), device="cuda"), 1,
                          torch.zeros((64, 21), device="cuda"))
