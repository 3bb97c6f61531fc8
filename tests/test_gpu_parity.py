"""CUDA path (through the C ABI) against the CPU oracle, element by element.

Bars: visibility, tile rectangles, tile offsets, per-tile order, final transmittance, contributor
counts and list bounds bit-exact; projected means/conics/opacity/depth bitwise; colour within
1e-5; tokens within 1e-4 relative L2 per Gaussian (floor 1e-3 x median norm).
"""
import math

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


def _full_check(sc, obs, lam=1.0, fused=True):
    g = PU.gpu_run(sc, obs, lam, fused=fused)
    o = O.run(sc, obs, "f", lam=lam)
    near = PU.compare_projection(sc, g, o["proj"]) if sc.G > 0 else np.zeros(0, bool)
    PU.compare_lists(g, o["lists"])
    PU.compare_render(g, o)
    assert g["pairs"] == int(o["last"].sum())
    if sc.G > 0:
        PU.compare_tokens(g["tokens"], o["tokens"], exclude=near)
    return g, o


def _replay_traversals(sc, o, union_lanes=9):
    """How many warp blocks (8x4 pixels of a 16x16 tile) the score replay runs as per-pixel walks
    and how many as the union loop: a warp takes the union loop when its pixels' composited pairs
    P are at least union_lanes times the entries U that some pixel of the block composited.
    Counted here from the oracle's per-pixel composited entries."""
    p, L = o["proj"], o["lists"]
    TX, TY = O.n_tiles(sc.H, sc.W)
    walk = union = 0
    for v in range(sc.V):
        for t in range(TX * TY):
            seg = L["ids"][L["off"][v, t]:L["off"][v, t + 1]]
            pos = {int(gg): k for k, gg in enumerate(seg)}
            tx, ty = t % TX, t // TX
            for w in range(8):
                x0, y0 = tx * 16 + (w % 2) * 8, ty * 16 + (w // 2) * 4
                U, P = set(), 0
                for lane in range(32):
                    i, j = x0 + lane % 8, y0 + lane // 8
                    if i >= sc.W or j >= sc.H:
                        continue
                    tr = O.trace(p, L, sc.H, sc.W, sc.bg, v, i, j, "f", cap=8192)
                    U |= {pos[int(gg)] for gg in tr[:, 0]}
                    P += int(o["n_contrib"][v, j, i])
                if U:
                    union += P >= union_lanes * len(U)
                    walk += P < union_lanes * len(U)
    return walk, union


@pytest.mark.parametrize("fused", [True, False], ids=["render_score", "two_calls"])
@pytest.mark.parametrize("cfg", [1, 2])
def test_small_configs_full_parity(cfg, fused):
    """Full parity on the two small workloads, through splat_render_score (render and replay in
    one kernel) and through splat_render + splat_score_replay. Both of the score replay's
    traversals run here: on the three-layer scene about two thirds of the warp blocks walk their
    pixels' entries and a third take the union loop (checked below), so the token comparison
    covers both."""
    sc = scenes.make(cfg)
    obs = O.observe(sc, "f")
    g, o = _full_check(sc, obs, fused=fused)
    assert g["n_contrib"].max() > 1
    if cfg == 2:
        walk, union = _replay_traversals(sc, o)
        assert walk > 100 and union > 100, (walk, union)


def test_exact_depth_ties_keep_index_order():
    sc = scenes.make(1)  # every Gaussian of a plane has the same camera depth
    obs = O.observe(sc, "f")
    g = PU.gpu_run(sc, obs)
    o = O.run(sc, obs, "f")
    PU.compare_lists(g, o["lists"])
    # inside each tile, equal depths appear in increasing index
    rec = o["proj"]["rec"][0]
    off, ids = g["off"][0], g["ids"]
    for t in range(off.shape[0] - 1):
        seg = ids[off[t]:off[t + 1]]
        d = rec[seg, 5]
        key = np.lexsort((seg, d))
        assert (key == np.arange(len(seg))).all()


@pytest.mark.parametrize("deg", [0, 2, 3])
def test_sh_degrees_and_ragged_image(deg):
    sc = scenes.tiny_scene(40 + deg, 300, 37, 53, V=3, deg=deg, hi_sigma=0.2)
    obs = np.random.default_rng(deg).uniform(0, 1, (sc.V, sc.H, sc.W, 3)).astype(np.float32)
    _full_check(sc, obs, lam=0.5)



def test_clamp_scene_tokens():
    """Both score masks active: Gaussian 1 saturates at alpha = 0.99 on a few pixel centres
    (M_alpha removes those pixels from its opacity and centre scores) and the red channel of
    Gaussian 2 is clamped (M_color removes it from the SH block). The oracle's masks are pinned to
    finite differences on this scene; the GPU tokens meet the usual bar against them."""
    sc = scenes.clamp_scene()
    obs = np.random.default_rng(5).uniform(0.2, 0.8, (sc.V, sc.H, sc.W, 3)).astype(np.float32)
    g, o = _full_check(sc, obs)
    flags = g["rec"][:, :, 15].view(np.int32)
    assert ((flags[:, 2] & 7) == 6).all()  # red clamped in every view, on the GPU side too
    p, L = o["proj"], o["lists"]
    n_sat = 0
    for v in range(sc.V):
        for j in range(sc.H):
            for i in range(sc.W):
                tr = O.trace(p, L, sc.H, sc.W, sc.bg, v, i, j, "f")
                n_sat += int(((tr[:, 0] == 1) & (tr[:, 1] == np.float32(0.99))).sum())
    assert n_sat >= 4  # alpha clamp reached with the kernels' fp32 decisions
    assert np.abs(g["tokens"][2, 4::3][: sc.d]).max() == 0.0  # clamped channel: zero SH score

def test_long_tile_list():
    """One 16x16 tile with 12000 overlapping Gaussians: a list of more than 8192 entries (many
    32-entry chunks per warp, several counting-sort blocks for one tile) in bit-exact order, with
    the render and tokens at their usual bars."""
    sc = scenes.tiny_scene(7, 12000, 16, 16, V=1, deg=1, depth_range=(1.0, 60.0),
                           log_scale_mean=math.log(0.05))
    obs = np.full((1, 16, 16, 3), 0.3, np.float32)
    g, o = _full_check(sc, obs)
    assert o["lists"]["n"] > 8192


def test_mixed_footprints_in_one_warp():
    """Instance emission with very uneven rectangles side by side in depth order: Gaussians that
    cover every tile of a ragged 7 x 10 tile grid, culled ones (no instance) and small ones,
    G not a multiple of 32."""
    sc = scenes.tiny_scene(21, 1061, 100, 150, V=2, deg=1, log_scale_mean=math.log(0.02))
    rng = np.random.default_rng(5)
    big = rng.choice(sc.G, 90, replace=False)
    sc.log_scales[big] = math.log(3.0)  # footprint larger than the image
    culled = rng.choice(np.setdiff1d(np.arange(sc.G), big), 200, replace=False)
    sc.means[culled, 2] = -1.0
    obs = np.random.default_rng(2).uniform(0, 1, (2, 100, 150, 3)).astype(np.float32)
    g, o = _full_check(sc, obs)
    rect = o["proj"]["rect"]
    counts = (rect[..., 2] - rect[..., 0]) * (rect[..., 3] - rect[..., 1])
    assert counts.max() == 70 and (counts == 0).sum() >= 2 * 200


def test_step_beside_large_copies_on_other_streams():
    """The step's host exchange (instance counts out, view starts back) goes through mapped
    memory, not a copy engine: a render + replay enqueued while 1 GiB host->device and
    device->host copies are in flight on two other streams gives the same bits as a quiet run
    (both in deterministic mode, so the sums do not depend on the order of the additions), and
    the binning's count readback does not wait for those copies to finish."""
    import time
    import torch
    from gaussian_splatting_raster_b200 import runner
    sc = scenes.make(2)
    obs = O.observe(sc, "f")
    quiet = PU.gpu_run(sc, obs, with_acc=False, det=True)
    n = 256 * 1024 * 1024  # 1 GiB of float32 each way
    h_src = torch.empty(n, dtype=torch.float32).pin_memory()
    h_dst = torch.empty(n, dtype=torch.float32).pin_memory()
    d_dst = torch.empty(n, device="cuda")
    d_src = torch.zeros(n, device="cuda")
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ds = runner.to_device(sc)
    ws = runner.workspace_for(ds)
    ws.deterministic(True)
    out = runner.alloc_outputs(ds)
    obs_t = torch.as_tensor(obs).cuda()
    # one step first: a workspace grows its instance lists on first use, and a device allocation
    # synchronises with every stream (steady-state steps allocate nothing)
    runner.render_and_score(ws, ds, obs_t, out)
    torch.cuda.synchronize()
    copies_done = torch.cuda.Event()
    with torch.cuda.stream(s_in):
        d_dst.copy_(h_src, non_blocking=True)
    with torch.cuda.stream(s_out):
        h_dst.copy_(d_src, non_blocking=True)
        copies_done.record(s_out)
    t0 = time.perf_counter()
    runner.render_and_score(ws, ds, obs_t, out)  # bin_sort returns once its counts are read
    t_step = time.perf_counter() - t0
    in_flight = not copies_done.query()
    torch.cuda.synchronize()
    assert (out.img.cpu().numpy() == quiet["img"]).all()
    assert (out.n_contrib.cpu().numpy() == quiet["n_contrib"]).all()
    assert (out.tokens.cpu().numpy() == quiet["tokens"]).all()
    ws.close()
    # the copies take tens of ms; the readback must not have waited for them
    assert in_flight, f"the step ({t_step * 1e3:.1f} ms) ended after the copies"


def test_empty_scene_and_all_culled():
    sc = scenes.tiny_scene(3, 5, 20, 24, V=2)
    sc.means[:, 2] = -1.0  # all behind the cameras
    obs = np.zeros((2, 20, 24, 3), np.float32)
    g, o = _full_check(sc, obs)
    assert sum(g["n_per_view"]) == 0
    assert (g["img"] == 0).all() and (g["T"] == 1).all()
    # G = 0
    sc0 = scenes.tiny_scene(3, 1, 20, 24, V=1)
    for name in ("means", "log_scales", "quats", "opac", "sh"):
        setattr(sc0, name, getattr(sc0, name)[:0])
    sc0.bg = np.array([0.25, 0.5, 0.75], np.float32)
    g0 = PU.gpu_run(sc0, np.zeros((1, 20, 24, 3), np.float32), with_acc=False)
    assert (g0["img"] == sc0.bg).all() and g0["tokens"].shape == (0, 21)


def test_nonzero_background_and_lambda():
    sc = scenes.tiny_scene(9, 200, 48, 64, V=2, deg=1)
    sc.bg = np.array([0.1, 0.6, 0.3], np.float32)
    obs = np.random.default_rng(1).uniform(0, 1, (2, 48, 64, 3)).astype(np.float32)
    _full_check(sc, obs, lam=2.5)


def test_calls_out_of_order_and_bad_arguments():
    import torch
    from gaussian_splatting_raster_b200 import SplatError, Workspace
    ws = Workspace(16, 1, 16, 16, 1)
    with pytest.raises(SplatError) as e:
        ws.bin_sort()
    assert e.value.code == -3
    z = torch.zeros((16, 3), device="cuda")
    with pytest.raises(SplatError) as e:  # more Gaussians than the workspace holds
        ws.project(torch.zeros((17, 3), device="cuda"), torch.zeros((17, 3), device="cuda"),
                   torch.zeros((17, 4), device="cuda"), torch.zeros((17,), device="cuda"),
                   torch.zeros((17, 4, 3), device="cuda"), torch.eye(4, device="cuda")[None],
                   torch.ones((1, 4), device="cuda"), 16, 16)
    assert e.value.code == -2
    with pytest.raises(TypeError):  # host tensor
        ws.project(z.cpu(), z, z, z[:, 0], torch.zeros((16, 4, 3), device="cuda"),
                   torch.eye(4, device="cuda")[None], torch.ones((1, 4), device="cuda"), 16, 16)
    ws.close()


def test_render_score_equals_two_calls():
    """ReSplat-scale workload: splat_render_score gives the image, final T, contributor counts,
    list bounds and tile lists of splat_render bit for bit, and the tokens of splat_score_replay
    up to the order of the fp32 reductions."""
    sc = scenes.make(3)
    obs = scenes.smooth_observation(91, sc.V, sc.H, sc.W)
    a = PU.gpu_run(sc, obs, fused=True)
    b = PU.gpu_run(sc, obs, fused=False)
    for k in ("img", "T", "n_contrib", "last", "off", "ids", "rec", "rect"):
        assert np.array_equal(a[k], b[k]), k
    err = PU.token_errors(a["tokens"].astype(np.float64), b["tokens"].astype(np.float64))
    assert err.max() <= 1e-5, err.max()
    assert np.abs(a["acc"] - b["acc"]).max() <= 1e-5 * np.abs(b["acc"]).max()


def test_repeated_replays_start_from_cleared_sums():
    """The projection clears the replay's per-(view, Gaussian) sums; a replay that finds them
    already used (a second replay after one projection, here after splat_render_score) clears them
    itself, so every call gives the same tokens (up to the order of the fp32 reductions); twice
    the sums would double q_g and change every token."""
    import torch
    from gaussian_splatting_raster_b200 import runner
    sc = scenes.make(2)
    obs = O.observe(sc, "f")
    ds = runner.to_device(sc)
    ws = runner.workspace_for(ds)
    out = runner.alloc_outputs(ds)
    obs_t = torch.as_tensor(obs).cuda()
    runner.render_and_score(ws, ds, obs_t, out)
    z1 = out.tokens.cpu().numpy().astype(np.float64)
    for _ in range(2):
        ws.score_replay(obs_t, out.tokens)
        z = out.tokens.cpu().numpy().astype(np.float64)
        assert PU.token_errors(z, z1).max() <= 1e-5
    ws.render_score(ds.bg, obs_t, out.img, out.T, out.n_contrib, out.tokens)
    z = out.tokens.cpu().numpy().astype(np.float64)
    assert PU.token_errors(z, z1).max() <= 1e-5
    ws.close()


def test_most_tiles_a_workspace_holds():
    """An image of 7,264 16x16 tiles (the largest the binning's per-warp shared-memory counts
    hold) renders and scores like the oracle; one tile more is refused at workspace creation."""
    from gaussian_splatting_raster_b200 import SplatError, Workspace
    with pytest.raises(SplatError) as e:
        Workspace(16, 1, 16, 16 * 7265, 1)
    assert e.value.code == -2
    sc = scenes.tiny_scene(61, 300, 16, 16 * 7264, V=1, deg=1)
    obs = np.random.default_rng(61).uniform(0, 1, (1, 16, 16 * 7264, 3)).astype(np.float32)
    _full_check(sc, obs)


@pytest.mark.parametrize("cfg", [3, 4, 5])
def test_full_size_sampled(cfg):
    """Full-size workloads: projection and every tile list compared in full; render on sampled
    tiles; tokens of sampled Gaussians (the oracle replays every tile those Gaussians touch)."""
    sc = scenes.make(cfg)
    obs = scenes.smooth_observation(77 + cfg, sc.V, sc.H, sc.W)
    g = PU.gpu_run(sc, obs)
    p = O.project(sc, "f")
    near = PU.compare_projection(sc, g, p)
    L = O.bin_lists(p, sc.H, sc.W)
    PU.compare_lists(g, L)
    rng = np.random.default_rng(cfg)
    TX, TY = O.n_tiles(sc.H, sc.W)
    # sampled Gaussians (visible somewhere, no colour near-tie) and the tiles they touch
    cand = np.nonzero(p["valid"].any(0) & ~near)[0]
    gs = rng.choice(cand, size=64, replace=False)
    sel = set()
    for v in range(sc.V):
        for gg in gs:
            if p["valid"][v, gg]:
                x0, y0, x1, y1 = p["rect"][v, gg]
                sel.update((v, ty * TX + tx) for ty in range(y0, y1) for tx in range(x0, x1))
    # plus random tiles for the image checks
    sel.update((int(rng.integers(sc.V)), int(rng.integers(TX * TY))) for _ in range(16))
    sel = np.array(sorted(sel), np.int32)
    r = O.render(p, L, sc.H, sc.W, sc.bg, "f", sel=sel)
    mask = np.zeros((sc.V, sc.H, sc.W), bool)
    for v, t in sel:
        tx, ty = t % TX, t // TX
        mask[v, ty * 16:(ty + 1) * 16, tx * 16:(tx + 1) * 16] = True
    PU.compare_render(g, r, mask)
    acc = O.replay(p, L, r, obs, sc.sh_degree, sc.H, sc.W, "f", sel=sel)["acc"]
    z = O.finalize(p, acc, sc)
    PU.compare_tokens(g["tokens"], z, which=gs)
    # the accumulated supports of the sampled Gaussians agree too
    np.testing.assert_allclose(g["acc"][:, gs, 0], acc[:, gs, 0], rtol=1e-5, atol=1e-6)
