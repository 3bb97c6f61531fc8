"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and compare with the
CPU oracle (fp32 decision mode)."""
from __future__ import annotations

import numpy as np

from oracle import oracle as O

# tolerances (see the design notes): colour 1e-5 absolute; tokens 1e-4 relative L2 per Gaussian
# with a floor of 1e-3 x the median token norm
COLOUR_ATOL = 1e-5
TOKEN_RTOL = 1e-4
TOKEN_FLOOR = 1e-3
# the SH basis is evaluated by different formulas on the two sides (Cartesian polynomials in fp32
# vs associated Legendre functions in double), so SH colours agree to a few ulp, not bitwise
SH_COLOUR_ATOL = 4e-6


def gpu_run(scene, obs, lam=1.0, with_acc=True, det=False, fused=True):
    """The CUDA path over one scene; det=True uses the deterministic accumulation mode (sums
    independent of the order of the additions); fused=False renders and scores with two calls
    (splat_render, splat_score_replay) instead of splat_render_score."""
    import torch
    from gaussian_splatting_raster_b200 import runner

    ds = runner.to_device(scene)
    ws = runner.workspace_for(ds)
    if det:
        ws.deterministic(True)
    out = runner.alloc_outputs(ds)
    obs_t = torch.as_tensor(np.ascontiguousarray(obs, np.float32)).cuda()
    n = runner.render_and_score(ws, ds, obs_t, out, lam, fused=fused)
    V, G, H, W = ds.V, ds.G, ds.H, ds.W
    TX, TY = O.n_tiles(H, W)
    res = dict(n_per_view=n, img=out.img, T=out.T, n_contrib=out.n_contrib, tokens=out.tokens)
    if G > 0:
        rec = torch.empty((V, G, 16), dtype=torch.float32, device="cuda")
        rect = torch.empty((V, G, 4), dtype=torch.int32, device="cuda")
        ws.copy_projection(rec, rect)
        res["rec"], res["rect"] = rec, rect
    off = torch.empty((V, TX * TY + 1), dtype=torch.int64, device="cuda")
    ids = torch.empty((max(sum(n), 1),), dtype=torch.int32, device="cuda")
    ws.copy_tile_lists(off, ids)
    last = torch.empty((V, H, W), dtype=torch.int32, device="cuda")
    ws.copy_last(last)
    res["off"], res["ids"], res["last"] = off, ids[: sum(n)], last
    if with_acc and G > 0:
        acc = torch.empty((V, G, 8), dtype=torch.float64, device="cuda")
        ws.copy_accumulators(acc)
        res["acc"] = acc
    res["pairs"] = ws.pair_count()
    res["launches"] = ws.launch_count
    torch.cuda.synchronize()
    out_np = {k: (v.cpu().numpy() if hasattr(v, "cpu") else v) for k, v in res.items()}
    ws.close()
    return out_np


def compare_projection(scene, g, p):
    """Bitwise on everything that decides an integer or feeds alpha; SH colours to a few ulp."""
    valid_g = (g["rec"][..., 15].view(np.int32) & 256) != 0
    assert (valid_g == (p["valid"] == 1)).all(), "visibility differs"
    v = valid_g
    gr, orr = g["rec"][v].astype(np.float64), p["rec"][v]
    # GPU record: mx my a b c o cr cg cb cut ex ey z xc yc flags
    pairs = [(0, 0), (1, 1), (2, 2), (3, 3), (4, 4), (5, 6), (12, 5), (13, 10), (14, 11)]
    for gi, oi in pairs:
        bad = gr[:, gi] != orr[:, oi]
        assert not bad.any(), f"record field {gi} differs in {bad.sum()} places"
    assert (g["rect"][v] == p["rect"][v]).all(), "tile rectangles differ"
    assert (g["rect"][~v] == 0).all()
    col_g, col_o = gr[:, 6:9], orr[:, 7:10]
    assert np.abs(col_g - col_o).max(initial=0) <= SH_COLOUR_ATOL
    m_g = g["rec"][v][:, 15].view(np.int32) & 7
    m_o = orr[:, 13].astype(np.int32)
    diff = m_g != m_o
    # a clamp decision may only differ where the pre-clamp colour is within rounding of zero:
    # the channels whose bits differ have colours of at most a few ulp on both sides
    ch_diff = ((m_g ^ m_o)[:, None] >> np.arange(3)[None, :]) & 1 == 1
    if ch_diff.any():
        assert np.maximum(col_g[ch_diff], col_o[ch_diff]).max() < 1e-5
    # Gaussians with such a near-tie are excluded from the token comparison
    near = np.zeros(p["valid"].shape, bool)
    near[v] = diff
    return near.any(0)


def compare_lists(g, L):
    assert (g["off"] == L["off"]).all(), "tile offsets differ"
    assert g["ids"].shape[0] == L["n"]
    assert (g["ids"] == L["ids"]).all(), "per-tile order differs"


def compare_render(g, r, mask=None):
    sel = (slice(None),) if mask is None else (mask,)
    img_g, img_o = g["img"][sel], r["img"][sel]
    assert np.abs(img_g - img_o).max(initial=0) <= COLOUR_ATOL
    assert (g["T"][sel] == r["T"][sel].astype(np.float32)).all(), "final transmittance differs"
    assert (g["n_contrib"][sel] == r["n_contrib"][sel]).all(), "contributor counts differ"
    assert (g["last"][sel] == r["last"][sel]).all(), "list bounds differ"


def token_errors(zg, zo):
    norms = np.linalg.norm(zo, axis=1)
    floor = TOKEN_FLOOR * max(np.median(norms), 1e-30)
    return np.linalg.norm(zg - zo, axis=1) / np.maximum(norms, floor)


def compare_tokens(zg, zo, exclude=None, which=None):
    idx = np.arange(zo.shape[0]) if which is None else np.asarray(which)
    if exclude is not None:
        idx = idx[~exclude[idx]]
    err = token_errors(zg[idx].astype(np.float64), zo[idx])
    assert err.max(initial=0) <= TOKEN_RTOL, f"token error {err.max()} at {idx[err.argmax()]}"
    return err


# renderer backward -------------------------------------------------------------------------------
GRAD_RTOL = 1e-4
GRAD_BLOCK_RTOL = 1e-3
GRAD_VARIANTS = ("raw", "detached", "support", "pscale")


def grad_blocks(K):
    return {"mean": (0, 3), "log_scale": (3, 6), "quat": (6, 10), "opacity": (10, 11),
            "sh": (11, K)}


def gpu_backward(scene, obs, variants=GRAD_VARIANTS):
    import torch
    from gaussian_splatting_raster_b200 import grad_dim, runner

    ds = runner.to_device(scene)
    ws = runner.workspace_for(ds)
    out = runner.alloc_outputs(ds)
    obs_t = torch.as_tensor(np.ascontiguousarray(obs, np.float32)).cuda()
    K = grad_dim(ds.deg)
    grads = {k: torch.full((ds.G, K), float("nan"), dtype=torch.float32, device="cuda")
             for k in variants}
    runner.render_and_backward(ws, ds, obs_t, out, grads)
    res = {k: v for k, v in grads.items()}
    res.update(img=out.img, T=out.T, n_contrib=out.n_contrib)
    if ds.G > 0:
        rec = torch.empty((ds.V, ds.G, 16), dtype=torch.float32, device="cuda")
        rect = torch.empty((ds.V, ds.G, 4), dtype=torch.int32, device="cuda")
        ws.copy_projection(rec, rect)
        res["rec"], res["rect"] = rec, rect
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in res.items()}
    res["launches"] = ws.launch_count
    ws.close()
    return res


def compare_grads(gg, go, which=None, exclude=None, rtol=GRAD_RTOL, block_rtol=GRAD_BLOCK_RTOL):
    """Two bars. (1) Per Gaussian, the whole row with every block scaled by that block's median
    norm over the Gaussians: relative L2 <= rtol (floor 1e-3), the bar the tokens meet. (2) Per
    Gaussian and block: relative L2 <= block_rtol (floor 1e-3 x the block's median norm); looser,
    because a block that is a sum of terms of both signs (the opacity logit's above all) can be
    far smaller than its terms, and its fp32 rounding is relative to the terms. Returns the worst
    block errors."""
    K = go.shape[1]
    idx = np.arange(go.shape[0]) if which is None else np.asarray(which)
    if exclude is not None:
        idx = idx[~exclude[idx]]
    worst = {}
    gs, os_ = [], []
    for name, (lo, hi) in grad_blocks(K).items():
        o = go[idx, lo:hi]
        g = gg[idx, lo:hi].astype(np.float64)
        assert np.isfinite(g).all(), f"{name}: non-finite gradient"
        norms = np.linalg.norm(o, axis=1)
        nz = norms[norms > 0]
        if nz.size == 0:
            assert (g == 0).all(), f"{name}: expected zeros"
            worst[name] = 0.0
            continue
        med = np.median(nz)
        err = np.linalg.norm(g - o, axis=1) / np.maximum(norms, TOKEN_FLOOR * med)
        worst[name] = float(err.max())
        assert err.max() <= block_rtol, f"{name}: error {err.max()} at Gaussian {idx[err.argmax()]}"
        gs.append(g / med)
        os_.append(o / med)
    if gs:
        g, o = np.concatenate(gs, 1), np.concatenate(os_, 1)
        n = np.linalg.norm(o, axis=1)
        err = np.linalg.norm(g - o, axis=1) / np.maximum(n, TOKEN_FLOOR)
        worst["row"] = float(err.max())
        assert err.max() <= rtol, f"row error {err.max()} at Gaussian {idx[err.argmax()]}"
    return worst
