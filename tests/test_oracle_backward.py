"""Pins of the oracle's renderer backward (the gradient comparators of "Relation to Gradient" in
"Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting"):

* the SH-basis gradient (polynomial form) against the basis by its definition and central
  differences along the sphere;
* the raw gradient of L = 1/2 sum |C_hat - C_obs|^2 against central finite differences of the
  oracle's own render, for every parameter of every Gaussian (means, log-scales, quaternions,
  opacity logits, SH), at SH degrees 0, 1 and 3, and with the tangent clamp, the alpha clamp and
  the colour clamp active;
* raw and detached gradients against PyTorch autograd through a dense renderer written here from
  the forward definitions (per-pixel depth order, no tiles; spherical-coordinate SH);
* the support normaliser against the weights-sum invariant, and the parameter-scale variant
  against finite differences in units of the Gaussian's size.
"""
import copy
import math

import numpy as np
import pytest

from oracle import oracle as O
from synth import scenes

BLOCKS = {"means": 0, "log_scales": 3, "quats": 6, "opac": 10, "sh": 11}


def _copy(sc):
    s2 = copy.copy(sc)
    for k in BLOCKS:
        setattr(s2, k, getattr(sc, k).copy())
    return s2


def _loss(sc, obs):
    p = O.project(sc, "d")
    L = O.bin_lists(p, sc.H, sc.W)
    r = O.render(p, L, sc.H, sc.W, sc.bg, "d")
    return 0.5 * ((r["img"] - obs) ** 2).sum()


def _obs(sc, seed):
    return np.random.default_rng(seed).uniform(0.2, 0.8, (sc.V, sc.H, sc.W, 3)).astype(np.float32)


def _tiny(seed, deg):
    return scenes.tiny_scene(seed, 4, 24, 32, V=2, deg=deg, opac_mean=0.0, opac_sigma=0.5,
                             log_scale_mean=math.log(0.06))


def _clamp_scene():
    """Gaussian 0 centred beyond 1.3x the half field of view (tangent clamp) but reaching the
    image; Gaussian 1 opaque and small (alpha clamped at 0.99 near its centre); Gaussian 2 with a
    colour channel clamped at zero."""
    sc = _tiny(41, 1)
    sc.means[0] = [2.1, 0.1, 3.0]
    sc.log_scales[0] = np.log([0.35, 0.3, 0.4])
    sc.opac[1] = 6.0
    sc.log_scales[1] = np.log([0.15, 0.12, 0.1])
    sc.sh[2, 0, 0] = -3.0
    return sc


# ------------------------------------------------------------------------------------------------

def test_sh_gradient_matches_definition_and_sphere_differences():
    rng = np.random.default_rng(0)
    d = rng.normal(size=(64, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    B, dB = O.sh_poly_grad(3, d)
    np.testing.assert_allclose(B, O.sh_basis(3, d), atol=1e-14)
    h = 1e-6
    for i in range(d.shape[0]):
        t = rng.normal(size=3)
        t -= d[i] * (t @ d[i])
        t /= np.linalg.norm(t)
        dp, dm = d[i] + h * t, d[i] - h * t
        dp, dm = dp / np.linalg.norm(dp), dm / np.linalg.norm(dm)
        fd = (O.sh_basis(3, dp[None])[0] - O.sh_basis(3, dm[None])[0]) / (2 * h)
        np.testing.assert_allclose(dB[i] @ t, fd, atol=5e-9)


def _fd_check(sc, seed, h=1e-5, tol=2e-7):
    obs = _obs(sc, seed)
    g = O.run_backward(sc, obs, "d")["raw"]
    for name, col0 in BLOCKS.items():
        arr = getattr(sc, name)
        for gi in range(sc.G):
            for c in range(arr[gi].size):
                full = (gi,) + (np.unravel_index(c, arr[gi].shape) if arr.ndim > 1 else ())
                sp, sm = _copy(sc), _copy(sc)
                getattr(sp, name)[full] += h
                getattr(sm, name)[full] -= h
                # the inputs are fp32: divide by the perturbation actually stored
                step = float(getattr(sp, name)[full]) - float(getattr(sm, name)[full])
                fd = (_loss(sp, obs) - _loss(sm, obs)) / step
                an = g[gi, col0 + c]
                scale = np.abs(g[gi]).max()
                assert abs(fd - an) <= tol * scale, (name, gi, c, fd, an)


@pytest.mark.parametrize("seed,deg", [(21, 1), (22, 1), (23, 1), (31, 0), (32, 3)])
def test_raw_gradient_equals_central_differences(seed, deg):
    _fd_check(_tiny(seed, deg), seed)


def test_raw_gradient_with_clamps_active():
    sc = _clamp_scene()
    p = O.project(sc, "d")
    u = p["rec"][:, 0, 10] / p["rec"][:, 0, 12]
    lim = 1.3 * 0.5 * sc.W / sc.intrin[:, 0]
    assert (np.abs(u) > lim).all() and p["valid"][:, 0].all()  # tangent clamp in every view
    assert (p["rec"][:, 2, 13] == 6).all()                    # red channel of Gaussian 2 clamped
    L = O.bin_lists(p, sc.H, sc.W)
    alphas = []
    for v in range(sc.V):
        i, j = int(p["rec"][v, 1, 0]), int(p["rec"][v, 1, 1])
        tr = O.trace(p, L, sc.H, sc.W, sc.bg, v, i, j, "d")
        alphas += list(tr[tr[:, 0] == 1, 1])
    assert max(alphas) == pytest.approx(0.99)                 # alpha clamp reached
    r = O.render(p, L, sc.H, sc.W, sc.bg, "d")
    assert (r["n_contrib"] > 0).any()
    _fd_check(sc, 41)


# ------------------------------------------------------------------------------------------------
# autograd through a dense renderer written from the forward definitions

def _sh_torch(deg, dirs):
    """Real SH with the Condon-Shortley phase through spherical coordinates (autograd-able)."""
    import torch
    x, y, z = dirs[:, 0], dirs[:, 1], dirs[:, 2]
    ct = z
    st = torch.sqrt(x * x + y * y)
    phi = torch.atan2(y, x)
    P = {}
    for m in range(deg + 1):
        pmm = torch.ones_like(ct)
        for i in range(1, m + 1):
            pmm = pmm * (-(2.0 * i - 1.0)) * st
        P[(m, m)] = pmm
        if m + 1 <= deg:
            P[(m + 1, m)] = ct * (2.0 * m + 1.0) * pmm
        for l in range(m + 2, deg + 1):
            P[(l, m)] = ((2.0 * l - 1.0) * ct * P[(l - 1, m)] - (l + m - 1.0) * P[(l - 2, m)]) / (l - m)
    out = []
    for l in range(deg + 1):
        for m in range(-l, l + 1):
            am = abs(m)
            K = math.sqrt((2 * l + 1) / (4 * math.pi) * math.factorial(l - am) / math.factorial(l + am))
            if m == 0:
                out.append(K * P[(l, 0)])
            elif m > 0:
                out.append(math.sqrt(2) * K * P[(l, am)] * torch.cos(am * phi))
            else:
                out.append(math.sqrt(2) * K * P[(l, am)] * torch.sin(am * phi))
    return torch.stack(out, 1)


def _dense_loss(sc, obs, p, params, detach_cov=False, detach_dir=False):
    import torch
    means, lsc, quats, opac, sh = params
    qn = quats / quats.norm(dim=1, keepdim=True)
    w, x, y, z = qn.unbind(1)
    Rq = torch.stack([
        torch.stack([1 - 2 * (y * y + z * z), 2 * (x * y - w * z), 2 * (x * z + w * y)], 1),
        torch.stack([2 * (x * y + w * z), 1 - 2 * (x * x + z * z), 2 * (y * z - w * x)], 1),
        torch.stack([2 * (x * z - w * y), 2 * (y * z + w * x), 1 - 2 * (x * x + y * y)], 1)], 1)
    M = Rq * torch.exp(lsc)[:, None, :]
    Sig = M @ M.transpose(1, 2)
    o = torch.sigmoid(opac)
    H, W = sc.H, sc.W
    loss = torch.zeros((), dtype=torch.float64)
    ii, jj = np.meshgrid(np.arange(W), np.arange(H))
    px = torch.tensor(ii.ravel() + 0.5, dtype=torch.float64)
    py = torch.tensor(jj.ravel() + 0.5, dtype=torch.float64)
    for v in range(sc.V):
        Rv = torch.tensor(sc.viewmats[v, :3, :3].astype(np.float64))
        tv = torch.tensor(sc.viewmats[v, :3, 3].astype(np.float64))
        fx, fy, cx, cy = (float(a) for a in sc.intrin[v])
        xc = means @ Rv.T + tv
        X, Y, Z = xc.unbind(1)
        limx, limy = 1.3 * 0.5 * W / fx, 1.3 * 0.5 * H / fy
        uc = torch.clamp(X / Z, -limx, limx)
        vc = torch.clamp(Y / Z, -limy, limy)
        zero = torch.zeros_like(Z)
        J = torch.stack([torch.stack([fx / Z, zero, -fx * uc / Z], 1),
                         torch.stack([zero, fy / Z, -fy * vc / Z], 1)], 1)
        Sc = Rv @ Sig @ Rv.T
        S2 = J @ Sc @ J.transpose(1, 2) + 0.3 * torch.eye(2, dtype=torch.float64)
        Q = torch.linalg.inv(S2)
        if detach_cov:
            Q = Q.detach()
        mx, my = fx * X / Z + cx, fy * Y / Z + cy
        cam = -(Rv.T @ tv)
        dv = means - cam
        dirs = dv / dv.norm(dim=1, keepdim=True)
        if detach_dir:
            dirs = dirs.detach()
        col = torch.clamp(torch.einsum("gk,gkc->gc", _sh_torch(sc.sh_degree, dirs), sh) + 0.5,
                          min=0.0)
        # per pixel, every visible Gaussian whose tile rectangle holds the pixel, by (depth, index)
        vis = np.nonzero(p["valid"][v])[0]
        order = vis[np.lexsort((vis, p["rec"][v, vis, 5]))]
        dx = px[:, None] - mx[None, order]
        dy = py[:, None] - my[None, order]
        Qo = Q[order]
        pw = -0.5 * (Qo[:, 0, 0] * dx * dx + Qo[:, 1, 1] * dy * dy) - Qo[:, 0, 1] * dx * dy
        al = torch.clamp(o[order] * torch.exp(pw), max=0.99)
        rect = p["rect"][v, order]
        tx, ty = (ii.ravel() // 16)[:, None], (jj.ravel() // 16)[:, None]
        listed = (tx >= rect[None, :, 0]) & (tx < rect[None, :, 2]) & (ty >= rect[None, :, 1]) & \
                 (ty < rect[None, :, 3])
        # the rasteriser's decisions, taken on the values, then held fixed
        a_np, pw_np = al.detach().numpy(), pw.detach().numpy()
        use = listed & (pw_np <= 0) & (a_np >= 1.0 / 255.0)
        keep = np.zeros_like(use)
        T = np.ones(use.shape[0])
        alive = np.ones(use.shape[0], bool)
        for k in range(use.shape[1]):
            u = use[:, k] & alive
            Tn = T * (1 - a_np[:, k])
            stop = u & (Tn < 1e-4)
            alive &= ~stop
            u &= ~stop
            keep[:, k] = u
            T = np.where(u, Tn, T)
        ae = al * torch.tensor(keep.astype(np.float64))
        Tex = torch.cumprod(torch.cat([torch.ones_like(ae[:, :1]), 1 - ae], 1), 1)
        C = (Tex[:, :-1, None] * ae[:, :, None] * col[order][None]).sum(1) + \
            Tex[:, -1:] * torch.tensor(sc.bg.astype(np.float64))[None]
        r = C - torch.tensor(obs[v].reshape(-1, 3).astype(np.float64))
        loss = loss + 0.5 * (r * r).sum()
    return loss


def _autograd(sc, obs, p, **kw):
    import torch
    params = [torch.tensor(getattr(sc, k).astype(np.float64), requires_grad=True)
              for k in ("means", "log_scales", "quats", "opac", "sh")]
    _dense_loss(sc, obs, p, params, **kw).backward()
    cols = []
    for t in params:
        gt = t.grad if t.grad is not None else torch.zeros_like(t)
        cols.append(gt.reshape(sc.G, -1).numpy())
    return np.concatenate(cols, 1)


@pytest.mark.parametrize("which", ["tiny1", "tiny3", "clamps", "three_layer"])
def test_gradients_equal_autograd_of_dense_renderer(which):
    if which == "three_layer":
        sc = scenes.tiny_scene(7, 40, 40, 56, V=2, deg=2, opac_mean=1.0)
    elif which == "clamps":
        sc = _clamp_scene()
    else:
        sc = _tiny(22, int(which[-1]))
    obs = _obs(sc, 5)
    out = O.run_backward(sc, obs, "d")
    p = out["proj"]
    ref = _autograd(sc, obs, p)
    for lo, hi in ((0, 3), (3, 6), (6, 10), (10, 11), (11, ref.shape[1])):
        assert np.abs(ref[:, lo:hi]).max() > 0  # every block is exercised
    scale = np.abs(ref).max(axis=1, keepdims=True)
    assert np.abs(out["raw"] - ref).max() <= 1e-9 * max(scale.max(), 1e-30)
    np.testing.assert_allclose(out["raw"], ref, rtol=1e-7, atol=1e-9 * scale.max())
    ref_d = _autograd(sc, obs, p, detach_cov=True, detach_dir=True)
    np.testing.assert_allclose(out["detached"], ref_d, rtol=1e-7, atol=1e-9 * scale.max())
    assert (out["detached"][:, 3:10] == 0).all()


def test_support_normaliser_sums_to_coverage():
    """q_g = eps + sum_v (eps + sum_p w); summed over Gaussians the weights give the coverage
    sum_p (1 - T_final) of every pixel (weights plus final transmittance make one)."""
    sc = scenes.tiny_scene(7, 40, 40, 56, V=2, deg=2, opac_mean=1.0)
    obs = _obs(sc, 6)
    out = O.run_backward(sc, obs, "d")
    raw, sup = out["raw"], out["support"]
    k = np.argmax(np.abs(raw), axis=1)
    q = raw[np.arange(sc.G), k] / sup[np.arange(sc.G), k]
    nv = out["proj"]["valid"].sum(0)
    eps = 1e-6
    cover = (1.0 - out["T"]).sum()
    assert abs((q - eps - eps * nv).sum() - cover) <= 1e-9 * cover
    np.testing.assert_allclose(sup * q[:, None], raw, rtol=1e-12, atol=1e-300)


def test_parameter_scale_mean_block_equals_differences_in_gaussian_units():
    sc = _tiny(23, 1)
    obs = _obs(sc, 23)
    out = O.run_backward(sc, obs, "d")
    for g in range(sc.G):
        sig = math.exp(float(np.mean(sc.log_scales[g].astype(np.float64))))
        for c in range(3):
            sp, sm = _copy(sc), _copy(sc)
            sp.means[g, c] += 1e-5 * sig
            sm.means[g, c] -= 1e-5 * sig
            step = (float(sp.means[g, c]) - float(sm.means[g, c])) / sig
            fd = (_loss(sp, obs) - _loss(sm, obs)) / step
            scale = np.abs(out["pscale"][g]).max()
            assert abs(fd - out["pscale"][g, c]) <= 2e-7 * scale
        np.testing.assert_array_equal(out["pscale"][g, 3:], out["raw"][g, 3:])


def test_fp32_decision_mode_agrees_with_double():
    sc = _tiny(22, 1)
    obs = _obs(sc, 22)
    a = O.run_backward(sc, obs, "f")["raw"]
    b = O.run_backward(sc, obs, "d")["raw"]
    err = np.linalg.norm(a - b, axis=1) / np.linalg.norm(b, axis=1)
    assert err.max() < 1e-4
