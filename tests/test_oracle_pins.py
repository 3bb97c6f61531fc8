"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Sources: "Research Proposal: Renderer Score Tokens for Recurrent Gaussian Splatting" (sections
"Two-Stage Algorithm" and "Exact Score Operators"); the 3DGS primitive as summarised on the ATSplat
page ("prerequisites"). Each test names what it pins and against what: closed forms, a brute-force
per-pixel sort without tiles, a back-to-front suffix composite, central finite differences of the
squared residual loss, numpy's eigvalsh, numpy's exp, scipy's spherical harmonics and quadrature.
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.spatial.transform import Rotation
from scipy import special

from oracle import oracle as O
from synth import scenes

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------------------------------
# exp written from Cody & Waite's method, against numpy's exp in double

def test_exp_cw_within_two_ulp_of_exact():
    rng = np.random.default_rng(0)
    x = np.concatenate([np.linspace(-86.9, 88.0, 400001), rng.uniform(-30, 0, 200000),
                        -np.logspace(-8, 1.9, 5000), [0.0, -0.0, 1.0, -1.0]]).astype(np.float32)
    y = O.exp_f(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    ulp = np.spacing(ref.astype(np.float32)).astype(np.float64)
    err = np.abs(y - ref) / ulp
    assert err.max() <= 2.0, err.max()
    assert O.exp_f(np.array([0.0], np.float32))[0] == 1.0
    # underflow region maps to zero, as the rasteriser's thresholds assume
    assert O.exp_f(np.array([-87.5, -100.0, -1e30], np.float32)).tolist() == [0.0, 0.0, 0.0]


# ------------------------------------------------------------------------------------------------
# SH basis: orthonormal on the sphere, and equal to scipy's complex SH turned real

def _quadrature(n_t=24, n_p=48):
    ct, wt = np.polynomial.legendre.leggauss(n_t)
    ph = (np.arange(n_p) + 0.5) * 2 * np.pi / n_p
    CT, PH = np.meshgrid(ct, ph, indexing="ij")
    ST = np.sqrt(1 - CT ** 2)
    dirs = np.stack([ST * np.cos(PH), ST * np.sin(PH), CT], -1).reshape(-1, 3)
    w = (wt[:, None] * np.full(n_p, 2 * np.pi / n_p)[None, :]).reshape(-1)
    return dirs, w


def test_sh_basis_orthonormal():
    dirs, w = _quadrature()
    B = O.sh_basis(3, dirs)
    gram = (B * w[:, None]).T @ B
    np.testing.assert_allclose(gram, np.eye(16), atol=1e-12)


def test_sh_basis_matches_scipy_and_closed_forms():
    rng = np.random.default_rng(1)
    d = rng.standard_normal((500, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    B = O.sh_basis(3, d)
    theta = np.arccos(np.clip(d[:, 2], -1, 1))
    phi = np.arctan2(d[:, 1], d[:, 0])
    for l in range(4):
        for m in range(-l, l + 1):
            Yc = special.sph_harm_y(l, abs(m), theta, phi)  # includes the Condon-Shortley phase
            if m == 0:
                ref = Yc.real
            elif m > 0:
                ref = math.sqrt(2) * Yc.real
            else:
                ref = math.sqrt(2) * Yc.imag
            np.testing.assert_allclose(B[:, l * l + l + m], ref, atol=1e-12)
    c1 = math.sqrt(3 / (4 * math.pi))
    np.testing.assert_allclose(B[:, 0], 0.5 / math.sqrt(math.pi), atol=1e-15)
    np.testing.assert_allclose(B[:, 1:4], c1 * np.stack([-d[:, 1], d[:, 2], -d[:, 0]], 1),
                               atol=1e-14)


# ------------------------------------------------------------------------------------------------
# eigenvalues against numpy

def test_eig3_matches_eigvalsh():
    rng = np.random.default_rng(2)
    mats = []
    for _ in range(300):
        M = rng.standard_normal((3, 3))
        mats.append(M @ M.T + 1.0 * np.eye(3))
    # near-degenerate and rank-2-plus-lambda cases like A = lambda I + sum gamma J^T J
    for _ in range(100):
        J = rng.standard_normal((2, 3)) * 40
        mats.append(np.eye(3) + J.T @ J)
    mats.append(np.eye(3) * 2.5)
    mats.append(np.diag([3.0, 3.0, 1.0]))
    A = np.stack(mats)
    ev = O.eig3(A)
    ref = np.linalg.eigvalsh(A)[:, ::-1]
    np.testing.assert_allclose(ev, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


# ------------------------------------------------------------------------------------------------
# projection

def _one(means, log_scales, quats, opac, sh, viewmats, intrin, H, W, deg=0):
    sc = scenes.Scene(name="one", means=np.asarray(means, np.float32),
                      log_scales=np.asarray(log_scales, np.float32),
                      quats=np.asarray(quats, np.float32), opac=np.asarray(opac, np.float32),
                      sh=np.asarray(sh, np.float32), sh_degree=deg,
                      viewmats=np.asarray(viewmats, np.float32),
                      intrin=np.asarray(intrin, np.float32), H=H, W=W,
                      bg=np.zeros(3, np.float32))
    return sc


def test_projection_on_axis_golden():
    """Closed form (hand-derived values stored in tests/golden/on_axis_gaussian.json)."""
    g = json.load(open(os.path.join(GOLDEN, "on_axis_gaussian.json")))
    i = g["input"]
    s = math.log(i["scale"])
    sc = _one([[0, 0, i["z"]]], [[s, s, s]], [[1, 0, 0, 0]], [i["opacity_logit"]],
              np.zeros((1, 1, 3)), np.eye(4)[None], [[i["fx"], i["fx"], i["cx"], i["cy"]]],
              i["H"], i["W"])
    p = O.project(sc, "d")
    rec = p["rec"][0, 0]
    e = g["expected"]
    assert p["valid"][0, 0] == 1
    np.testing.assert_allclose([rec[O.F["mx"]], rec[O.F["my"]]], e["mu2d"], atol=1e-12)
    # the inputs are fp32 (log-scale rounded), hence 1e-6 rather than double precision
    np.testing.assert_allclose([rec[O.F["qa"]], rec[O.F["qb"]], rec[O.F["qc"]]], e["conic"],
                               rtol=1e-6, atol=1e-15)
    np.testing.assert_allclose(rec[O.F["opac"]], e["opacity"], rtol=1e-12)
    assert p["rect"][0, 0].tolist() == e["tile_rect"]
    # the fp32 mode agrees with the closed form to fp32 precision and on the integer rectangle
    pf = O.project(sc, "f")
    assert pf["rect"][0, 0].tolist() == e["tile_rect"]
    np.testing.assert_allclose(pf["rec"][0, 0, 2:5], e["conic"], rtol=1e-6)


def _project_ref(mean, log_scale, quat, vm, K):
    """EWA covariance from first principles: Sigma3D from scipy's rotation, the projection
    Jacobian by central differences of the pinhole map."""
    R = vm[:3, :3].astype(np.float64)
    t = vm[:3, 3].astype(np.float64)
    xc = R @ mean + t
    q = np.asarray(quat, np.float64)
    Rq = Rotation.from_quat([q[1], q[2], q[3], q[0]]).as_matrix()
    S = np.diag(np.exp(log_scale))
    Sig = R @ (Rq @ S @ S @ Rq.T) @ R.T
    fx, fy, cx, cy = K

    def pi(x):
        return np.array([fx * x[0] / x[2] + cx, fy * x[1] / x[2] + cy])
    h = 1e-6 * np.abs(xc).max()
    J = np.stack([(pi(xc + h * e) - pi(xc - h * e)) / (2 * h) for e in np.eye(3)], 1)
    return pi(xc), J @ Sig @ J.T + 0.3 * np.eye(2), xc


def test_projection_matches_linearised_pinhole():
    sc = scenes.tiny_scene(5, 40, 64, 96, V=3, deg=0)
    p = O.project(sc, "d")
    n = 0
    for v in range(sc.V):
        for g in range(sc.G):
            if not p["valid"][v, g]:
                continue
            mu, Sig2, xc = _project_ref(sc.means[g].astype(np.float64),
                                        sc.log_scales[g].astype(np.float64), sc.quats[g],
                                        sc.viewmats[v], sc.intrin[v].astype(np.float64))
            fx, fy = sc.intrin[v, :2]
            if abs(xc[0] / xc[2]) > 1.3 * 0.5 * sc.W / fx or abs(xc[1] / xc[2]) > 1.3 * 0.5 * sc.H / fy:
                continue  # tangent clamp active: covariance Jacobian deliberately differs
            rec = p["rec"][v, g]
            Q = np.array([[rec[2], rec[3]], [rec[3], rec[4]]])
            np.testing.assert_allclose(np.linalg.inv(Q), Sig2, rtol=1e-7)
            np.testing.assert_allclose(rec[:2], mu, rtol=1e-12, atol=1e-9)
            np.testing.assert_allclose(rec[10:13], xc, rtol=1e-12, atol=1e-12)
            lam = np.linalg.eigvalsh(Sig2).max()
            r = math.ceil(3 * math.sqrt(lam))
            x0 = min(max(math.floor((mu[0] - r) / 16), 0), (sc.W + 15) // 16)
            x1 = min(max(math.floor((mu[0] + r) / 16) + 1, 0), (sc.W + 15) // 16)
            assert p["rect"][v, g, 0] == x0 and p["rect"][v, g, 2] == x1
            n += 1
    assert n > 60


def test_culling_rules():
    vm = np.eye(4)[None]
    K = [[64.0, 64.0, 32.0, 32.0]]
    means = [[0, 0, 2.0], [0, 0, -1.0], [0, 0, 0.005], [np.nan, 0, 2], [0, 0, 2.0], [500.0, 0, 2]]
    quats = [[1, 0, 0, 0], [1, 0, 0, 0], [1, 0, 0, 0], [1, 0, 0, 0], [0, 0, 0, 0], [1, 0, 0, 0]]
    sc = _one(means, np.full((6, 3), math.log(0.05)), quats, np.zeros(6), np.zeros((6, 1, 3)),
              vm, K, 64, 64)
    for mode in "fd":
        assert O.project(sc, mode)["valid"][0].tolist() == [1, 0, 0, 0, 0, 0]


# ------------------------------------------------------------------------------------------------
# render closed forms and invariants

def _single(bg, opac_logit=1.5, colour=(0.9, 0.4, 0.1)):
    Y00 = 0.5 / math.sqrt(math.pi)
    sh = ((np.asarray(colour) - 0.5) / Y00).reshape(1, 1, 3)
    sc = _one([[0.05, -0.03, 2.0]], [[math.log(0.06), math.log(0.03), math.log(0.04)]],
              [[0.9, 0.1, -0.2, 0.3]], [opac_logit], sh, np.eye(4)[None],
              [[64.0, 64.0, 32.0, 32.0]], 64, 64)
    sc.bg = np.asarray(bg, np.float32)
    return sc


def test_single_gaussian_composite_closed_form():
    """One Gaussian: C_hat = alpha c + (1 - alpha) bg, T = 1 - alpha, and the suffix behind it is
    the background, so C+ = bg and the opacity score sum is T alpha <r, c - bg>."""
    bg = np.array([0.2, 0.5, 0.7], np.float32).astype(np.float64)  # the inputs are fp32
    sc = _single(bg)
    p = O.project(sc, "d")
    L = O.bin_lists(p, 64, 64)
    r = O.render(p, L, 64, 64, bg, "d")
    rec = p["rec"][0, 0]
    jj, ii = np.meshgrid(np.arange(64) + 0.5, np.arange(64) + 0.5, indexing="ij")
    dx, dy = ii - rec[0], jj - rec[1]
    G = np.exp(-0.5 * (rec[2] * dx * dx + 2 * rec[3] * dx * dy + rec[4] * dy * dy))
    alpha = np.minimum(0.99, rec[6] * G)
    x0, y0, x1, y1 = p["rect"][0, 0]
    inside = np.zeros((64, 64), bool)
    inside[y0 * 16:y1 * 16, x0 * 16:x1 * 16] = True
    alpha = np.where(inside & (alpha >= 1 / 255), alpha, 0.0)
    c = rec[7:10]
    np.testing.assert_allclose(r["img"][0], alpha[..., None] * c + (1 - alpha[..., None]) * bg,
                               atol=1e-14)
    np.testing.assert_allclose(r["T"][0], 1 - alpha, atol=1e-14)
    assert (r["n_contrib"][0] == (alpha > 0)).all()
    # suffix recovery returns the background
    jv, iv = np.nonzero(alpha > 0.05)
    for j, i in list(zip(jv, iv))[::37]:
        tr = O.trace(p, L, 64, 64, bg, 0, i, j, "d")
        assert tr.shape[0] == 1
        np.testing.assert_allclose(tr[0, 6:9], bg, atol=1e-12)
    obs = np.random.default_rng(3).uniform(0, 1, (1, 64, 64, 3)).astype(np.float32)
    acc = O.replay(p, L, r, obs, 0, 64, 64, "d")["acc"][0, 0]
    res = r["img"][0] - obs[0]
    rho = (res * (c - bg)).sum(-1)
    # 1e-9: the suffix denominator carries the +1e-12 of the recovery equation
    np.testing.assert_allclose(acc[4], (alpha * rho).sum(), rtol=1e-9)
    np.testing.assert_allclose(acc[0], alpha.sum(), rtol=1e-12)


@pytest.mark.parametrize("mode,tol", [("d", 1e-12), ("f", 2e-6)])
def test_weights_plus_final_transmittance_is_one(mode, tol):
    """sum_k T_k alpha_k + T_final = 1 at every pixel (telescoping of T_{k+1} = T_k (1 - alpha_k)),
    checked over whole views through the accumulated supports."""
    sc = scenes.make(2)
    obs = np.zeros((sc.V, sc.H, sc.W, 3), np.float32)
    out = O.run(sc, obs, mode)
    for v in range(sc.V):
        total_w = out["acc"][v, :, 0].sum()
        npx = sc.H * sc.W
        assert abs(total_w + out["T"][v].sum() - npx) <= tol * npx
    # and per pixel along a few traces
    for (v, i, j) in [(0, 10, 20), (1, 64, 64), (3, 100, 5), (2, 127, 127)]:
        tr = O.trace(out["proj"], out["lists"], sc.H, sc.W, sc.bg, v, i, j, mode)
        w = tr[:, 1] * tr[:, 2]
        assert abs(w.sum() + out["T"][v, j, i] - 1.0) <= 10 * tol


def _brute_force_render(sc, proj):
    """Per pixel: every visible Gaussian whose tile rectangle contains the pixel's tile, in one
    global (depth, index) order with no per-tile lists, composited front to back in double."""
    V, G = proj["valid"].shape
    rec, rect = proj["rec"], proj["rect"]
    img = np.zeros((V, sc.H, sc.W, 3))
    T = np.ones((V, sc.H, sc.W))
    nc = np.zeros((V, sc.H, sc.W), np.int64)
    for v in range(V):
        vis = np.nonzero(proj["valid"][v])[0]
        order = vis[np.lexsort((vis, rec[v, vis, 5]))]
        for j in range(sc.H):
            for i in range(sc.W):
                tx, ty = i // 16, j // 16
                px, py = i + 0.5, j + 0.5
                Tp, C, n = 1.0, np.zeros(3), 0
                for g in order:
                    x0, y0, x1, y1 = rect[v, g]
                    if not (x0 <= tx < x1 and y0 <= ty < y1):
                        continue
                    r_ = rec[v, g]
                    dx, dy = px - r_[0], py - r_[1]
                    pw = -0.5 * (r_[2] * dx * dx + r_[4] * dy * dy) - r_[3] * dx * dy
                    if pw > 0:
                        continue
                    a = min(0.99, r_[6] * math.exp(pw))
                    if a < 1 / 255:
                        continue
                    Tn = Tp * (1 - a)
                    if Tn < 1e-4:
                        break
                    C = C + a * Tp * r_[7:10]
                    Tp = Tn
                    n += 1
                img[v, j, i] = C + Tp * sc.bg
                T[v, j, i] = Tp
                nc[v, j, i] = n
    return img, T, nc


@pytest.mark.parametrize("which", ["two_plane", "tiny"])
def test_tiled_lists_equal_brute_force_global_sort(which):
    """Binning + per-tile order equals a global per-pixel sort without tiles. The two-plane
    scene has exact depth ties (all Gaussians of a plane share z), exercising the index tie-break."""
    if which == "two_plane":
        sc = scenes.make(1)
    else:
        sc = scenes.tiny_scene(11, 60, 40, 56, V=2, deg=1)
    p = O.project(sc, "d")
    L = O.bin_lists(p, sc.H, sc.W)
    r = O.render(p, L, sc.H, sc.W, sc.bg, "d")
    img, T, nc = _brute_force_render(sc, p)
    np.testing.assert_allclose(r["img"], img, atol=1e-12)
    np.testing.assert_allclose(r["T"], T, atol=1e-12)
    assert (r["n_contrib"] == nc).all()


def test_tile_rectangles_cut_only_beyond_three_sigma():
    """The tile rectangle of a Gaussian covers its 3-sigma footprint (radius ceil(3 sqrt(lambda_max)),
    rounded out to whole tiles), so a pixel outside it lies more than 3 sigma out along an axis and
    its exponent is below -4.5 -- but alpha = o G can still reach 1/255 there (G >= e^-4.5 = 0.011).
    Against a render of the same records with no rectangle test: the tiled render differs only at
    pixels where some Gaussian outside its rectangle would have composited, every such Gaussian's
    exponent is below -4.5 (a smaller radius or a rectangle off by a tile breaks this), and on this
    scene of large, nearly opaque Gaussians some pixels do differ (the truncation the rasteriser's
    rule implies)."""
    sc = scenes.tiny_scene(3, 40, 64, 64, V=1, deg=0, log_scale_mean=math.log(0.3),
                           opac_mean=3.0, opac_sigma=0.5)
    p = O.project(sc, "d")
    tiled = O.render(p, O.bin_lists(p, sc.H, sc.W), sc.H, sc.W, sc.bg, "d")
    rec, rect, valid = p["rec"][0], p["rect"][0], p["valid"][0]
    ids = np.nonzero(valid)[0]
    order = ids[np.lexsort((ids, rec[ids, 5]))]
    r, rr = rec[order], rect[order]
    n_diff = 0
    for j in range(sc.H):
        for i in range(sc.W):
            dx, dy = i + 0.5 - r[:, 0], j + 0.5 - r[:, 1]
            pw = -0.5 * (r[:, 2] * dx * dx + r[:, 4] * dy * dy) - r[:, 3] * dx * dy
            a = np.minimum(0.99, r[:, 6] * np.exp(np.minimum(pw, 0.0)))
            ok = (pw <= 0) & (a >= 1 / 255)
            tx, ty = i // 16, j // 16
            inside = (rr[:, 0] <= tx) & (tx < rr[:, 2]) & (rr[:, 1] <= ty) & (ty < rr[:, 3])
            Tp, C = 1.0, np.zeros(3)
            for k in np.nonzero(ok)[0]:  # every valid Gaussian, no rectangle test
                Tn = Tp * (1 - a[k])
                if Tn < 1e-4:
                    break
                C = C + a[k] * Tp * r[k, 7:10]
                Tp = Tn
            C = C + Tp * sc.bg
            cut = ok & ~inside
            assert (pw[cut] < -4.5).all(), (i, j, pw[cut].max())
            # the same entries give the same sums up to the order of the products (1e-12)
            same = (np.abs(C - tiled["img"][0, j, i]).max() <= 1e-12
                    and abs(Tp - tiled["T"][0, j, i]) <= 1e-12)
            if not same:
                assert cut.any(), (i, j)
                n_diff += 1
    assert n_diff > 0


@pytest.mark.parametrize("mode", ["d", "f"])
def test_suffix_recovery_equals_back_to_front_composite(mode):
    """C+_k from the recovery equation equals the directly composited suffix
    (sum_{j>k} T_j alpha_j c_j + T_final bg) / (T_k (1 - alpha_k))."""
    sc = scenes.make(2)
    sc.bg = np.array([0.1, 0.3, 0.2], np.float32)
    p = O.project(sc, mode)
    L = O.bin_lists(p, sc.H, sc.W)
    rng = np.random.default_rng(4)
    worst = 0.0
    checked = 0
    for _ in range(60):
        v, i, j = int(rng.integers(sc.V)), int(rng.integers(sc.W)), int(rng.integers(sc.H))
        tr = O.trace(p, L, sc.H, sc.W, sc.bg, v, i, j, mode)
        n = tr.shape[0]
        if n == 0:
            continue
        a, T, c, Cp = tr[:, 1], tr[:, 2], tr[:, 3:6], tr[:, 6:9]
        Tfin = T[-1] * (1 - a[-1])
        for k in range(n):
            suffix = (T[k + 1:, None] * a[k + 1:, None] * c[k + 1:]).sum(0) + Tfin * sc.bg
            direct = suffix / (T[k] * (1 - a[k]))
            err = np.abs(Cp[k] - direct).max() / max(1.0, np.abs(direct).max())
            worst = max(worst, err)
            checked += 1
    assert checked > 200
    assert worst <= (1e-10 if mode == "d" else 1e-3), worst


# ------------------------------------------------------------------------------------------------
# finite differences: the unmasked, unnormalised scores are the gradient of L = 1/2 sum |r|^2

def _fd_scene(seed):
    sc = scenes.tiny_scene(seed, 4, 24, 32, V=2, deg=1, opac_mean=0.0, opac_sigma=0.5,
                           log_scale_mean=math.log(0.06))
    return sc


def _loss(sc, rec, L, obs, proj_valid):
    p = dict(valid=proj_valid, rec=rec)
    r = O.render(p, L, sc.H, sc.W, sc.bg, "d")
    return 0.5 * ((r["img"] - obs) ** 2).sum(), r


@pytest.mark.parametrize("seed", [21, 22, 23])
def test_scores_equal_central_finite_differences(seed):
    sc = _fd_scene(seed)
    p = O.project(sc, "d")
    assert p["valid"].all()
    L = O.bin_lists(p, sc.H, sc.W)
    obs = np.random.default_rng(seed).uniform(0.2, 0.8, (sc.V, sc.H, sc.W, 3)).astype(np.float32)
    r = O.render(p, L, sc.H, sc.W, sc.bg, "d")
    assert r["n_contrib"].max() <= sc.G and (r["T"] > 1e-3).all()  # no early stop
    acc = O.replay(p, L, r, obs, sc.sh_degree, sc.H, sc.W, "d")["acc"]
    rec = p["rec"]
    assert (rec[..., 6] * 1.0 < 0.99).all()  # no alpha clamp: masks are all ones
    assert (rec[..., 13] == 7).all()         # no colour clamp
    h = 1e-5

    def L_of_scene(s2):
        p2 = O.project(s2, "d")
        assert (p2["rect"] == p["rect"]).all()
        return _loss(sc, p2["rec"], L, obs, p2["valid"])[0]

    def rel(a, b):
        return np.abs(np.asarray(a) - np.asarray(b)).max() / np.abs(b).max()

    # opacity logit: sum_v (1 - o) Sa
    fd, an = [], []
    for g in range(sc.G):
        s_p, s_m = _copy(sc), _copy(sc)
        s_p.opac[g] += h
        s_m.opac[g] -= h
        # the inputs are fp32: divide by the perturbation actually stored
        fd.append((L_of_scene(s_p) - L_of_scene(s_m))
                  / (float(s_p.opac[g]) - float(s_m.opac[g])))
        an.append(sum((1 - rec[v, g, 6]) * acc[v, g, 4] for v in range(sc.V)))
    assert rel(an, fd) < 1e-6, (an, fd)

    # SH coefficients: sum_v M_color Swr_ch B_k
    B = p["B"]
    fd, an = [], []
    for g in range(sc.G):
        for k in range(sc.d):
            for ch in range(3):
                s_p, s_m = _copy(sc), _copy(sc)
                s_p.sh[g, k, ch] += h
                s_m.sh[g, k, ch] -= h
                fd.append((L_of_scene(s_p) - L_of_scene(s_m))
                          / (float(s_p.sh[g, k, ch]) - float(s_m.sh[g, k, ch])))
                an.append(sum(acc[v, g, 1 + ch] * B[v, g, k] for v in range(sc.V)))
    assert rel(an, fd) < 1e-6

    # projected centre (conic, colour, order held fixed): Sigma2D^{-1} Sd per view
    fd, an = [], []
    for v in range(sc.V):
        for g in range(sc.G):
            for ax in range(2):
                rp, rm = rec.copy(), rec.copy()
                rp[v, g, ax] += h
                rm[v, g, ax] -= h
                fd.append((_loss(sc, rp, L, obs, p["valid"])[0]
                           - _loss(sc, rm, L, obs, p["valid"])[0]) / (2 * h))
                Q = np.array([[rec[v, g, 2], rec[v, g, 3]], [rec[v, g, 3], rec[v, g, 4]]])
                an.append((Q @ acc[v, g, 5:7])[ax])
    assert rel(an, fd) < 1e-6

    # 3-D mean through the projected centres only: sum_v J_gv^T Sigma^{-1} Sd = b_mu * q_g
    tokens = O.finalize(p, acc, sc, lam=1.0)
    qg = 1e-6 + sum(1e-6 + acc[v, :, 0] for v in range(sc.V))
    fd, an = [], []
    for g in range(sc.G):
        for ax in range(3):
            ls, xs = [], []
            for sgn in (1, -1):
                s2 = _copy(sc)
                s2.means[g, ax] += sgn * h
                xs.append(float(s2.means[g, ax]))
                p2 = O.project(s2, "d")
                rr = rec.copy()
                rr[:, g, 0:2] = p2["rec"][:, g, 0:2]
                ls.append(_loss(sc, rr, L, obs, p["valid"])[0])
            fd.append((ls[0] - ls[1]) / (xs[0] - xs[1]))
            an.append(tokens[g, ax] * qg[g])
    assert rel(an, fd) < 2e-6, (an, fd)

    # the finalised appearance blocks are the same gradients divided by q_g
    for g in range(sc.G):
        ga = sum((1 - rec[v, g, 6]) * acc[v, g, 4] for v in range(sc.V))
        np.testing.assert_allclose(tokens[g, 3] * qg[g], ga, rtol=1e-10)



def test_score_masks_equal_central_differences_with_clamps_active():
    """The replay's masks against the derivative they stand for. "Exact Score Operators" defines
    M_alpha and M_color as the clamp-aware local VJP: where alpha = min(0.99, o G) sits at 0.99,
    or a colour channel at its zero clamp, the derivative through that path is zero. On a scene
    where both clamps are active (Gaussian 1 saturates at alpha = 0.99 on a few pixel centres,
    the red channel of Gaussian 2 is clamped in every view), central differences of
    L = 1/2 sum |C_hat - C_obs|^2 (no skip, stop or clamp decision flips within +-h) equal, per
    Gaussian: the opacity-logit score sum_v (1 - o) Sa, the finalised SH block times q_g
    (sum_v M_color Swr (x) B), the projected-centre score Sigma2D^{-1} Sd of every view, and the
    finalised mean block times q_g (3-D mean through the projected centres). The same scores equal
    the renderer backward's gradient for the opacity logit and the SH coefficients, and the scene
    is checked to be sensitive: the pixels the masks remove carry far more than the tolerance."""
    sc = scenes.clamp_scene()
    p = O.project(sc, "d")
    assert p["valid"].all()
    rec = p["rec"]
    assert (rec[:, 2, 13] == 6).all() and (rec[:, [0, 1, 3, 4, 5], 13] == 7).all()
    L = O.bin_lists(p, sc.H, sc.W)
    obs = np.random.default_rng(5).uniform(0.2, 0.8, (sc.V, sc.H, sc.W, 3)).astype(np.float32)
    r = O.render(p, L, sc.H, sc.W, sc.bg, "d")
    acc = O.replay(p, L, r, obs, sc.sh_degree, sc.H, sc.W, "d")["acc"]
    tokens = O.finalize(p, acc, sc, lam=1.0)
    qg = 1e-6 + sum(1e-6 + acc[v, :, 0] for v in range(sc.V))
    d = sc.d
    h = 1e-5
    tol = 1e-6

    # the alpha clamp is reached, and what the clamped pixels would add to Gaussian 1's opacity
    # and centre scores is far above the tolerance
    clamped_sa = np.zeros(sc.V)
    clamped_sd = np.zeros((sc.V, 2))
    n_clamped = 0
    for v in range(sc.V):
        for j in range(sc.H):
            for i in range(sc.W):
                tr = O.trace(p, L, sc.H, sc.W, sc.bg, v, i, j, "d")
                for row in tr[(tr[:, 0] == 1) & (tr[:, 1] >= 0.99)]:
                    assert row[1] == 0.99
                    rr = r["img"][v, j, i] - obs[v, j, i]
                    wrho = row[2] * row[1] * float(rr @ (row[3:6] - row[6:9]))
                    clamped_sa[v] += wrho
                    clamped_sd[v] += wrho * np.array([i + 0.5 - rec[v, 1, 0],
                                                      j + 0.5 - rec[v, 1, 1]])
                    n_clamped += 1
    assert n_clamped >= 4

    def rel(a, b):
        a, b = np.asarray(a, float), np.asarray(b, float)
        return np.abs(a - b).max() / max(np.abs(b).max(), 1e-12)

    def L_of_scene(s2):
        p2 = O.project(s2, "d")
        assert (p2["rect"] == p["rect"]).all()
        return _loss(sc, p2["rec"], L, obs, p2["valid"])[0]

    # opacity logit, per Gaussian: sum_v (1 - o) Sa
    sa = np.array([sum((1 - rec[v, g, 6]) * acc[v, g, 4] for v in range(sc.V))
                   for g in range(sc.G)])
    for g in range(sc.G):
        s_p, s_m = _copy(sc), _copy(sc)
        s_p.opac[g] += h
        s_m.opac[g] -= h
        fd = (L_of_scene(s_p) - L_of_scene(s_m)) / (float(s_p.opac[g]) - float(s_m.opac[g]))
        assert rel(sa[g], fd) < tol, (g, sa[g], fd)
        np.testing.assert_allclose(tokens[g, 3] * qg[g], sa[g], rtol=1e-10)
    without_mask = sa[1] + sum((1 - rec[v, 1, 6]) * clamped_sa[v] for v in range(sc.V))
    assert rel(without_mask, sa[1]) > 1e3 * tol

    # SH coefficients, per Gaussian: the finalised block times q_g = sum_v M_color Swr (x) B
    for g in range(sc.G):
        fd = np.zeros((d, 3))
        for k in range(d):
            for ch in range(3):
                s_p, s_m = _copy(sc), _copy(sc)
                s_p.sh[g, k, ch] += h
                s_m.sh[g, k, ch] -= h
                fd[k, ch] = ((L_of_scene(s_p) - L_of_scene(s_m))
                             / (float(s_p.sh[g, k, ch]) - float(s_m.sh[g, k, ch])))
        an = tokens[g, 4:4 + 3 * d].reshape(d, 3) * qg[g]
        assert rel(an, fd) < tol, (g, an, fd)
        if g == 2:
            assert (fd[:, 0] == 0).all() and (an[:, 0] == 0).all()  # clamped channel
            unmasked_red = sum(acc[v, 2, 1] * p["B"][v, 2, :d] for v in range(sc.V))
            assert np.abs(unmasked_red).max() > 1e3 * tol * np.abs(fd).max()

    # projected centre, per view and Gaussian: Sigma2D^{-1} Sd (a step of 1e-4 px: at 1e-5 the
    # rounding of L, ~1e-14, is 1e-6 of the smallest centre score here)
    hc = 1e-4
    for v in range(sc.V):
        for g in range(sc.G):
            fd = np.zeros(2)
            for ax in range(2):
                rp, rm = rec.copy(), rec.copy()
                rp[v, g, ax] += hc
                rm[v, g, ax] -= hc
                fd[ax] = (_loss(sc, rp, L, obs, p["valid"])[0]
                          - _loss(sc, rm, L, obs, p["valid"])[0]) / (2 * hc)
            Q = np.array([[rec[v, g, 2], rec[v, g, 3]], [rec[v, g, 3], rec[v, g, 4]]])
            an = Q @ acc[v, g, 5:7]
            assert rel(an, fd) < tol, (v, g, an, fd)
            if g == 1:
                assert rel(Q @ (acc[v, 1, 5:7] + clamped_sd[v]), an) > 1e3 * tol

    # 3-D mean through the projected centres: the finalised mean block times q_g
    for g in range(sc.G):
        fd = np.zeros(3)
        for ax in range(3):
            ls, xs = [], []
            for sgn in (1, -1):
                s2 = _copy(sc)
                s2.means[g, ax] += sgn * h
                xs.append(float(s2.means[g, ax]))
                p2 = O.project(s2, "d")
                rr = rec.copy()
                rr[:, g, 0:2] = p2["rec"][:, g, 0:2]
                ls.append(_loss(sc, rr, L, obs, p["valid"])[0])
            fd[ax] = (ls[0] - ls[1]) / (xs[0] - xs[1])
        assert rel(tokens[g, 0:3] * qg[g], fd) < 2 * tol, (g, tokens[g, 0:3] * qg[g], fd)

    # the renderer backward's raw gradient: the same opacity-logit and SH derivatives
    raw = O.run_backward(sc, obs, "d")["raw"]
    np.testing.assert_allclose(raw[:, 10], sa, rtol=1e-9, atol=1e-12 * np.abs(sa).max())
    sh_an = tokens[:, 4:4 + 3 * d] * qg[:, None]
    np.testing.assert_allclose(raw[:, 11:11 + 3 * d], sh_an, rtol=1e-9,
                               atol=1e-12 * np.abs(sh_an).max())


def _copy(sc):
    import dataclasses
    return dataclasses.replace(sc, means=sc.means.copy(), opac=sc.opac.copy(), sh=sc.sh.copy())


# ------------------------------------------------------------------------------------------------
# finalize: conditioning statistics with the Jacobian from finite differences

def test_conditioning_statistics_with_fd_jacobian():
    sc = scenes.tiny_scene(31, 6, 32, 32, V=3, deg=1)
    obs = np.random.default_rng(0).uniform(0, 1, (sc.V, sc.H, sc.W, 3)).astype(np.float32)
    out = O.run(sc, obs, "d", lam=0.7)
    acc, p = out["acc"], out["proj"]
    D = 9 + 3 * sc.d
    for g in range(sc.G):
        vis = [v for v in range(sc.V) if p["valid"][v, g]]
        q = np.array([1e-6 + acc[v, g, 0] for v in vis])
        qg = 1e-6 + q.sum()
        A = 0.7 * np.eye(3)
        for gam, v in zip(q / qg, vis):
            _, _, _ = None, None, None
            fx, fy, cx, cy = sc.intrin[v].astype(np.float64)
            R = sc.viewmats[v, :3, :3].astype(np.float64)
            t = sc.viewmats[v, :3, 3].astype(np.float64)

            def pi(m):
                x = R @ m + t
                return np.array([fx * x[0] / x[2] + cx, fy * x[1] / x[2] + cy])
            m0 = sc.means[g].astype(np.float64)
            hh = 1e-6
            J = np.stack([(pi(m0 + hh * e) - pi(m0 - hh * e)) / (2 * hh) for e in np.eye(3)], 1)
            A += gam * J.T @ J
        ev = np.linalg.eigvalsh(A)[::-1]
        tr = np.trace(A)
        z = out["tokens"][g]
        np.testing.assert_allclose(z[D - 4:D - 1], ev / (tr + 1e-6), rtol=1e-7, atol=1e-12)
        np.testing.assert_allclose(z[D - 1], math.log(tr + 1e-6), rtol=1e-8)
        np.testing.assert_allclose(z[D - 5], math.log(qg), rtol=1e-12)


def test_sh_score_factoring_equals_literal_per_pixel_sum():
    """M_color (sum_p w r) (x) B equals the printed per-pixel form sum_p M_color w [B (x) r]."""
    sc = scenes.make(2)
    obs = O.observe(sc, "f")
    for mode in "fd":
        out = O.run(sc, obs, mode, sh_literal=True)
        acc, B, rec = out["acc"], out["proj"]["B"][..., :sc.d], out["proj"]["rec"]
        cm = rec[..., 13].astype(int)
        mask = np.stack([(cm >> ch) & 1 for ch in range(3)], -1)  # [V, G, 3]
        fact = B[..., :, None] * (acc[..., None, 1:4] * mask[..., None, :])
        np.testing.assert_allclose(out["sh_literal"], fact, rtol=1e-9,
                                   atol=1e-12 * np.abs(fact).max())


def test_empty_and_degenerate_inputs():
    sc = scenes.tiny_scene(3, 5, 16, 16)
    sc.means[:, 2] = -1.0  # everything behind the camera
    obs = np.zeros((1, 16, 16, 3), np.float32)
    out = O.run(sc, obs, "f")
    assert out["lists"]["n"] == 0
    assert (out["img"] == 0).all() and (out["T"] == 1).all() and (out["n_contrib"] == 0).all()
    D = 9 + 3 * sc.d
    z = out["tokens"]
    assert np.isfinite(z).all()
    assert (z[:, :4 + 3 * sc.d] == 0).all()
    np.testing.assert_allclose(z[:, D - 5], math.log(1e-6))
    np.testing.assert_allclose(z[:, D - 4:D - 1], 1.0 / (3.0 + 1e-6))
