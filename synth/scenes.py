"""Seeded synthetic scenes for the render + score-replay path.

This module only draws random numbers and places cameras and Gaussians. It holds none of the
method's arithmetic (no projection, no colour evaluation, no compositing): both the CPU oracle and
the CUDA path consume what it returns, and neither is imported here.

Conventions shared by both consumers (the layout of the inputs, not a computation):

* ``means``      float32 [G, 3]  world-space centres.
* ``log_scales`` float32 [G, 3]  per-axis log standard deviations.
* ``quats``      float32 [G, 4]  rotation quaternion (w, x, y, z), not necessarily unit length.
* ``opac``       float32 [G]     opacity logits a (opacity = sigmoid(a)).
* ``sh``         float32 [G, d, 3] spherical-harmonic coefficients, d = (deg + 1)^2.
* ``viewmats``   float32 [V, 4, 4] world -> camera, row major; camera axes x right, y down,
  z forward (OpenCV).
* ``intrin``     float32 [V, 4]  (fx, fy, cx, cy) in pixels; pixel (i, j) covers [i, i + 1).

The recipes follow the workloads named for this path: a two-plane occlusion toy, a three-layer
occlusion diagnostic, pixel-aligned ReSplat/DepthSplat-scale scenes (one Gaussian per context
pixel, mu = o + d * r, from the ATSplat page's description of pixel-aligned feed-forward 3DGS) and
an ATSplat-style anchor scene (mu = p_i + delta_mu_ik with K = 16 offsets per anchor, same page).
They stand in for DL3DV, which is not available here.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# value of the degree-0 real spherical harmonic, used only to turn a drawn colour into the
# DC coefficient that produces it (the recipes specify colours, the inputs are coefficients)
_Y00 = 0.5 / math.sqrt(math.pi)


@dataclasses.dataclass
class Scene:
    name: str
    means: np.ndarray
    log_scales: np.ndarray
    quats: np.ndarray
    opac: np.ndarray
    sh: np.ndarray
    sh_degree: int
    viewmats: np.ndarray
    intrin: np.ndarray
    H: int
    W: int
    bg: np.ndarray
    # the perturbed copy whose render is the observation (same layout as above)
    obs_means: np.ndarray | None = None
    obs_sh: np.ndarray | None = None
    obs_noise_sigma: float = 0.0
    seed: int = 0

    @property
    def G(self) -> int:
        return int(self.means.shape[0])

    @property
    def V(self) -> int:
        return int(self.viewmats.shape[0])

    @property
    def d(self) -> int:
        return (self.sh_degree + 1) ** 2

    def observed_scene(self) -> "Scene":
        """The perturbed copy whose render (plus pixel noise) is the observed image."""
        return dataclasses.replace(self, means=self.obs_means, sh=self.obs_sh,
                                   obs_means=None, obs_sh=None)

    def pixel_noise(self) -> np.ndarray:
        """Seeded N(0, sigma) pixel noise [V, H, W, 3] added to the observation render."""
        rng = np.random.default_rng(self.seed + 7919)
        return (rng.standard_normal((self.V, self.H, self.W, 3), dtype=np.float32)
                * np.float32(self.obs_noise_sigma))


# ----------------------------------------------------------------------------------------------
# cameras

def _look_dir_rotation(forward: np.ndarray, down_hint=(0.0, 1.0, 0.0)) -> np.ndarray:
    """Rows = camera x (right), y (down), z (forward) axes in world coordinates."""
    f = np.asarray(forward, np.float64)
    f = f / np.linalg.norm(f)
    dn = np.asarray(down_hint, np.float64)
    right = np.cross(dn, f)
    right /= np.linalg.norm(right)
    down = np.cross(f, right)
    return np.stack([right, down, f])


def _viewmat(R: np.ndarray, centre: np.ndarray) -> np.ndarray:
    M = np.eye(4)
    M[:3, :3] = R
    M[:3, 3] = -R @ np.asarray(centre, np.float64)
    return M


def _axis_angle(axis: np.ndarray, angle: float) -> np.ndarray:
    a = axis / np.linalg.norm(axis)
    K = np.array([[0, -a[2], a[1]], [a[2], 0, -a[0]], [-a[1], a[0], 0]])
    return np.eye(3) + math.sin(angle) * K + (1 - math.cos(angle)) * (K @ K)


def _jitter(rng, viewmat: np.ndarray, deg: float = 1.0, trans: float = 0.02) -> np.ndarray:
    """Rotate the camera by `deg` degrees about a random axis and shift its centre by N(0, trans)."""
    R = viewmat[:3, :3]
    c = -R.T @ viewmat[:3, 3]
    Rj = _axis_angle(rng.standard_normal(3), math.radians(deg)) @ R
    cj = c + rng.normal(0.0, trans, 3)
    return _viewmat(Rj, cj)


def _random_quats(rng, n: int) -> np.ndarray:
    q = rng.standard_normal((n, 4))
    return q / np.linalg.norm(q, axis=1, keepdims=True)


def _sh_from_colour(rng, colour: np.ndarray, deg: int, hi_sigma: float) -> np.ndarray:
    n = colour.shape[0]
    d = (deg + 1) ** 2
    sh = np.empty((n, d, 3), np.float32)
    sh[:, 0, :] = (colour - 0.5) / _Y00
    if d > 1:
        sh[:, 1:, :] = rng.standard_normal((n, d - 1, 3), dtype=np.float32) * np.float32(hi_sigma)
    return sh


def _smooth_field(rng, H: int, W: int, n_waves: int = 8, max_cycles: float = 3.0) -> np.ndarray:
    """Sum of random low-frequency 2-D cosines (at most `max_cycles` cycles per image)."""
    yy, xx = np.meshgrid((np.arange(H) + 0.5) / H, (np.arange(W) + 0.5) / W, indexing="ij")
    f = np.zeros((H, W))
    for _ in range(n_waves):
        fx, fy = rng.uniform(-max_cycles, max_cycles, 2)
        ph = rng.uniform(0, 2 * math.pi)
        amp = rng.uniform(0.5, 1.0)
        f += amp * np.cos(2 * math.pi * (fx * xx + fy * yy) + ph)
    return f


def _f32(*arrs):
    return [np.ascontiguousarray(a, dtype=np.float32) for a in arrs]


def _finish(name, seed, means, log_scales, quats, opac, sh, deg, viewmats, intrin, H, W,
            rng, mean_sigma=0.01, colour_sigma=0.05, noise_sigma=0.0) -> Scene:
    G = means.shape[0]
    obs_means = means + rng.normal(0.0, mean_sigma, (G, 3))
    obs_sh = sh.copy()
    obs_sh[:, 0, :] += (rng.normal(0.0, colour_sigma, (G, 3)) / _Y00).astype(np.float32)
    means, log_scales, quats, opac, sh, obs_means, obs_sh = _f32(
        means, log_scales, quats, opac, sh, obs_means, obs_sh)
    viewmats, intrin = _f32(viewmats, intrin)
    return Scene(name=name, means=means, log_scales=log_scales, quats=quats, opac=opac, sh=sh,
                 sh_degree=deg, viewmats=viewmats, intrin=intrin, H=H, W=W,
                 bg=np.zeros(3, np.float32), obs_means=obs_means, obs_sh=obs_sh,
                 obs_noise_sigma=noise_sigma, seed=seed)


# ----------------------------------------------------------------------------------------------
# the five workloads

def two_plane(seed: int = 1001) -> Scene:
    """256 Gaussians on the planes z = 2 and z = 4, one 64x64 view at the origin looking +z."""
    rng = np.random.default_rng(seed)
    H = W = 64
    fx = fy = 64.0
    cx = cy = 32.0
    G = 256
    z = np.repeat([2.0, 4.0], G // 2)
    x = rng.uniform(-1, 1, G) * z * (W / 2) / fx
    y = rng.uniform(-1, 1, G) * z * (H / 2) / fy
    means = np.stack([x, y, z], 1)
    log_scales = rng.normal(math.log(0.05), 0.3, (G, 3))
    quats = _random_quats(rng, G)
    opac = rng.normal(0.0, 1.5, G)
    sh = _sh_from_colour(rng, rng.uniform(0, 1, (G, 3)), 0, 0.0)
    viewmats = np.eye(4)[None]
    intrin = np.array([[fx, fy, cx, cy]])
    return _finish("two_plane", seed, means, log_scales, quats, opac, sh, 0, viewmats, intrin,
                   H, W, rng)


def three_layer(seed: int = 1002) -> Scene:
    """4096 Gaussians in three depth layers, 4 views 128x128 on a 30 degree arc at radius 5."""
    rng = np.random.default_rng(seed)
    H = W = 128
    G = 4096
    layer = np.arange(G) % 3
    z = np.array([1.5, 2.5, 3.5])[layer] + rng.normal(0, 0.05, G)
    xy = rng.uniform(-2.5, 2.5, (G, 2))
    means = np.concatenate([xy, z[:, None]], 1)
    log_scales = rng.normal(math.log(0.04), 0.4, (G, 3))
    quats = _random_quats(rng, G)
    opac = rng.normal(0.5, 1.5, G)
    sh = _sh_from_colour(rng, rng.uniform(0, 1, (G, 3)), 1, 0.3)
    views = []
    for deg in (-15.0, -5.0, 5.0, 15.0):
        t = math.radians(deg)
        centre = np.array([5 * math.sin(t), 0.0, -5 * math.cos(t)])
        views.append(_viewmat(_look_dir_rotation(-centre), centre))
    viewmats = np.stack(views)
    intrin = np.tile([[128.0, 128.0, 64.0, 64.0]], (4, 1))
    return _finish("three_layer", seed, means, log_scales, quats, opac, sh, 1, viewmats, intrin,
                   H, W, rng, noise_sigma=0.01)


def _pixel_aligned(name, seed, n_ctx, n_tgt, H, W, deg, hi_sigma, noise_sigma) -> Scene:
    rng = np.random.default_rng(seed)
    fx = fy = 0.86 * W
    cx, cy = W / 2.0, H / 2.0
    ctx_x = np.linspace(-0.5, 0.5, n_ctx)
    shared = _smooth_field(rng, H, W)
    means, scales = [], []
    v_pix, u_pix = np.meshgrid(np.arange(H) + 0.5, np.arange(W) + 0.5, indexing="ij")
    for vi in range(n_ctx):
        f = shared + 0.1 * _smooth_field(rng, H, W)
        f = (f - f.min()) / (f.max() - f.min())
        depth = 1.0 / (0.01 + 0.99 * f)                       # inverse depth in [1/100, 1]
        centre = np.array([ctx_x[vi], 0.0, 0.0])
        ray = np.stack([(u_pix - cx) / fx, (v_pix - cy) / fy, np.ones_like(u_pix)], -1)
        mu = centre + depth[..., None] * ray                  # mu = o + d * r (camera R = I)
        means.append(mu.reshape(-1, 3))
        scales.append(np.repeat((0.8 * depth / fx).reshape(-1, 1), 3, 1))
    means = np.concatenate(means)
    G = means.shape[0]
    log_scales = np.log(np.concatenate(scales)) + rng.normal(0, 0.2, (G, 3))
    quats = _random_quats(rng, G)
    opac = rng.normal(1.0, 1.0, G)
    sh = _sh_from_colour(rng, rng.uniform(0, 1, (G, 3)), deg, hi_sigma)
    tgt_idx = np.round(np.linspace(0, n_ctx - 1, n_tgt)).astype(int)
    viewmats = np.stack([_jitter(rng, _viewmat(np.eye(3), [ctx_x[i], 0.0, 0.0]))
                         for i in tgt_idx])
    intrin = np.tile([[fx, fy, cx, cy]], (n_tgt, 1))
    return _finish(name, seed, means, log_scales, quats, opac, sh, deg, viewmats, intrin, H, W,
                   rng, noise_sigma=noise_sigma)


def resplat_pixel_aligned(seed: int = 1003) -> Scene:
    """8 context views 256x448 backprojected one Gaussian per pixel (917,504), SH degree 2,
    scored in 8 jittered target views."""
    return _pixel_aligned("resplat_256x448_8v", seed, 8, 8, 256, 448, 2, 0.1, 0.0)


def resplat_views(n_views: int, seed: int = 1003) -> Scene:
    """The ReSplat-scale layout with n_views context views backprojected (n_views x 114,688
    Gaussians) scored in the same number of target views: the view-count scaling workloads
    (4/8/16/32 views at 256x448)."""
    return _pixel_aligned(f"resplat_256x448_{n_views}v", seed, n_views, n_views, 256, 448, 2, 0.1,
                          0.0)


def atsplat_anchor(seed: int = 1004) -> Scene:
    """19,456 anchors x 16 offsets = 311,296 Gaussians, SH degree 2, 4 target views 512x960."""
    rng = np.random.default_rng(seed)
    H, W = 512, 960
    fx = fy = 0.86 * W
    cx, cy = W / 2.0, H / 2.0
    K = 16
    anchors = []
    for ax in (-0.3, 0.3):
        n = 9728
        u = rng.uniform(0, W, n)
        v = rng.uniform(0, H, n)
        depth = rng.uniform(1, 20, n)
        p = np.stack([ax + depth * (u - cx) / fx, depth * (v - cy) / fy, depth], 1)
        anchors.append((p, depth))
    p = np.concatenate([a[0] for a in anchors])
    depth = np.concatenate([a[1] for a in anchors])
    means = (p[:, None, :] + rng.standard_normal((p.shape[0], K, 3))
             * (0.05 * depth)[:, None, None]).reshape(-1, 3)
    dG = np.repeat(depth, K)
    G = means.shape[0]
    log_scales = np.log(0.01 * dG)[:, None] + rng.normal(0, 0.3, (G, 3))
    quats = _random_quats(rng, G)
    opac = rng.normal(0.0, 1.5, G)
    sh = _sh_from_colour(rng, rng.uniform(0, 1, (G, 3)), 2, 0.1)
    viewmats = np.stack([_jitter(rng, _viewmat(np.eye(3), [x, 0.0, 0.0]))
                         for x in np.linspace(-0.3, 0.3, 4)])
    intrin = np.tile([[fx, fy, cx, cy]], (4, 1))
    return _finish("atsplat_anchor_512x960", seed, means, log_scales, quats, opac, sh, 2,
                   viewmats, intrin, H, W, rng)


def depthsplat_dense(seed: int = 1005) -> Scene:
    """12 context views 512x960 pixel-aligned (5,898,240 Gaussians), SH degree 3, 4 jittered
    target views, observation noise N(0, 0.01)."""
    return _pixel_aligned("depthsplat_512x960_12v", seed, 12, 4, 512, 960, 3, 0.1, 0.01)


CONFIGS = {
    1: two_plane,
    2: three_layer,
    3: resplat_pixel_aligned,
    4: atsplat_anchor,
    5: depthsplat_dense,
}


def make(cfg: int) -> Scene:
    return CONFIGS[cfg](1000 + cfg)


# ----------------------------------------------------------------------------------------------
# small helpers for tests

def tiny_scene(seed: int, G: int, H: int, W: int, V: int = 1, deg: int = 1,
               depth_range=(2.0, 4.0), log_scale_mean=math.log(0.08), opac_mean=0.0,
               opac_sigma=1.0, colour_range=(0.2, 0.8), hi_sigma=0.05) -> Scene:
    """Few Gaussians in front of V cameras near the origin looking +z (for closed-form and
    finite-difference checks)."""
    rng = np.random.default_rng(seed)
    fx = fy = float(max(H, W))
    cx, cy = W / 2.0, H / 2.0
    z = rng.uniform(*depth_range, G)
    x = rng.uniform(-0.3, 0.3, G) * z * (W / 2) / fx
    y = rng.uniform(-0.3, 0.3, G) * z * (H / 2) / fy
    means = np.stack([x, y, z], 1)
    log_scales = log_scale_mean + rng.normal(0, 0.2, (G, 3))
    quats = _random_quats(rng, G)
    opac = rng.normal(opac_mean, opac_sigma, G)
    sh = _sh_from_colour(rng, rng.uniform(*colour_range, (G, 3)), deg, hi_sigma)
    views = []
    for vi in range(V):
        ang = math.radians(4.0 * (vi - (V - 1) / 2))
        centre = np.array([0.3 * (vi - (V - 1) / 2), 0.05 * vi, -0.1 * vi])
        views.append(_viewmat(_axis_angle(np.array([0.0, 1.0, 0.0]), ang), centre))
    viewmats = np.stack(views)
    intrin = np.tile([[fx, fy, cx, cy]], (V, 1))
    return _finish(f"tiny{seed}", seed, means, log_scales, quats, opac, sh, deg, viewmats, intrin,
                   H, W, rng)


def smooth_observation(seed: int, V: int, H: int, W: int) -> np.ndarray:
    """A smooth seeded colour field [V, H, W, 3] in [0, 1] used as the observed image where a
    render of the perturbed scene is too costly for the oracle (full-size sampled checks)."""
    rng = np.random.default_rng(seed)
    out = np.empty((V, H, W, 3), np.float32)
    for v in range(V):
        for c in range(3):
            f = _smooth_field(rng, H, W, n_waves=4)
            out[v, :, :, c] = 0.5 + 0.2 * f / 4.0
    return out


def clamp_scene(seed: int = 51, G: int = 6, H: int = 24, W: int = 32, V: int = 2) -> Scene:
    """A tiny scene in which the renderer's two clamps are active: Gaussian 1 is opaque (logit 7)
    and wide (about 8 px standard deviation in the images) at the back, so alpha = min(0.99, o G)
    saturates at 0.99 on the pixel centres within about 1 px of its projected centre; Gaussian 2
    has a DC red coefficient of -3, so its red channel is below zero before the colour clamp in
    every view. The other Gaussians are drawn as in ``tiny_scene``."""
    sc = tiny_scene(seed, G, H, W, V=V, deg=1, opac_mean=0.0, opac_sigma=0.5,
                    log_scale_mean=math.log(0.06))
    sc.means[1] = [0.02, -0.03, 3.8]
    sc.log_scales[1] = np.log([0.95, 0.9, 1.0])
    sc.opac[1] = 7.0
    sc.sh[2, 0, 0] = -3.0
    return sc
