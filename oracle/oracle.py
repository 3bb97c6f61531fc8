"""ctypes binding of the CPU oracle (``splat_oracle.cpp``).

TEST INFRASTRUCTURE ONLY: imported by the tests, ``__graft_entry__.smoke()`` and the bench's
CPU-baseline leg. The product path (``gaussian_splatting_raster_b200``) never imports it.

``mode`` is ``"f"`` (fp32 working precision, the decisions taken exactly as an fp32
implementation takes them) or ``"d"`` (fp64 "truth").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "splat_oracle.cpp")
LIB = os.path.join(HERE, "libsplat_oracle.so")

TILE = 16
NF = 16        # fields per (view, Gaussian) record
NB = 16        # SH basis slots
ACC_N = 8      # q, Swr[3], Sa, Sd[2], composited pixel count
ACCB_N = 10    # backward sums: q, Swr[3], H, Hd[2], Hdd[3]
GRAD_BLOCKS = dict(mean=(0, 3), log_scale=(3, 6), quat=(6, 10), opacity=(10, 11))
F = dict(mx=0, my=1, qa=2, qb=3, qc=4, depth=5, opac=6, c0=7, c1=8, c2=9, xc=10, yc=11, zc=12,
         cmask=13, tiles=14)


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (fp-contract off, no fast math, OpenMP)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["g++", "-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-fPIC", "-shared", "-Wall", "-Wno-unknown-pragmas", SRC, "-o", LIB + ".tmp"]
        subprocess.check_call(cmd)
        os.replace(LIB + ".tmp", LIB)
    return LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        P = ctypes.c_void_p
        i32, i64, f32, f64 = ctypes.c_int, ctypes.c_longlong, ctypes.c_float, ctypes.c_double
        L.orc_exp_f.restype = f32
        L.orc_exp_f.argtypes = [f32]
        L.orc_exp_f_vec.argtypes = [P, P, i64]
        L.orc_sh_basis.argtypes = [i32, P, i64, P]
        L.orc_eig3.argtypes = [P, i64, P]
        L.orc_num_threads.restype = i32
        L.orc_set_threads.argtypes = [i32]
        for m in "fd":
            getattr(L, f"orc_project_{m}").argtypes = [P, P, P, P, P, i32, i32, P, P, i32, i32,
                                                       i32, P, P, P, P]
            getattr(L, f"orc_project_{m}").restype = i32
            getattr(L, f"orc_render_{m}").argtypes = [P, P, P, i32, i32, i32, i32, P, P, i32,
                                                      P, P, P, P]
            getattr(L, f"orc_render_{m}").restype = i64
            getattr(L, f"orc_replay_{m}").argtypes = [P, P, i32, P, P, i32, i32, i32, i32, P, P,
                                                      P, P, i32, P, P]
            getattr(L, f"orc_trace_{m}").argtypes = [P, P, P, i32, i32, i32, i32, P, i32, i32,
                                                     i32, i32, P]
            getattr(L, f"orc_trace_{m}").restype = i32
        L.orc_bin.argtypes = [P, P, P, i32, i32, i32, i32, P, P]
        L.orc_bin.restype = i64
        L.orc_finalize.argtypes = [P, P, P, P, P, P, i32, i32, i32, f64, P]
        L.orc_partials.argtypes = [P, P, P, P, P, P, P, i32, i32, i32, P]
        for m in "fd":
            getattr(L, f"orc_backward_{m}").argtypes = [P, P, P, i32, i32, i32, i32, P, P, P, P,
                                                        P, i32, P]
        L.orc_grad_finalize.argtypes = [P, P, P, P, P, P, P, P, P, i32, i32, i32, i32, i32, i32,
                                        P, P, P, P]
        L.orc_sh_poly_grad.argtypes = [i32, P, i64, P, P]
        for m in "fd":
            getattr(L, f"orc_render_features_{m}").argtypes = [P, P, P, i32, i32, i32, i32, P, P,
                                                               i32, P, i32, P]
            getattr(L, f"orc_scatter_{m}").argtypes = [P, P, P, i32, i32, i32, i32, P, P, i32, P,
                                                       i32, P]
        L.orc_finalize_partials.argtypes = [P, i32, i32, f64, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


def n_tiles(H: int, W: int) -> tuple[int, int]:
    return (W + TILE - 1) // TILE, (H + TILE - 1) // TILE


# ----------------------------------------------------------------------------------------------
# individual steps

def exp_f(x: np.ndarray) -> np.ndarray:
    x = _c(x, np.float32)
    y = np.empty_like(x)
    lib().orc_exp_f_vec(_p(x), _p(y), x.size)
    return y


def sh_basis(deg: int, dirs: np.ndarray) -> np.ndarray:
    dirs = _c(dirs, np.float64).reshape(-1, 3)
    out = np.zeros((dirs.shape[0], NB))
    lib().orc_sh_basis(deg, _p(dirs), dirs.shape[0], _p(out))
    return out[:, : (deg + 1) ** 2]


def eig3(A: np.ndarray) -> np.ndarray:
    A = _c(A, np.float64).reshape(-1, 9)
    ev = np.zeros((A.shape[0], 3))
    lib().orc_eig3(_p(A), A.shape[0], _p(ev))
    return ev


def project(scene, mode: str = "f") -> dict:
    G, V, H, W, deg = scene.G, scene.V, scene.H, scene.W, scene.sh_degree
    ins = [_c(scene.means, np.float32), _c(scene.log_scales, np.float32),
           _c(scene.quats, np.float32), _c(scene.opac, np.float32), _c(scene.sh, np.float32)]
    vm, K = _c(scene.viewmats, np.float32), _c(scene.intrin, np.float32)
    valid = np.zeros((V, G), np.int32)
    rec = np.zeros((V, G, NF))
    rect = np.zeros((V, G, 4), np.int32)
    B = np.zeros((V, G, NB))
    rc = getattr(lib(), f"orc_project_{mode}")(*[_p(a) for a in ins], G, deg, _p(vm), _p(K), V,
                                               H, W, _p(valid), _p(rec), _p(rect), _p(B))
    if rc != 0:
        raise ValueError("oracle projection rejected its arguments")
    return dict(valid=valid, rec=rec, rect=rect, B=B)


def bin_lists(proj: dict, H: int, W: int) -> dict:
    valid, rec, rect = proj["valid"], proj["rec"], proj["rect"]
    V, G = valid.shape
    TX, TY = n_tiles(H, W)
    off = np.zeros((V, TX * TY + 1), np.int64)
    n = lib().orc_bin(_p(valid), _p(rec), _p(rect), G, V, H, W, _p(off), None)
    ids = np.zeros(max(n, 1), np.int32)
    lib().orc_bin(_p(valid), _p(rec), _p(rect), G, V, H, W, _p(off), _p(ids))
    return dict(off=off, ids=ids[:n], n=int(n))


def _sel(sel, V, nt):
    if sel is None:
        return None, -1
    s = _c(np.asarray(sel).reshape(-1, 2), np.int32)
    return s, s.shape[0]


def render(proj, lists, H, W, bg, mode="f", sel=None) -> dict:
    V, G = proj["valid"].shape
    TX, TY = n_tiles(H, W)
    s, ns = _sel(sel, V, TX * TY)
    img = np.zeros((V, H, W, 3))
    Tf = np.zeros((V, H, W))
    nc = np.zeros((V, H, W), np.int32)
    last = np.zeros((V, H, W), np.int32)
    bg = _c(bg, np.float32)
    ids = lists["ids"] if lists["n"] > 0 else np.zeros(1, np.int32)
    ev = getattr(lib(), f"orc_render_{mode}")(
        _p(proj["rec"]), _p(lists["off"]), _p(ids), G, V, H, W, _p(bg),
        _p(s) if s is not None else None, ns, _p(img), _p(Tf), _p(nc), _p(last))
    return dict(img=img, T=Tf, n_contrib=nc, last=last, evaluated=int(ev))


def replay(proj, lists, rend, obs, deg, H, W, mode="f", sel=None, sh_literal=False) -> dict:
    V, G = proj["valid"].shape
    TX, TY = n_tiles(H, W)
    s, ns = _sel(sel, V, TX * TY)
    acc = np.zeros((V, G, ACC_N))
    shl = np.zeros((V, G, NB, 3)) if sh_literal else None
    obs = _c(obs, np.float32)
    ids = lists["ids"] if lists["n"] > 0 else np.zeros(1, np.int32)
    getattr(lib(), f"orc_replay_{mode}")(
        _p(proj["rec"]), _p(proj["B"]), deg, _p(lists["off"]), _p(ids), G, V, H, W,
        _p(_c(rend["img"], np.float64)), _p(obs), _p(_c(rend["last"], np.int32)),
        _p(s) if s is not None else None, ns, _p(acc), _p(shl) if shl is not None else None)
    out = dict(acc=acc)
    if sh_literal:
        out["sh_literal"] = shl[:, :, : (deg + 1) ** 2, :]
    return out


def finalize(proj, acc, scene, lam: float = 1.0) -> np.ndarray:
    V, G = proj["valid"].shape
    d = (scene.sh_degree + 1) ** 2
    tokens = np.zeros((G, 9 + 3 * d))
    lib().orc_finalize(_p(proj["valid"]), _p(proj["rec"]), _p(proj["B"]), _p(_c(acc, np.float64)),
                       _p(_c(scene.viewmats, np.float32)), _p(_c(scene.intrin, np.float32)),
                       G, V, scene.sh_degree, float(lam), _p(tokens))
    return tokens


def partials(proj, acc, scene, views=None) -> np.ndarray:
    """Per-Gaussian sums [G, 11 + 3d] over the views in `views` (all when None)."""
    V, G = proj["valid"].shape
    d = (scene.sh_degree + 1) ** 2
    out = np.zeros((G, 11 + 3 * d))
    use = None
    if views is not None:
        use = np.zeros(V, np.int32)
        use[list(views)] = 1
    lib().orc_partials(_p(proj["valid"]), _p(proj["rec"]), _p(proj["B"]), _p(_c(acc, np.float64)),
                       _p(_c(scene.viewmats, np.float32)), _p(_c(scene.intrin, np.float32)),
                       _p(use) if use is not None else None, G, V, scene.sh_degree, _p(out))
    return out


def finalize_partials(P, sh_degree: int, lam: float = 1.0) -> np.ndarray:
    """Tokens from summed partials."""
    P = _c(P, np.float64)
    G = P.shape[0]
    tokens = np.zeros((G, 9 + 3 * (sh_degree + 1) ** 2))
    lib().orc_finalize_partials(_p(P), G, sh_degree, float(lam), _p(tokens))
    return tokens


def sh_poly_grad(deg: int, dirs: np.ndarray):
    """SH basis [n, d] and its gradient [n, d, 3] by the polynomial form of the basis."""
    dirs = _c(dirs, np.float64).reshape(-1, 3)
    n = dirs.shape[0]
    B, dB = np.zeros((n, NB)), np.zeros((n, NB, 3))
    lib().orc_sh_poly_grad(deg, _p(dirs), n, _p(B), _p(dB))
    d = (deg + 1) ** 2
    return B[:, :d], dB[:, :d]


def backward(proj, lists, rend, obs, bg, H, W, mode="f", sel=None) -> np.ndarray:
    """Per-(view, Gaussian) sums of the renderer backward [V, G, 10]."""
    V, G = proj["valid"].shape
    TX, TY = n_tiles(H, W)
    s, ns = _sel(sel, V, TX * TY)
    accb = np.zeros((V, G, ACCB_N))
    ids = lists["ids"] if lists["n"] > 0 else np.zeros(1, np.int32)
    getattr(lib(), f"orc_backward_{mode}")(
        _p(proj["rec"]), _p(lists["off"]), _p(ids), G, V, H, W,
        _p(_c(rend["img"], np.float64)), _p(_c(obs, np.float32)), _p(_c(bg, np.float32)),
        _p(_c(rend["last"], np.int32)), _p(s) if s is not None else None, ns, _p(accb))
    return accb


def grad_dim(sh_degree: int) -> int:
    return 11 + 3 * (sh_degree + 1) ** 2


def gradients(proj, accb, scene, mode="f") -> dict:
    """raw / detached / support / pscale gradients [G, 11 + 3d] from the backward sums."""
    V, G = proj["valid"].shape
    K = grad_dim(scene.sh_degree)
    out = {k: np.zeros((G, K)) for k in ("raw", "detached", "support", "pscale")}
    lib().orc_grad_finalize(
        _p(proj["valid"]), _p(proj["rec"]), _p(_c(accb, np.float64)),
        _p(_c(scene.means, np.float32)), _p(_c(scene.log_scales, np.float32)),
        _p(_c(scene.quats, np.float32)), _p(_c(scene.sh, np.float32)),
        _p(_c(scene.viewmats, np.float32)), _p(_c(scene.intrin, np.float32)), G, V, scene.H,
        scene.W, scene.sh_degree, 1 if mode == "f" else 0, _p(out["raw"]), _p(out["detached"]),
        _p(out["support"]), _p(out["pscale"]))
    return out


def run_backward(scene, obs, mode: str = "f") -> dict:
    """Projection, binning, render and the renderer backward with its four gradient variants."""
    p = project(scene, mode)
    L = bin_lists(p, scene.H, scene.W)
    r = render(p, L, scene.H, scene.W, scene.bg, mode)
    accb = backward(p, L, r, obs, scene.bg, scene.H, scene.W, mode)
    return dict(proj=p, lists=L, **r, accb=accb, **gradients(p, accb, scene, mode))


def render_features(proj, lists, rend, feats, H, W, mode="f", sel=None) -> np.ndarray:
    """Per-Gaussian attributes [G, C] composited with the render's weights -> [V, H, W, C]."""
    V, G = proj["valid"].shape
    TX, TY = n_tiles(H, W)
    s, ns = _sel(sel, V, TX * TY)
    feats = _c(feats, np.float32).reshape(G, -1)
    C = feats.shape[1]
    out = np.zeros((V, H, W, C))
    ids = lists["ids"] if lists["n"] > 0 else np.zeros(1, np.int32)
    getattr(lib(), f"orc_render_features_{mode}")(
        _p(proj["rec"]), _p(lists["off"]), _p(ids), G, V, H, W, _p(_c(rend["last"], np.int32)),
        _p(feats) if G > 0 else None, C, _p(s) if s is not None else None, ns, _p(out))
    return out


def scatter(proj, lists, rend, pixel_map, H, W, mode="f", sel=None) -> np.ndarray:
    """Per-pixel map [V, H, W, C] scattered to the Gaussians with the render's weights -> [G, C]."""
    V, G = proj["valid"].shape
    TX, TY = n_tiles(H, W)
    s, ns = _sel(sel, V, TX * TY)
    m = _c(pixel_map, np.float32).reshape(V, H, W, -1)
    C = m.shape[3]
    out = np.zeros((G, C))
    ids = lists["ids"] if lists["n"] > 0 else np.zeros(1, np.int32)
    getattr(lib(), f"orc_scatter_{mode}")(
        _p(proj["rec"]), _p(lists["off"]), _p(ids), G, V, H, W, _p(_c(rend["last"], np.int32)),
        _p(m), C, _p(s) if s is not None else None, ns, _p(out))
    return out


def attribution(proj, lists, rend, obs, H, W, mode="f", sel=None) -> np.ndarray:
    """Scalar attribution per Gaussian [G, 3]: alphaT coverage sum w, PRIMU-style error
    sum w |r| (r = C_hat - C_obs), and the error per coverage sum w |r| / (sum w + 1e-6)."""
    r = np.asarray(rend["img"], np.float64) - np.asarray(obs, np.float64)
    rn = np.sqrt((r * r).sum(-1)).astype(np.float32)
    m = np.stack([np.ones_like(rn), rn], -1)
    s = scatter(proj, lists, rend, m, H, W, mode, sel)
    return np.concatenate([s, (s[:, 1] / (s[:, 0] + 1e-6))[:, None]], 1)


def trace(proj, lists, H, W, bg, v, i, j, mode="d", cap=4096) -> np.ndarray:
    V, G = proj["valid"].shape
    out = np.zeros((cap, 10))
    ids = lists["ids"] if lists["n"] > 0 else np.zeros(1, np.int32)
    n = getattr(lib(), f"orc_trace_{mode}")(_p(proj["rec"]), _p(lists["off"]), _p(ids), G, V, H,
                                           W, _p(_c(bg, np.float32)), v, i, j, cap, _p(out))
    return out[:n]


# ----------------------------------------------------------------------------------------------
# whole path

def observe(scene, mode: str = "f") -> np.ndarray:
    """Observation image: the render of the perturbed copy plus the scene's pixel noise."""
    sc = scene.observed_scene()
    p = project(sc, mode)
    L = bin_lists(p, sc.H, sc.W)
    r = render(p, L, sc.H, sc.W, sc.bg, mode)
    obs = r["img"].astype(np.float32)
    if scene.obs_noise_sigma > 0:
        obs = obs + scene.pixel_noise()
    return obs


def run(scene, obs, mode: str = "f", lam: float = 1.0, sel=None, sh_literal=False) -> dict:
    """Projection, binning, render, replay and (when sel is None) token finalisation."""
    p = project(scene, mode)
    L = bin_lists(p, scene.H, scene.W)
    r = render(p, L, scene.H, scene.W, scene.bg, mode, sel)
    rp = replay(p, L, r, obs, scene.sh_degree, scene.H, scene.W, mode, sel, sh_literal)
    out = dict(proj=p, lists=L, **r, **rp)
    out["tokens"] = finalize(p, rp["acc"], scene, lam)
    return out
