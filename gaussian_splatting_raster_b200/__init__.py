"""B200-native tile-based Gaussian-splatting render + analytic score replay.

Thin ctypes binding of ``libsplat.so`` (C ABI in ``include/splat.h``). Every step of the path runs
in the library's CUDA kernels; this module only checks tensor arguments and passes device pointers
and the current CUDA stream. There is no CPU fallback: without the built library or a CUDA device
the calls raise.
"""
from __future__ import annotations

import ctypes
import os

from .build import LIB, LIB_CHECKED, build  # noqa: F401

__all__ = ["Workspace", "SplatError", "load_library", "LIB", "build", "token_dim",
           "partials_dim", "grad_dim", "finalize_partials"]

_ERRORS = {
    -1: "INVALID_ARG", -2: "CAPACITY", -3: "STATE", -4: "CUDA", -5: "BOUNDS",
    -6: "DEVICE_TIMEOUT", -7: "OOM",
}

# every symbol include/splat.h declares (checked against the header by the tests)
EXPORTS = [
    "splat_ws_create", "splat_ws_destroy", "splat_last_error", "splat_project",
    "splat_bin_sort", "splat_render", "splat_score_replay", "splat_render_score",
    "splat_copy_projection",
    "splat_copy_tile_lists", "splat_copy_last", "splat_copy_accumulators", "splat_pair_count",
    "splat_launch_count", "splat_profile_enable", "splat_profile_read", "splat_kernel_name",
    "splat_sort_depths_noalloc", "splat_score_partials", "splat_finalize_partials",
    "splat_backward", "splat_render_features", "splat_scatter", "splat_attribution",
    "splat_set_deterministic", "splat_check_status", "splat_checked_build",
]


KERNEL_GROUPS = 17  # SPLAT_NUM_KERNELS


class SplatError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"splat error {code} ({_ERRORS.get(code, '?')}): {msg}")
        self.code = code


_lib = None


def load_library(path: str | None = None):
    """Load libsplat.so (raises OSError when it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB
    if not os.path.exists(p):
        raise OSError(f"libsplat.so not built at {p}; run gaussian_splatting_raster_b200.build()")
    L = ctypes.CDLL(p)
    V, I, LL, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_float
    L.splat_ws_create.argtypes = [ctypes.POINTER(V), I, I, I, I, I]
    L.splat_ws_create.restype = I
    L.splat_ws_destroy.argtypes = [V]
    L.splat_ws_destroy.restype = None
    L.splat_last_error.argtypes = [V]
    L.splat_last_error.restype = ctypes.c_char_p
    L.splat_project.argtypes = [V, V, V, V, V, V, I, I, V, V, I, I, I, V]
    L.splat_project.restype = I
    L.splat_bin_sort.argtypes = [V, ctypes.POINTER(LL), V]
    L.splat_bin_sort.restype = I
    L.splat_render.argtypes = [V, V, V, V, V, V]
    L.splat_render.restype = I
    L.splat_score_replay.argtypes = [V, V, F, V, V]
    L.splat_score_replay.restype = I
    L.splat_render_score.argtypes = [V, V, V, F, V, V, V, V, V]
    L.splat_render_score.restype = I
    L.splat_copy_projection.argtypes = [V, V, V, V]
    L.splat_copy_projection.restype = I
    L.splat_copy_tile_lists.argtypes = [V, V, V, V]
    L.splat_copy_tile_lists.restype = I
    L.splat_copy_last.argtypes = [V, V, V]
    L.splat_copy_last.restype = I
    L.splat_copy_accumulators.argtypes = [V, V, V]
    L.splat_copy_accumulators.restype = I
    L.splat_pair_count.argtypes = [V, ctypes.POINTER(LL), V]
    L.splat_pair_count.restype = I
    L.splat_launch_count.argtypes = [V]
    L.splat_launch_count.restype = LL
    L.splat_profile_enable.argtypes = [V, I]
    L.splat_profile_enable.restype = I
    L.splat_profile_read.argtypes = [V, V, V, I]
    L.splat_profile_read.restype = I
    L.splat_kernel_name.argtypes = [I]
    L.splat_kernel_name.restype = ctypes.c_char_p
    L.splat_score_partials.argtypes = [V, V, V, V]
    L.splat_score_partials.restype = I
    L.splat_finalize_partials.argtypes = [V, I, I, F, V, V]
    L.splat_finalize_partials.restype = I
    L.splat_backward.argtypes = [V, V, V, V, V, V, V, V, V, V]
    L.splat_backward.restype = I
    L.splat_render_features.argtypes = [V, V, I, V, V]
    L.splat_render_features.restype = I
    L.splat_scatter.argtypes = [V, V, I, V, V]
    L.splat_scatter.restype = I
    L.splat_attribution.argtypes = [V, V, V, V]
    L.splat_attribution.restype = I
    L.splat_set_deterministic.argtypes = [V, I]
    L.splat_set_deterministic.restype = I
    L.splat_check_status.argtypes = [V, V]
    L.splat_check_status.restype = I
    L.splat_checked_build.argtypes = []
    L.splat_checked_build.restype = I
    if path is None:
        _lib = L
    return L


def token_dim(sh_degree: int) -> int:
    return 9 + 3 * (sh_degree + 1) ** 2


def partials_dim(sh_degree: int) -> int:
    return 11 + 3 * (sh_degree + 1) ** 2


def grad_dim(sh_degree: int) -> int:
    """Row width of the gradients: mean (3), log-scale (3), quaternion (4), opacity logit, SH."""
    return 11 + 3 * (sh_degree + 1) ** 2


def finalize_partials(partials, sh_degree: int, tokens, lam: float = 1.0, stream=None):
    """Tokens [n, 9 + 3d] from summed per-Gaussian partials [n, 11 + 3d] (any slice of rows)."""
    import torch
    n = partials.shape[0]
    rc = load_library().splat_finalize_partials(
        _ptr(partials, "partials", torch.float32, (n, partials_dim(sh_degree))), n, sh_degree,
        ctypes.c_float(lam), _ptr(tokens, "tokens", torch.float32, (n, token_dim(sh_degree))),
        _stream(stream))
    if rc != 0:
        raise SplatError(rc, "finalize from partials failed")


def _stream(stream):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t, name, dtype, shape=None):
    import torch
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return ctypes.c_void_p(t.data_ptr())


class Workspace:
    """Library-owned workspace (records, tile lists, accumulators) for problems up to the given
    maxima. Calls enqueue on the current torch CUDA stream unless one is passed."""

    def __init__(self, max_G: int, max_V: int, max_H: int, max_W: int, max_sh_degree: int = 3,
                 lib=None):
        """lib: a loaded library to use instead of the default one (e.g. the checked build,
        load_library(LIB_CHECKED))."""
        self._L = lib if lib is not None else load_library()
        h = ctypes.c_void_p()
        rc = self._L.splat_ws_create(ctypes.byref(h), max_G, max_V, max_H, max_W, max_sh_degree)
        if rc != 0:
            raise SplatError(rc, "workspace creation failed")
        self._h = h
        self.G = self.V = self.H = self.W = self.deg = 0

    def close(self):
        if getattr(self, "_h", None):
            self._L.splat_ws_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def _check(self, rc):
        if rc != 0:
            raise SplatError(rc, self._L.splat_last_error(self._h).decode())

    # -- the path -------------------------------------------------------------------------------
    def project(self, means, log_scales, quats, opac_logits, sh, viewmats, intrin, H, W,
                stream=None):
        import torch
        G = means.shape[0]
        V = viewmats.shape[0]
        d = sh.shape[1] if sh.dim() == 3 else 1
        deg = {1: 0, 4: 1, 9: 2, 16: 3}.get(d)
        if deg is None:
            raise ValueError("sh must be [G, (deg+1)^2, 3] with deg <= 3")
        f = torch.float32
        args = [_ptr(means, "means", f, (G, 3)), _ptr(log_scales, "log_scales", f, (G, 3)),
                _ptr(quats, "quats", f, (G, 4)), _ptr(opac_logits, "opac_logits", f, (G,)),
                _ptr(sh, "sh", f, (G, d, 3))]
        self._check(self._L.splat_project(
            self._h, *args, G, deg, _ptr(viewmats, "viewmats", f, (V, 4, 4)),
            _ptr(intrin, "intrin", f, (V, 4)), V, H, W, _stream(stream)))
        self.G, self.V, self.H, self.W, self.deg = G, V, H, W, deg

    def bin_sort(self, stream=None) -> list[int]:
        out = (ctypes.c_longlong * max(self.V, 1))()
        self._check(self._L.splat_bin_sort(self._h, out, _stream(stream)))
        return [int(out[i]) for i in range(self.V)]

    def render(self, bg, img, T_final, n_contrib, stream=None):
        import torch
        V, H, W = self.V, self.H, self.W
        self._check(self._L.splat_render(
            self._h, _ptr(bg, "bg", torch.float32, (3,)),
            _ptr(img, "img", torch.float32, (V, H, W, 3)),
            _ptr(T_final, "T_final", torch.float32, (V, H, W)),
            _ptr(n_contrib, "n_contrib", torch.int32, (V, H, W)), _stream(stream)))

    def score_replay(self, obs, tokens, lam: float = 1.0, stream=None):
        import torch
        V, H, W = self.V, self.H, self.W
        self._check(self._L.splat_score_replay(
            self._h, _ptr(obs, "obs", torch.float32, (V, H, W, 3)), ctypes.c_float(lam),
            _ptr(tokens, "tokens", torch.float32, (self.G, token_dim(self.deg))),
            _stream(stream)))

    def render_score(self, bg, obs, img, T_final, n_contrib, tokens, lam: float = 1.0,
                     stream=None):
        """render followed by score_replay in one call (one fused kernel in the default mode)."""
        import torch
        V, H, W = self.V, self.H, self.W
        self._check(self._L.splat_render_score(
            self._h, _ptr(bg, "bg", torch.float32, (3,)),
            _ptr(obs, "obs", torch.float32, (V, H, W, 3)), ctypes.c_float(lam),
            _ptr(img, "img", torch.float32, (V, H, W, 3)),
            _ptr(T_final, "T_final", torch.float32, (V, H, W)),
            _ptr(n_contrib, "n_contrib", torch.int32, (V, H, W)),
            _ptr(tokens, "tokens", torch.float32, (self.G, token_dim(self.deg))),
            _stream(stream)))

    def score_partials(self, obs, partials, stream=None):
        """Replay of this workspace's views; per-Gaussian sums [G, 11 + 3d] instead of tokens."""
        import torch
        V, H, W = self.V, self.H, self.W
        self._check(self._L.splat_score_partials(
            self._h, _ptr(obs, "obs", torch.float32, (V, H, W, 3)),
            _ptr(partials, "partials", torch.float32, (self.G, partials_dim(self.deg))),
            _stream(stream)))

    def backward(self, obs, log_scales, quats, sh, raw=None, detached=None, support=None,
                 pscale=None, stream=None):
        """Renderer backward of 1/2 sum |C_hat - C_obs|^2 after render: the requested gradient
        variants, each [G, 11 + 3d] fp32 (None skips a variant). log_scales, quats, sh are the
        arrays given to project."""
        import torch
        G, d, f = self.G, (self.deg + 1) ** 2, torch.float32
        K = grad_dim(self.deg)
        outs = [_ptr(t, n, f, (G, K)) for t, n in ((raw, "raw"), (detached, "detached"),
                                                    (support, "support"), (pscale, "pscale"))]
        self._check(self._L.splat_backward(
            self._h, _ptr(obs, "obs", f, (self.V, self.H, self.W, 3)),
            _ptr(log_scales, "log_scales", f, (G, 3)), _ptr(quats, "quats", f, (G, 4)),
            _ptr(sh, "sh", f, (G, d, 3)), *outs, _stream(stream)))

    def render_features(self, feats, out, stream=None):
        """Composite per-Gaussian attributes feats [G, C] with the last render's weights into
        out [V, H, W, C]."""
        import torch
        C = feats.shape[1] if feats.dim() == 2 else 0
        self._check(self._L.splat_render_features(
            self._h, _ptr(feats, "feats", torch.float32, (self.G, C)), C,
            _ptr(out, "out", torch.float32, (self.V, self.H, self.W, C)), _stream(stream)))

    def scatter(self, pixel_map, out, stream=None):
        """Scatter a per-pixel map [V, H, W, C] to the Gaussians with the last render's weights
        into out [G, C] (the adjoint of render_features)."""
        import torch
        C = pixel_map.shape[3] if pixel_map.dim() == 4 else 0
        self._check(self._L.splat_scatter(
            self._h, _ptr(pixel_map, "map", torch.float32, (self.V, self.H, self.W, C)), C,
            _ptr(out, "out", torch.float32, (self.G, C)), _stream(stream)))

    def attribution(self, obs, out, stream=None):
        """Scalar attribution [G, 3]: alphaT coverage, PRIMU-style error, error per coverage."""
        import torch
        self._check(self._L.splat_attribution(
            self._h, _ptr(obs, "obs", torch.float32, (self.V, self.H, self.W, 3)),
            _ptr(out, "out", torch.float32, (self.G, 3)), _stream(stream)))

    # -- inspection -----------------------------------------------------------------------------
    def copy_projection(self, rec, rect, stream=None):
        import torch
        self._check(self._L.splat_copy_projection(
            self._h, _ptr(rec, "rec", torch.float32, (self.V, self.G, 16)),
            _ptr(rect, "rect", torch.int32, (self.V, self.G, 4)), _stream(stream)))

    def copy_tile_lists(self, tile_offsets, ids, stream=None):
        import torch
        self._check(self._L.splat_copy_tile_lists(
            self._h, _ptr(tile_offsets, "tile_offsets", torch.int64),
            _ptr(ids, "ids", torch.int32), _stream(stream)))

    def copy_last(self, last, stream=None):
        import torch
        self._check(self._L.splat_copy_last(
            self._h, _ptr(last, "last", torch.int32, (self.V, self.H, self.W)), _stream(stream)))

    def copy_accumulators(self, acc, stream=None):
        import torch
        self._check(self._L.splat_copy_accumulators(
            self._h, _ptr(acc, "acc", torch.float64, (self.V, self.G, 8)), _stream(stream)))

    def pair_count(self, stream=None) -> int:
        out = ctypes.c_longlong()
        self._check(self._L.splat_pair_count(self._h, ctypes.byref(out), _stream(stream)))
        return int(out.value)

    @property
    def launch_count(self) -> int:
        return int(self._L.splat_launch_count(self._h))

    def check_status(self, stream=None):
        """Raise SplatError(BOUNDS) when a bounds check of the checked build failed since the
        last call (synchronises the stream; a no-op check in the release build)."""
        self._check(self._L.splat_check_status(self._h, _stream(stream)))

    def deterministic(self, enable: bool = True):
        """Fixed-point integer accumulation in the replay and the backward: bitwise reproducible
        tokens and gradients (off by default)."""
        self._check(self._L.splat_set_deterministic(self._h, 1 if enable else 0))

    def profile(self, enable: bool = True):
        """Bracket every kernel with CUDA events (per-kernel device time)."""
        self._check(self._L.splat_profile_enable(self._h, 1 if enable else 0))

    def profile_read(self, reset: bool = True) -> dict:
        """{kernel group name: (milliseconds, timed launches)} since the last reset."""
        n = KERNEL_GROUPS
        ms = (ctypes.c_double * n)()
        cnt = (ctypes.c_longlong * n)()
        self._check(self._L.splat_profile_read(self._h, ms, cnt, 1 if reset else 0))
        return {self._L.splat_kernel_name(i).decode(): (float(ms[i]), int(cnt[i]))
                for i in range(n)}
