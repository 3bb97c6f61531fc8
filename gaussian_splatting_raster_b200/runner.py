"""Device-memory plumbing around the C ABI: move a scene's arrays into CUDA tensors, allocate the
outputs, and issue the four calls in order. No arithmetic of the method happens here."""
from __future__ import annotations

import dataclasses

from . import Workspace, token_dim


@dataclasses.dataclass
class DeviceScene:
    means: "object"
    log_scales: "object"
    quats: "object"
    opac: "object"
    sh: "object"
    viewmats: "object"
    intrin: "object"
    bg: "object"
    H: int
    W: int

    @property
    def G(self):
        return int(self.means.shape[0])

    @property
    def V(self):
        return int(self.viewmats.shape[0])

    @property
    def deg(self):
        return {1: 0, 4: 1, 9: 2, 16: 3}[int(self.sh.shape[1])]


def to_device(scene, device="cuda") -> DeviceScene:
    import torch

    def t(a):
        return torch.as_tensor(a, dtype=torch.float32).contiguous().to(device)
    return DeviceScene(t(scene.means), t(scene.log_scales), t(scene.quats), t(scene.opac),
                       t(scene.sh), t(scene.viewmats), t(scene.intrin), t(scene.bg), scene.H,
                       scene.W)


@dataclasses.dataclass
class Outputs:
    img: "object"
    T: "object"
    n_contrib: "object"
    tokens: "object"


def alloc_outputs(ds: DeviceScene, device="cuda") -> Outputs:
    import torch
    V, H, W = ds.V, ds.H, ds.W
    return Outputs(torch.empty((V, H, W, 3), dtype=torch.float32, device=device),
                   torch.empty((V, H, W), dtype=torch.float32, device=device),
                   torch.empty((V, H, W), dtype=torch.int32, device=device),
                   torch.empty((ds.G, token_dim(ds.deg)), dtype=torch.float32, device=device))


def render(ws: Workspace, ds: DeviceScene, out: Outputs, stream=None) -> list[int]:
    ws.project(ds.means, ds.log_scales, ds.quats, ds.opac, ds.sh, ds.viewmats, ds.intrin, ds.H,
               ds.W, stream)
    n = ws.bin_sort(stream)
    ws.render(ds.bg, out.img, out.T, out.n_contrib, stream)
    return n


def render_and_score(ws: Workspace, ds: DeviceScene, obs, out: Outputs, lam: float = 1.0,
                     stream=None, fused: bool = True) -> list[int]:
    """Project, bin, render and score. fused: render and replay through splat_render_score (one
    kernel); otherwise splat_render, then splat_score_replay."""
    if not fused:
        n = render(ws, ds, out, stream)
        ws.score_replay(obs, out.tokens, lam, stream)
        return n
    ws.project(ds.means, ds.log_scales, ds.quats, ds.opac, ds.sh, ds.viewmats, ds.intrin, ds.H,
               ds.W, stream)
    n = ws.bin_sort(stream)
    ws.render_score(ds.bg, obs, out.img, out.T, out.n_contrib, out.tokens, lam, stream)
    return n


def render_and_backward(ws: Workspace, ds: DeviceScene, obs, out: Outputs, grads: dict,
                        stream=None) -> list[int]:
    """Render, then the renderer backward into the variants named in `grads` (raw, detached,
    support, pscale -> [G, 11 + 3d] fp32 tensors)."""
    n = render(ws, ds, out, stream)
    ws.backward(obs, ds.log_scales, ds.quats, ds.sh, stream=stream, **grads)
    return n


def workspace_for(ds: DeviceScene, lib=None) -> Workspace:
    return Workspace(max(ds.G, 1), ds.V, ds.H, ds.W, ds.deg, lib=lib)
