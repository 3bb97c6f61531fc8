"""View-sharded render + score replay over several GPUs (one process per GPU).

Every cross-view quantity of a Gaussian's token is a sum over views ("Research Proposal: Renderer
Score Tokens for Recurrent Gaussian Splatting", "Exact Score Operators": q_g, the covector
pullback b, s^alpha, s^SH and the conditioning matrix A are gamma-weighted view sums with
gamma_gv / q_gv = 1 / q_g). So each rank projects all Gaussians into its own contiguous block of
views, renders and replays them, and writes per-Gaussian partial sums; one reduce-scatter over the
Gaussian axis (NCCL over NVLink on GPUs) leaves each rank the complete sums of its slice of
Gaussians, which it turns into tokens. The only exchange is that reduce-scatter of
G x (11 + 3d) fp32 sums.

Host-side logic only (partitioning, padding, the collective); all arithmetic runs in the library.
"""
from __future__ import annotations

import dataclasses

from . import finalize_partials, partials_dim, token_dim


def view_ranges(V: int, world: int) -> list[tuple[int, int]]:
    """Contiguous, balanced view blocks [lo, hi) per rank (empty blocks when V < world)."""
    base, extra = divmod(V, world)
    out, lo = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((lo, lo + n))
        lo += n
    return out


def padded_rows(G: int, world: int) -> int:
    """Gaussian rows padded to a multiple of the world size (equal reduce-scatter shards)."""
    return ((G + world - 1) // world) * world


def row_range(G: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [lo, hi) of the unpadded Gaussians owned by `rank` after the reduce-scatter."""
    per = padded_rows(G, world) // world
    lo = min(G, rank * per)
    return lo, min(G, lo + per)


def reduce_partials(partials_padded, group=None):
    """Sum the ranks' [G_pad, K] partials and return this rank's [G_pad / world, K] shard."""
    import torch
    import torch.distributed as dist
    world = dist.get_world_size(group)
    shard = torch.empty((partials_padded.shape[0] // world, partials_padded.shape[1]),
                        dtype=partials_padded.dtype, device=partials_padded.device)
    dist.reduce_scatter_tensor(shard, partials_padded, group=group)
    return shard


def sharded_tokens(ws, ds, obs, lam: float = 1.0, group=None):
    """Tokens of this rank's Gaussian rows, views split over the ranks of `group`.

    ws: a Workspace sized for all Gaussians and this rank's views; ds: the full DeviceScene;
    obs: [V, H, W, 3] observations of all views. Returns (tokens [hi - lo, 9 + 3d], (lo, hi),
    per-view render outputs of this rank's views or None when it holds no view, list instances
    per local view)."""
    import torch
    import torch.distributed as dist
    from . import runner

    rank, world = dist.get_rank(group), dist.get_world_size(group)
    G, deg = ds.G, ds.deg
    vlo, vhi = view_ranges(ds.V, world)[rank]
    Gp = padded_rows(G, world)
    partials = torch.zeros((Gp, partials_dim(deg)), dtype=torch.float32, device=ds.means.device)
    out, n = None, []
    if vhi > vlo:
        local = dataclasses.replace(ds, viewmats=ds.viewmats[vlo:vhi].contiguous(),
                                    intrin=ds.intrin[vlo:vhi].contiguous())
        out = runner.alloc_outputs(local)
        n = runner.render(ws, local, out)
        ws.score_partials(obs[vlo:vhi].contiguous(), partials[:G])
    shard = reduce_partials(partials, group)
    lo, hi = row_range(G, world, rank)
    tokens = torch.empty((hi - lo, token_dim(deg)), dtype=torch.float32, device=shard.device)
    if hi > lo:
        finalize_partials(shard[: hi - lo].contiguous(), deg, tokens, lam)
    return tokens, (lo, hi), out, n
