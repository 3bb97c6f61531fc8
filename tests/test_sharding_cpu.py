"""View-sharded scoring, host side: partitioning, the reduce-scatter of per-Gaussian partial sums
over the Gaussian axis, and finalisation of each rank's rows -- on CPU with gloo ranks, each
rank computing its partials with the CPU oracle from its own views only. The gathered tokens must
equal the single-process oracle's."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from gaussian_splatting_raster_b200 import sharding


def test_partition_helpers():
    assert sharding.view_ranges(4, 2) == [(0, 2), (2, 4)]
    assert sharding.view_ranges(5, 3) == [(0, 2), (2, 4), (4, 5)]
    assert sharding.view_ranges(2, 3) == [(0, 1), (1, 2), (2, 2)]
    assert sharding.padded_rows(10, 4) == 12
    rows = [sharding.row_range(10, 4, r) for r in range(4)]
    assert rows == [(0, 3), (3, 6), (6, 9), (9, 10)]
    assert sharding.row_range(2, 4, 3) == (2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, cfg, lam, outdir):
    import dataclasses

    import torch.distributed as dist

    from oracle import oracle as O
    from synth import scenes

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sc = scenes.make(cfg)
        obs = O.observe(sc, "d")
        vlo, vhi = sharding.view_ranges(sc.V, world)[rank]
        G = sc.G
        d = (sc.sh_degree + 1) ** 2
        Gp = sharding.padded_rows(G, world)
        part = np.zeros((Gp, 11 + 3 * d))
        if vhi > vlo:  # this rank sees only its views
            local = dataclasses.replace(sc, viewmats=sc.viewmats[vlo:vhi],
                                        intrin=sc.intrin[vlo:vhi])
            out = O.run(local, obs[vlo:vhi], "d", lam=lam)
            part[:G] = O.partials(out["proj"], out["acc"], local)
        shard = sharding.reduce_partials(torch.from_numpy(part), None).numpy()
        lo, hi = sharding.row_range(G, world, rank)
        tok = O.finalize_partials(shard[: hi - lo], sc.sh_degree, lam)
        np.save(os.path.join(outdir, f"rank{rank}.npy"), tok)
        np.save(os.path.join(outdir, f"rows{rank}.npy"), np.array([lo, hi]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3, 5])
def test_view_sharded_tokens_equal_single_process(world, tmp_path):
    from oracle import oracle as O
    from synth import scenes

    cfg, lam = 2, 0.8  # three-layer scene: 4 views, 4096 Gaussians
    mp.spawn(_rank, args=(world, _free_port(), cfg, lam, str(tmp_path)), nprocs=world, join=True)
    sc = scenes.make(cfg)
    obs = O.observe(sc, "d")
    ref = O.run(sc, obs, "d", lam=lam)["tokens"]
    got = np.zeros_like(ref)
    for r in range(world):
        lo, hi = np.load(tmp_path / f"rows{r}.npy")
        got[lo:hi] = np.load(tmp_path / f"rank{r}.npy")
    np.testing.assert_allclose(got, ref, rtol=1e-9, atol=1e-12)
