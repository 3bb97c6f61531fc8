"""The seeded synthetic workloads both sides consume: each configuration has the sizes the
benchmark tables state, the same seed gives the same arrays bit for bit, another seed does not,
and the layouts follow the conventions the library and the oracle assume (fp32, contiguous,
finite; cameras are rigid world-to-camera transforms with positive focal lengths)."""
import numpy as np
import pytest

from synth import scenes

# (G, V, H, W, SH degree) per configuration; the two largest take long to draw and are covered by
# the GPU parity tests and the benchmark
SIZES = {1: (256, 1, 64, 64, 0), 2: (4096, 4, 128, 128, 1), 4: (311296, 4, 512, 960, 2)}


@pytest.mark.parametrize("cfg", sorted(SIZES))
def test_configuration_sizes_and_layout(cfg):
    sc = scenes.make(cfg)
    G, V, H, W, deg = SIZES[cfg]
    assert (sc.G, sc.V, sc.H, sc.W, sc.sh_degree) == (G, V, H, W, deg)
    d = (deg + 1) ** 2
    assert sc.means.shape == (G, 3) and sc.log_scales.shape == (G, 3)
    assert sc.quats.shape == (G, 4) and sc.opac.shape == (G,) and sc.sh.shape == (G, d, 3)
    assert sc.viewmats.shape == (V, 4, 4) and sc.intrin.shape == (V, 4) and sc.bg.shape == (3,)
    for a in (sc.means, sc.log_scales, sc.quats, sc.opac, sc.sh, sc.viewmats, sc.intrin):
        assert a.dtype == np.float32 and a.flags.c_contiguous and np.isfinite(a).all()
    # world -> camera: orthonormal rotation block, last row (0, 0, 0, 1)
    R = sc.viewmats[:, :3, :3].astype(np.float64)
    assert np.allclose(R @ R.transpose(0, 2, 1), np.eye(3), atol=1e-5)
    assert np.allclose(sc.viewmats[:, 3], [0, 0, 0, 1])
    assert (sc.intrin[:, :2] > 0).all()
    # the observed copy perturbs means and colours only
    assert sc.obs_means.shape == sc.means.shape and sc.obs_sh.shape == sc.sh.shape


@pytest.mark.parametrize("cfg", [1, 2, 4])
def test_same_seed_same_bits(cfg):
    a, b = scenes.make(cfg), scenes.make(cfg)
    for name in ("means", "log_scales", "quats", "opac", "sh", "viewmats", "intrin", "bg",
                 "obs_means", "obs_sh"):
        assert np.array_equal(getattr(a, name), getattr(b, name)), name
    c = scenes.CONFIGS[cfg](1000 + cfg + 1)
    assert not np.array_equal(a.means, c.means)


def test_pixel_noise_is_seeded():
    sc = scenes.make(2)
    assert sc.obs_noise_sigma > 0
    assert np.array_equal(sc.pixel_noise(), sc.pixel_noise())
