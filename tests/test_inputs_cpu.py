"""The seeded input recipe: the properties the parity tests and the design notes rely on.
CPU only."""
import numpy as np
import pytest

from routing_dispatch_expert_moe_b200 import inputs as I


@pytest.mark.parametrize("name", sorted(I.CONFIGS))
def test_router_grids_keep_fp32_logits_exact(name):
    cfg = I.CONFIGS[name]
    assert I.fits_exact_fp32(cfg)
    Wg, off, _ = I.gen_router(cfg, 0)
    q = 256.0 if cfg.act == "f32" else 1024.0
    assert np.array_equal(np.rint(Wg * q), Wg * q)                 # on the weight grid
    if off is not None:
        assert np.array_equal(np.rint(off * 8192.0), off * 8192.0)
    Wn = I.gen_noise_router(cfg, 0)
    assert Wn.shape == Wg.shape and np.array_equal(np.rint(Wn * q), Wn * q)
    assert not np.array_equal(Wn, Wg)                              # its own stream


def test_token_ids_follow_zipf_frequencies():
    cfg = I.CONFIGS["c2_handbook"]
    ids = I.gen_token_ids(cfg, seed=0, T=200_000)
    assert ids.dtype == np.int32 and ids.min() >= 0 and ids.max() < 32768
    counts = np.sort(np.bincount(ids, minlength=32768))[::-1]
    h = sum(1.0 / r for r in range(1, 32769))                      # harmonic number H_32768
    assert counts[0] / ids.size == pytest.approx(1.0 / h, rel=0.05)   # about 9%
    assert counts[1] / counts[0] == pytest.approx(0.5, rel=0.1)       # rank 2 at half of rank 1
    assert np.array_equal(I.gen_token_ids(cfg, seed=4), I.gen_token_ids(cfg, seed=4))   # seeded


def test_noise_draws_are_standard_normal_and_seeded():
    cfg = I.small_config("n", T=4000, E=64)
    n = I.gen_noise(cfg, seed=1)
    assert n.shape == (4000, 64) and n.dtype == np.float32
    assert abs(float(n.mean())) < 0.01 and abs(float(n.std()) - 1.0) < 0.01
    assert np.array_equal(n, I.gen_noise(cfg, seed=1)) and not np.array_equal(n, I.gen_noise(cfg, seed=2))
