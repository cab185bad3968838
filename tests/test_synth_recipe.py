"""The seeded input recipe: deterministic per (seed, tensor, batch, head),
values exactly representable in the storage type and inside the library's
range precondition, standard-normal V and text tokens where the recipe says
so, and a 3D rotary embedding that rotates 22 / 21 / 21 channel pairs by the
t / y / w position."""
import numpy as np
import torch

from synth import CONFIGS
from synth import generator as g


def _small_hunyuan():
    # the HunyuanVideo recipe (normal V, 256 text tokens, RoPE) on 3 frames
    return CONFIGS["hunyuan"].replace(H=1, T=3, name="hunyuan_t3")


def test_slices_are_deterministic_and_distinct():
    cfg = CONFIGS["small"]
    a = g.gen_slice(cfg, "Q", 0, 1)
    assert np.array_equal(a, g.gen_slice(cfg, "Q", 0, 1))
    assert not np.array_equal(a, g.gen_slice(cfg, "Q", 0, 2))
    assert not np.array_equal(a, g.gen_slice(cfg, "K", 0, 1))
    assert not np.array_equal(a, g.gen_slice(cfg, "Q", 0, 1, seed=1))


def test_values_are_bf16_and_inside_the_range_precondition():
    cfg = _small_hunyuan()
    for t in "QKV":
        x = g.gen_slice(cfg, t, 0, 0)
        assert np.array_equal(torch.from_numpy(x).to(torch.bfloat16).float().numpy(), x)
        a = np.abs(x[x != 0])
        assert a.min() >= 2.0 ** -40 and a.max() < 2.0 ** 40 and np.all(np.isfinite(x))


def test_normal_v_and_text_tokens():
    cfg = _small_hunyuan()
    nv = cfg.T * cfg.Hg * cfg.W
    v = g.gen_slice(cfg, "V", 0, 0).astype(np.float64)
    q = g.gen_slice(cfg, "Q", 0, 0).astype(np.float64)
    assert v.shape == (nv + 256, cfg.D)
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1.0) < 0.01
    txt = q[nv:]
    assert abs(txt.mean()) < 0.02 and abs(txt.std() - 1.0) < 0.02


def test_rope_rotates_22_21_21_pairs_and_keeps_norms():
    cfg = CONFIGS["small"]
    x = np.random.default_rng(0).standard_normal((cfg.T * cfg.Hg * cfg.W, cfg.D))
    y = g._rope_3d(x, cfg)
    pair_norm = lambda z: np.hypot(z[:, 0::2], z[:, 1::2])
    assert np.allclose(pair_norm(x), pair_norm(y), rtol=1e-12)
    assert np.array_equal(y[0], x[0])                     # position (0, 0, 0): no rotation

    def moved_pairs(tok):
        d = np.abs(y[tok] - x[tok]).reshape(-1, 2).max(axis=1) > 1e-12
        return np.nonzero(d)[0]

    idx = lambda t, yy, w: (t * cfg.Hg + yy) * cfg.W + w
    assert moved_pairs(idx(1, 0, 0)).tolist() == list(range(0, 22))
    assert moved_pairs(idx(0, 1, 0)).tolist() == list(range(22, 43))
    assert moved_pairs(idx(0, 0, 1)).tolist() == list(range(43, 64))


def test_extreme_magnitudes_stay_inside_the_range():
    cfg = _small_hunyuan()
    x = g.gen_slice(cfg, "Q", 0, 0)
    y = g.with_extreme_magnitudes(x, "bf16", 3, frac_small=0.02, frac_zero=0.01, frac_large=0.01)
    assert np.array_equal(torch.from_numpy(y).to(torch.bfloat16).float().numpy(), y)
    a = np.abs(y[y != 0])
    assert a.min() >= 2.0 ** -40 and a.max() < 2.0 ** 40
    assert a.min() < 2.0 ** -38 and a.max() > 2.0 ** 38  # both ends are reached
    assert 0.005 < np.mean(y == 0) < 0.02
    assert np.array_equal(y, g.with_extreme_magnitudes(x, "bf16", 3, frac_small=0.02, frac_zero=0.01,
                                                       frac_large=0.01))
