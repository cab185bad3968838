"""GPU parity on inputs that reach far into the library's range precondition
(0 or 2^-40 <= |x| < 2^40): the centroid sums must stay exact (128-bit fixed
point), the certified assign must still decide every label as the float64
definition does, and the QRKC scores must not overflow, so labels, centroids,
masks and the CSR are compared bit for bit with the oracle.

Large magnitudes come as whole heads scaled by a power of two.  Mixing values
2^40 apart inside one head is accepted by the library too (exact sums), but
then the QRKC distance itself is ill-conditioned: float64 evaluations of it
by different valid formulas disagree by far more than the 1e-6 tie band, so
no bit-exact label comparison is defined there."""
import numpy as np
import pytest
import torch

from oracle import park_oracle as po
from synth import CONFIGS
from synth.generator import LayerConfig, gen_layer, with_extreme_magnitudes

import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def park():
    import block_sparse_attention_means_b200 as park
    return park


def _run(park, cfg, Q, K, V):
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    shape = park.Shape.of(cfg, dt)
    q, k, v = (pu.to_device(x, dt) for x in (Q, K, V))
    out = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, q.device, with_metric=True)
    O, r = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, cfg.p, cfg.iters, out=out)
    torch.cuda.synchronize()
    assert r.status_code() == 0, f"device status {r.status_code()}"
    return O, r


def _scale_heads(x, exps):
    """Multiply head h of [B, H, N, D] by 2^exps[h % len(exps)] (exact)."""
    y = np.array(x, dtype=np.float32, copy=True)
    for h in range(y.shape[1]):
        y[:, h] *= np.float32(2.0 ** exps[h % len(exps)])
    return y


# name -> (config, extreme-magnitude options, per-head power-of-two scales of Q and K,
#          whether outputs are compared)
CASES = {
    # 1 % of the elements at 2^-40 .. 2^-20, 0.2 % exact zeros
    "small_tiny_values": (CONFIGS["small"], dict(frac_small=0.01, frac_zero=0.002), (0,), True),
    # whole heads near the top of the range (values up to ~2^26, M up to ~2^50) and
    # near the bottom (2^-16 times unit scale), with the tiny values and zeros as
    # above: the QRKC operands use a scaled metric, the float32 scores must not
    # overflow, the 128-bit sums cover every magnitude
    "small_scaled_heads": (CONFIGS["small"], dict(frac_small=0.01, frac_zero=0.002), (0, 22, -16, 11), False),
    "tiny_f32_scaled": (CONFIGS["tiny"], dict(frac_small=0.02, frac_zero=0.005), (30,), False),
    "ragged": (LayerConfig("ragged", 2, 3, 3, 7, 11, 5, 128, "bf16", 9, 13, 4, 0.85, True, "normal"),
               dict(frac_small=0.03, frac_zero=0.01), (0,), True),
}


@pytest.mark.parametrize("name", list(CASES))
def test_extreme_magnitudes_match_oracle(park, name):
    cfg, kw, exps, check_out = CASES[name]
    Q, K, V = gen_layer(cfg, seed=21)
    Q = with_extreme_magnitudes(_scale_heads(Q, exps), cfg.dtype, 1, **kw)
    K = with_extreme_magnitudes(_scale_heads(K, exps), cfg.dtype, 2, **kw)
    V = with_extreme_magnitudes(V, cfg.dtype, 3, **kw)
    a = np.abs(np.concatenate([Q.ravel(), K.ravel()]))
    assert a[a > 0].min() < 2.0 ** -35 and a.max() < 2.0 ** 40
    ref = po.layer(Q, K, V, cfg.NQ, cfg.NK, cfg.p, cfg.iters, cfg.dtype)
    O, r = _run(park, cfg, Q, K, V)
    rep = {}
    fails = pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK, Q, K, cfg.p, rep)
    assert not fails, "\n".join(fails[:20])
    M = pu.np64(r.metric).reshape(-1, cfg.D, cfg.D)
    for bh, h in enumerate(ref):
        assert np.abs(M[bh] - h["M"]).max() / np.abs(h["M"]).max() < 1e-13
    if check_out:  # scaled heads make the Softmax one-hot; outputs are compared on unit-scale heads
        pu.assert_output_close(O, ref, cfg.dtype == "f32")
