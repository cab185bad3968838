"""GPU parity on inputs that reach both ends of the library's range
precondition (0 or 2^-40 <= |x| < 2^40): the centroid sums must stay exact
(128-bit fixed point), the certified assign must still decide every label as
the float64 definition does, and the QRKC scores must not overflow, so labels,
centroids, masks and the CSR are compared bit for bit with the oracle."""
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


CASES = {
    # 1 % of the elements at 2^-40 .. 2^-20, 0.2 % exact zeros
    "small_tiny_values": (CONFIGS["small"], dict(frac_small=0.01, frac_zero=0.002), True),
    # plus 0.05 % at 2^16 .. 2^40 in Q and K (M reaches 2^70 and more)
    "small_huge_values": (CONFIGS["small"], dict(frac_small=0.01, frac_zero=0.002, frac_large=0.0005), False),
    "tiny_f32": (CONFIGS["tiny"], dict(frac_small=0.02, frac_zero=0.005, frac_large=0.002), False),
    "ragged": (LayerConfig("ragged", 2, 3, 3, 7, 11, 5, 128, "bf16", 9, 13, 4, 0.85, True, "normal"),
               dict(frac_small=0.03, frac_zero=0.01), True),
}


@pytest.mark.parametrize("name", list(CASES))
def test_extreme_magnitudes_match_oracle(park, name):
    cfg, kw, check_out = CASES[name]
    Q, K, V = gen_layer(cfg, seed=21)
    Q = with_extreme_magnitudes(Q, cfg.dtype, 1, **kw)
    K = with_extreme_magnitudes(K, cfg.dtype, 2, **kw)
    V = with_extreme_magnitudes(V, cfg.dtype, 3, **{**kw, "frac_large": 0.0})
    small = np.abs(Q[(Q != 0) & (np.abs(Q) < 2.0 ** -20)])
    assert small.size > 0 and small.min() < 2.0 ** -35
    ref = po.layer(Q, K, V, cfg.NQ, cfg.NK, cfg.p, cfg.iters, cfg.dtype)
    O, r = _run(park, cfg, Q, K, V)
    rep = {}
    fails = pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK, Q, K, cfg.p, rep)
    assert not fails, "\n".join(fails[:20])
    M = pu.np64(r.metric).reshape(-1, cfg.D, cfg.D)
    for bh, h in enumerate(ref):
        assert np.abs(M[bh] - h["M"]).max() / np.abs(h["M"]).max() < 1e-13
    if check_out:  # huge inputs make the Softmax one-hot; outputs are compared where values stay unit-scale
        pu.assert_output_close(O, ref, cfg.dtype == "f32")
