"""Query-tile pairing on the tensor-core attention path: two 128-row query tiles
per CTA share every K/V tile (the tiles of one cluster, or two single-tile
clusters of a head over the union of their kept key clusters, each row still
masking what its own cluster does not keep).  The result must equal the
oracle's and the unpaired kernel's; the attended query-key pairs are the same."""
import numpy as np
import pytest
import torch

from oracle import park_oracle as po
from synth import CONFIGS
from synth.generator import LayerConfig, gen_layer, gen_uniform

import parity_util as pu

pytestmark = pytest.mark.gpu

NO_PAIR = 0x400
NO_PACK = 0x200


@pytest.fixture(scope="module")
def park():
    import block_sparse_attention_means_b200 as P
    return P


def _layer(park, cfg, flags, p, Q, K, V, sip=None):
    shape = park.Shape.of(cfg, torch.bfloat16)
    q, k, v = (pu.to_device(x, torch.bfloat16) for x in (Q, K, V))
    out = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, q.device,
                               sip_uniform=None if sip is None else torch.from_numpy(sip).to(q.device))
    out.flags |= flags
    O, r = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, p, cfg.iters, out=out)
    torch.cuda.synchronize()
    assert r.status_code() == 0, f"device status {r.status_code()}"
    return O, r


# clusters of about 128 rows (single tiles, paired across clusters), about 280 rows (tiles
# of one cluster paired), and a ragged grid with text tokens
CASES = {
    "small_single_tiles": CONFIGS["small"].replace(name="pair_single", NQ=16, NK=32),
    "small_multi_tiles": CONFIGS["small"].replace(name="pair_multi", NQ=7, NK=24),
    "ragged_text": LayerConfig("pair_ragged", 2, 3, 3, 9, 13, 40, 128, "bf16", 5, 11, 4, 0.85, True, "normal"),
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("pack", [True, False], ids=["packed", "unpacked"])
def test_pairing_matches_oracle_and_unpaired(park, name, pack):
    cfg = CASES[name]
    Q, K, V = gen_layer(cfg, 2)
    ref = po.layer(Q, K, V, cfg.NQ, cfg.NK, cfg.p, cfg.iters, cfg.dtype)
    base = 0 if pack else NO_PACK
    O1, r1 = _layer(park, cfg, base, cfg.p, Q, K, V)
    fails = pu.compare_retrieval(r1, ref, cfg.NQ, cfg.NK, Q, K, cfg.p)
    assert not fails, "\n".join(fails[:20])
    worst, mean = pu.assert_output_close(O1, ref, False)
    O0, r0 = _layer(park, cfg, base | NO_PAIR, cfg.p, Q, K, V)
    c1, c0 = r1.counters.cpu().tolist(), r0.counters.cpu().tolist()
    assert c1[5] == c0[5] and c1[6] == c0[6]  # the same attended pairs and query tiles
    d = torch.max(torch.abs(O1.float() - O0.float())).item()
    assert d <= 1e-2, d
    print(f"\n{name} packed={pack}: max abs {worst:.3g} mean abs {mean:.3g}; tile pairs {c0[7]} -> {c1[7]}, "
          f"paired vs unpaired max |dO| {d:.3g}")


def test_pairing_dense(park):
    """p = 1: every block kept, every pair of tiles shares its whole list: equals
    dense attention."""
    cfg = CONFIGS["small"].replace(name="pair_dense", NQ=16, NK=16, p=1.0)
    Q, K, V = gen_layer(cfg, 3)
    O, r = _layer(park, cfg, 0, 1.0, Q, K, V)
    got = pu.np64(O)
    for h in range(cfg.H):
        dense = po.dense_attention(Q[0, h], K[0, h], V[0, h], pu.scale_of(cfg.D))
        d = np.abs(got[0, h] - dense)
        assert d.max() <= pu.O_MAX_ABS and d.mean() <= pu.O_MEAN_ABS


def test_pairing_with_sip_weights(park):
    cfg = CASES["small_single_tiles"]
    ratio = float(np.float32(0.5))
    Q, K, V = gen_layer(cfg, 4)
    U = gen_uniform(cfg)
    ref = po.layer(Q.astype(np.float64), K.astype(np.float64), V.astype(np.float64), cfg.NQ, cfg.NK, ratio,
                   cfg.iters, cfg.dtype, sip_ratio=ratio, sip_u=U.astype(np.float64))
    O1, r1 = _layer(park, cfg, 0, ratio, Q, K, V, sip=U)
    fails = pu.compare_retrieval(r1, ref, cfg.NQ, cfg.NK)
    assert not fails, "\n".join(fails[:20])
    pu.assert_output_close(O1, ref, False)


def test_pairing_at_hunyuan_shape(park):
    """Two HunyuanVideo-shaped heads: paired and unpaired outputs agree, with the
    same attended pairs and fewer key-tile loads per query tile."""
    cfg = CONFIGS["hunyuan"].replace(H=2, name="hunyuan_h2")
    Q, K, V = gen_layer(cfg, 0)
    O1, r1 = _layer(park, cfg, 0, cfg.p, Q, K, V)
    O0, r0 = _layer(park, cfg, NO_PAIR, cfg.p, Q, K, V)
    c1, c0 = r1.counters.cpu().tolist(), r0.counters.cpu().tolist()
    assert c1[5] == c0[5] and c1[6] == c0[6]
    d = torch.max(torch.abs(O1.float() - O0.float())).item()
    assert d <= 1e-2, d
    print(f"\nwork items {c1[6]}, tile pairs {c0[7]} -> {c1[7]}, max |dO| {d:.3g}")
