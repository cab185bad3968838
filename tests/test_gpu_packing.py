"""Query-tile packing on the tensor-core attention path: the last tile of a
query cluster with several tiles shares the single tile of a smaller cluster,
every row still attending only to its own cluster's kept key clusters.  The
result must equal the oracle as without packing, with fewer work items and
(query tile, key tile) pairs."""
import numpy as np
import pytest
import torch

from oracle import park_oracle as po
from synth import CONFIGS
from synth.generator import gen_layer, gen_uniform

import parity_util as pu

pytestmark = pytest.mark.gpu

NO_PACK = 0x200


@pytest.fixture(scope="module")
def park():
    import block_sparse_attention_means_b200 as P
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return P


# 14 query clusters over 2048 rows: most spill into a second tile, a few can host
CFG = CONFIGS["small"].replace(name="small_pack", H=4, NQ=14, NK=32)


def _layer(park, cfg, flags, p, sip=None):
    Q, K, V = gen_layer(cfg, 0)
    shape = park.Shape.of(cfg, torch.bfloat16)
    q, k, v = (pu.to_device(x, torch.bfloat16) for x in (Q, K, V))
    out = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, q.device,
                               sip_uniform=None if sip is None else torch.from_numpy(sip).to(q.device))
    out.flags |= flags
    O, r = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, p, cfg.iters, out=out)
    torch.cuda.synchronize()
    assert r.status_code() == 0, f"device status {r.status_code()}"
    return O, r


def test_packing_matches_oracle_and_saves_tiles(park):
    cfg = CFG
    Q, K, V = gen_layer(cfg, 0)
    ref = po.layer(Q.astype(np.float64), K.astype(np.float64), V.astype(np.float64), cfg.NQ, cfg.NK, cfg.p,
                   cfg.iters, cfg.dtype)
    O1, r1 = _layer(park, cfg, 0, cfg.p)
    fails = pu.compare_retrieval(r1, ref, cfg.NQ, cfg.NK)
    assert not fails, "\n".join(fails[:20])
    pu.assert_output_close(O1, ref, False)
    O0, r0 = _layer(park, cfg, NO_PACK, cfg.p)
    pu.assert_output_close(O0, ref, False)
    c1, c0 = r1.counters.cpu().tolist(), r0.counters.cpu().tolist()
    assert c1[5] == c0[5]                       # the same attended query-key pairs
    assert c1[6] < c0[6] and c1[7] < c0[7]      # fewer work items and tile pairs
    assert torch.max(torch.abs(O1.float() - O0.float())).item() <= 1e-2


def test_packing_with_sip_weights(park):
    cfg = CFG
    ratio = float(np.float32(0.5))
    Q, K, V = gen_layer(cfg, 0)
    U = gen_uniform(cfg)
    ref = po.layer(Q.astype(np.float64), K.astype(np.float64), V.astype(np.float64), cfg.NQ, cfg.NK, ratio,
                   cfg.iters, cfg.dtype, sip_ratio=ratio, sip_u=U.astype(np.float64))
    O1, r1 = _layer(park, cfg, 0, ratio, sip=U)
    fails = pu.compare_retrieval(r1, ref, cfg.NQ, cfg.NK)
    assert not fails, "\n".join(fails[:20])
    pu.assert_output_close(O1, ref, False)
    _, r0 = _layer(park, cfg, NO_PACK, ratio, sip=U)
    assert r1.counters.cpu().tolist()[7] < r0.counters.cpu().tolist()[7]


def test_packing_at_hunyuan_shape(park):
    """Two HunyuanVideo-shaped heads: packed and unpacked outputs agree and the
    packing removes work items and tile pairs."""
    cfg = CONFIGS["hunyuan"].replace(H=2, name="hunyuan_h2")
    O1, r1 = _layer(park, cfg, 0, cfg.p)
    O0, r0 = _layer(park, cfg, NO_PACK, cfg.p)
    c1, c0 = r1.counters.cpu().tolist(), r0.counters.cpu().tolist()
    assert c1[5] == c0[5]
    assert c1[6] < c0[6] and c1[7] < c0[7]
    d = torch.max(torch.abs(O1.float() - O0.float())).item()
    assert d <= 1e-2, d
    print(f"\nwork items {c0[6]} -> {c1[6]}, tile pairs {c0[7]} -> {c1[7]}, max |dO| {d:.3g}")
