"""Selection variants measured against dense attention on one HunyuanVideo-shaped
head (N = 119056, NQ = NK = 930): the attention recall of the kept blocks (PARK
Table 1's quantity), the PAMA-to-block-mass total variation (PARK Table 4's
quantity) and the relative error of the attention output against dense
attention, all on 1024 sampled query rows, computed by the oracle's float64
diagnostics from the labels, centroids, masks, weights and outputs that the GPU
produced.  The values are printed (pytest -s); the assertions are sanity bounds
only, since the pages' absolute values are on real activations."""
import math

import numpy as np
import pytest
import torch

from oracle import park_oracle as po
from synth import CONFIGS
from synth.generator import gen_layer, gen_uniform

import parity_util as pu

pytestmark = pytest.mark.gpu

# flag bits of park_retrieval.flags and the p passed (a retrieval ratio for top-k and SIP)
VARIANTS = {"park (top-p 0.9)": (0x0, 0.9), "w/o QRKC": (0x4, 0.9), "w/o PAMA": (0x8, 0.9),
            "top-k 0.3": (0x10, 0.3), "SIP 0.3": (0x40, 0.3), "size prior": (0x20, 0.9),
            "HVA merge": (0x80, 0.9), "HVA local 3x15x20": (0x100, 0.9), "HVA both": (0x180, 0.9)}
WINDOW = (3, 15, 20)


def test_variant_recall_tv_and_output_error():
    import block_sparse_attention_means_b200 as park
    cfg = CONFIGS["hunyuan"].replace(H=1, name="hunyuan_h1")
    Q, K, V = gen_layer(cfg, 0)
    Q0, K0, V0 = (x[0, 0].astype(np.float64) for x in (Q, K, V))
    s = 1.0 / math.sqrt(cfg.D)
    rows = np.sort(np.random.default_rng(0).choice(cfg.N, 1024, replace=False))
    dense = po.dense_attention(Q0[rows], K0, V0, s)
    shape = park.Shape.of(cfg, torch.bfloat16)
    q, k, v = (pu.to_device(x, torch.bfloat16) for x in (Q, K, V))
    U = torch.from_numpy(gen_uniform(cfg)).to(q.device)
    print()
    for name, (flags, p) in VARIANTS.items():
        out = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, q.device, sip_uniform=U if flags & 0x40 else None,
                                   window=WINDOW if flags & 0x100 else None)
        out.flags = flags
        O, _ = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, p, cfg.iters, out=out)
        torch.cuda.synchronize()
        assert out.status_code() == 0
        ql, kl = out.q_labels.cpu().numpy()[0, 0], out.k_labels.cpu().numpy()[0, 0]
        mask = out.mask.cpu().numpy()[0, 0].astype(bool)
        CK = pu.np64(out.k_centroids)[0, 0]
        recall = po.block_recall(Q0, K0, ql, kl, mask, s, rows)
        tv = po.attention_tv(Q0[rows], K0, kl, cfg.NK, CK, s)
        live = np.bincount(kl, minlength=cfg.NK) > 0
        qlive = np.bincount(ql, minlength=cfg.NQ) > 0
        kept = mask[qlive][:, live].mean()
        Og = O[0, 0].float().cpu().numpy().astype(np.float64)[rows]
        err = np.linalg.norm(Og - dense) / np.linalg.norm(dense)
        print(f"{name:18s} recall {recall:.4f}  TV {tv:.4f}  kept {kept:.4f}  output rel. error {err:.4f}  "
              f"key tiles {int(out.counters[7].item())}")
        assert 0.0 < recall <= 1.0 + 1e-9
        assert 0.0 <= tv <= 1.0
        assert np.isfinite(err)
