"""GPU parity of the HyperVAttention options (PARK_FLAG_LOCAL_WINDOW,
PARK_FLAG_MERGE_Q) against the oracle: labels, centroids, permutations, masks
and CSR bit for bit, attention within the usual tolerance, and at the
HunyuanVideo shape the properties that hold at any size."""
import numpy as np
import pytest
import torch

from oracle import hva_oracle as hva
from oracle import park_oracle as po
from synth import CONFIGS
from synth.generator import gen_layer

import parity_util as pu

pytestmark = pytest.mark.gpu

# box (frames, rows, columns) per config: 8 boxes each
WINDOWS = {"tiny": (2, 4, 4), "small": (4, 8, 8), "small_text": (4, 8, 8), "small_ragged": (3, 5, 6)}


@pytest.fixture(scope="module")
def park():
    import block_sparse_attention_means_b200 as P
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    return P


def _cfg(name):
    if name == "small_text":
        return CONFIGS["small"].replace(name="small_text", H=2, n_text=64)
    if name == "small_ragged":  # boxes clipped at every grid edge, 1-2 centroids per box, text tokens
        return CONFIGS["small"].replace(name="small_ragged", H=2, n_text=24, NQ=48, NK=40)
    return CONFIGS[name]


def _run(park, name, window=None, merge=False, rounds=0, flags=0, p=None):
    cfg = _cfg(name)
    Q, K, V = gen_layer(cfg, 0)
    kw = {}
    if flags & 0x10:
        kw.update(topk_ratio=p)
    if window is not None:
        kw.update(grid=(cfg.T, cfg.Hg, cfg.W), window=window)
    if merge:
        kw.update(merge=True, merge_rounds=rounds or 8)
    p = cfg.p if p is None else p
    ref = po.layer(Q.astype(np.float64), K.astype(np.float64), V.astype(np.float64), cfg.NQ, cfg.NK, p,
                   cfg.iters, cfg.dtype, **kw)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    shape = park.Shape.of(cfg, dt)
    q, k, v = (pu.to_device(x, dt) for x in (Q, K, V))
    out = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, q.device, window=window, merge=merge, merge_rounds=rounds)
    out.flags |= flags | 0x200  # no query-tile packing: the tile-pair counter follows the merge cost model
    O, r = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, p, cfg.iters, out=out)
    torch.cuda.synchronize()
    assert r.status_code() == 0, f"device status {r.status_code()}"
    return cfg, ref, O, r


@pytest.mark.parametrize("name", ["tiny", "small", "small_text", "small_ragged"])
def test_local_window_matches_oracle(park, name):
    cfg, ref, O, r = _run(park, name, window=WINDOWS[name])
    fails = pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK)
    assert not fails, "\n".join(fails[:20])
    pu.assert_output_close(O, ref, cfg.dtype == "f32")
    # every video token's label lies in its box's centroid range
    win = hva.token_windows(cfg.T, cfg.Hg, cfg.W, cfg.n_text, WINDOWS[name])
    nW = int(win.max()) + 1
    ql = r.q_labels.cpu().numpy().reshape(-1, cfg.N)
    k0 = hva.window_starts(cfg.NQ, nW)
    grid = win >= 0
    for lab in ql:
        assert np.all(lab[grid] >= k0[win[grid]]) and np.all(lab[grid] < k0[win[grid] + 1])


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_merge_matches_oracle(park, name):
    cfg, ref, O, r = _run(park, name, merge=True)
    fails = pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK)
    assert not fails, "\n".join(fails[:20])
    pu.assert_output_close(O, ref, cfg.dtype == "f32")
    if cfg.dtype == "bf16":
        # the attention computed exactly the tile pairs the merge's cost model counts
        want = sum(hva.total_tile_cost(h["q_counts"], h["mask"], h["k_counts"]) for h in ref)
        assert int(r.counters[7].item()) == want


def test_merge_round_cap_matches_oracle(park):
    cfg, ref, O, r = _run(park, "small", merge=True, rounds=1)
    fails = pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK)
    assert not fails, "\n".join(fails[:20])


def test_merge_with_topk_and_ragged_windows(park):
    ratio = float(np.float32(0.3))
    cfg, ref, O, r = _run(park, "small_ragged", window=WINDOWS["small_ragged"], merge=True, flags=0x10, p=ratio)
    fails = pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK)
    assert not fails, "\n".join(fails[:20])
    pu.assert_output_close(O, ref, False)


def test_local_window_and_merge_together(park):
    cfg, ref, O, r = _run(park, "small_text", window=WINDOWS["small_text"], merge=True)
    fails = pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK)
    assert not fails, "\n".join(fails[:20])
    pu.assert_output_close(O, ref, False)


def test_hva_properties_at_hunyuan_shape(park):
    """HunyuanVideo shape (two heads, N = 119056, NQ = NK = 930): merging maps each
    query cluster to a root at or below it, gives the root the union of the kept
    sets and lowers the attention's tile pairs, which equal the cost model; the
    local-window assign (one warm-started iteration from known centroids) picks,
    for sampled tokens, the float64 nearest centroid of the token's box (all
    centroids for text tokens)."""
    cfg = CONFIGS["hunyuan"].replace(H=2, name="hunyuan_h2")
    Q, K, V = gen_layer(cfg, 0)
    shape = park.Shape.of(cfg, torch.bfloat16)
    q, k, v = (pu.to_device(x, torch.bfloat16) for x in (Q, K, V))
    dev = q.device
    plain = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, dev)
    plain.flags |= 0x200  # no query-tile packing: tile pairs as the merge cost model counts them
    _, r0 = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, cfg.p, cfg.iters, out=plain)
    merged = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, dev, merge=True)
    merged.flags |= 0x200
    _, r1 = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, cfg.p, cfg.iters, out=merged)
    torch.cuda.synchronize()
    assert r0.status_code() == 0 and r1.status_code() == 0
    l0, l1 = r0.q_labels.cpu().numpy(), r1.q_labels.cpu().numpy()
    m0, m1 = r0.mask.cpu().numpy().astype(bool), r1.mask.cpu().numpy().astype(bool)
    ko = r1.k_offsets.cpu().numpy()
    qo1 = r1.q_offsets.cpu().numpy()
    for h in range(cfg.H):
        root = np.full(cfg.NQ, -1)
        root[l0[0, h]] = l1[0, h]                    # one root per plain cluster ...
        assert np.array_equal(root[l0[0, h]], l1[0, h])
        live = root >= 0
        assert np.all(root[live] <= np.nonzero(live)[0])
        for r in np.nonzero(live)[0]:
            assert np.all(m1[0, h, root[r]] >= m0[0, h, r])
        gone = np.setdiff1d(np.nonzero(live)[0], root[live])
        assert not m1[0, h, gone].any()              # merged-away rows are empty
        assert len(gone) > 0
    want = sum(hva.total_tile_cost(np.diff(qo1[0, h]), m1[0, h], np.diff(ko[0, h])) for h in range(cfg.H))
    assert int(r1.counters[7].item()) == want
    assert int(r1.counters[7].item()) < int(r0.counters[7].item())

    # local windows: one iteration from r0's centroids
    window = (3, 15, 20)
    loc = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, dev, window=window)
    loc.q_centroids.copy_(r0.q_centroids)
    loc.k_centroids.copy_(r0.k_centroids)
    loc.flags |= 0x1 | 0x2                           # warm start both sides
    park.retrieve(q, k, shape, cfg.NQ, cfg.NK, cfg.p, 1, out=loc)
    torch.cuda.synchronize()
    assert loc.status_code() == 0
    win = hva.token_windows(cfg.T, cfg.Hg, cfg.W, cfg.n_text, window)
    nW = int(win.max()) + 1
    rng = np.random.default_rng(1)
    rows = np.concatenate([rng.choice(cfg.T * cfg.Hg * cfg.W, 1500, replace=False),
                           np.arange(cfg.T * cfg.Hg * cfg.W, cfg.N)[::8]])
    for side, X, lab, C in (("q", Q, loc.q_labels, r0.q_centroids), ("k", K, loc.k_labels, r0.k_centroids)):
        for h in range(cfg.H):
            Xh = X[0, h].astype(np.float64)
            Ch = pu.np64(C)[0, h]
            M = po.metric(Q[0, h].astype(np.float64)) if side == "k" else None
            got = lab.cpu().numpy()[0, h]
            k0 = hva.window_starts(Ch.shape[0], nW)
            for i in rows:
                lo, hi = (k0[win[i]], k0[win[i] + 1]) if win[i] >= 0 else (0, Ch.shape[0])
                d = po.distances(Xh[i:i + 1], Ch[lo:hi], M)[0]
                assert lo <= got[i] < hi
                j = got[i] - lo
                assert d[j] <= d.min() * (1 + 1e-9) + 1e-12, (side, h, i, got[i], lo + int(np.argmin(d)))
