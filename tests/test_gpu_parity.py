"""GPU parity: the CUDA path through the C ABI against the float64 oracle on
identical seeded inputs.  Labels, centroids, permutations, masks and the CSR
must be bit-exact; attention outputs within max-abs 2e-2 / mean-abs 2e-3
(bf16) or 1e-5 (float32)."""
import numpy as np
import pytest
import torch

from oracle import park_oracle as po
from synth import CONFIGS
from synth.generator import LayerConfig, gen_layer

import parity_util as pu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def park():
    import block_sparse_attention_means_b200 as park
    return park


def run_layer(park, cfg: LayerConfig, Q, K, V, p=None, NQ=None, NK=None, iters=None, with_metric=True):
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    shape = park.Shape.of(cfg, dt)
    NQ, NK = NQ or cfg.NQ, NK or cfg.NK
    q, k, v = (pu.to_device(x, dt) for x in (Q, K, V))
    out = park.alloc_retrieval(shape, NQ, NK, q.device, with_metric=with_metric)
    O, r = park.layer(q, k, v, shape, NQ, NK, cfg.p if p is None else p, iters or cfg.iters, out=out)
    torch.cuda.synchronize()
    assert r.status_code() == 0, f"device status {r.status_code()}"
    return O, r


def check_importance_bound(r, ref):
    """Every importance entry is within the row's reported relative bound of
    the oracle's float64 value (plus the float32 rounding of the output)."""
    imp = r.importance.cpu().numpy().astype(np.float64)
    bound = r.importance_bound.cpu().numpy().astype(np.float64)
    H = imp.shape[1]
    worst = 0.0
    for bh, h in enumerate(ref):
        b, hh = divmod(bh, H)
        want = h["importance"]
        slack = (bound[b, hh][:, None] + 2.0 ** -23) * want + 1e-30
        err = np.abs(imp[b, hh] - want)
        assert np.all(err <= slack), f"bh={bh}: importance outside its bound"
        live = (want > 0) & (bound[b, hh][:, None] > 0)  # rows certified in float32
        if live.any():
            worst = max(worst, float(np.max(err[live] / (bound[b, hh][:, None] * want + 1e-30)[live])))
    print(f"importance error / bound: max {worst:.3g}")


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_layer_matches_oracle(park, name):
    cfg = CONFIGS[name]
    Q, K, V = pu.inputs(name)
    ref = pu.oracle_layer(name)
    O, r = run_layer(park, cfg, Q, K, V)
    fails = pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK, Q, K, cfg.p)
    M = pu.np64(r.metric)
    for bh, h in enumerate(ref):
        rel = np.abs(M[0, bh] - h["M"]).max() / np.abs(h["M"]).max()
        assert rel < 1e-13, f"metric rel err {rel}"
    cnt = r.counters.cpu().numpy()
    print(f"\n{name}: counters {cnt.tolist()}")
    assert not fails, "\n".join(fails[:20])
    check_importance_bound(r, ref)
    worst, mean = pu.assert_output_close(O, ref, cfg.dtype == "f32")
    print(f"{name}: O max abs {worst:.3g} mean abs {mean:.3g}")
    pairs = sum(int(np.sum(np.bincount(h["q_labels"], minlength=cfg.NQ)[:, None] * h["mask"] *
                       np.bincount(h["k_labels"], minlength=cfg.NK)[None, :])) for h in ref)
    assert int(cnt[5]) == pairs
    assert int(cnt[4]) == sum(int(h["mask"].sum()) for h in ref)


# Selection variants (PARK Table 3 ablations, Table 10 top-k, the size prior):
# flag bits, oracle options, and the p passed (a retrieval ratio for top-k).
_RATIO = float(np.float32(0.3))  # the float32 value the C ABI receives
VARIANTS = {
    "no_qrkc": (0x4, (("qrkc", False),), None),
    "centroid_query": (0x8, (("pama_mode", "centroid"),), None),
    "topk": (0x10, (("topk_ratio", _RATIO),), _RATIO),
    "size_prior": (0x20, (("size_prior", True),), None),
    "all": (0x3C, (("pama_mode", "centroid"), ("qrkc", False), ("size_prior", True), ("topk_ratio", _RATIO)),
            _RATIO),
}


@pytest.mark.parametrize("variant", sorted(VARIANTS))
@pytest.mark.parametrize("name", ["tiny", "small"])
def test_selection_variants_match_oracle(park, name, variant):
    flags, opts, p = VARIANTS[variant]
    cfg = CONFIGS[name]
    p = cfg.p if p is None else p
    Q, K, V = pu.inputs(name)
    ref = pu.oracle_layer_variant(name, p, opts)
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    shape = park.Shape.of(cfg, dt)
    q, k, v = (pu.to_device(x, dt) for x in (Q, K, V))
    out = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, q.device)
    out.flags = flags
    O, r = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, p, cfg.iters, out=out)
    torch.cuda.synchronize()
    assert r.status_code() == 0, f"device status {r.status_code()}"
    fails = pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK)
    assert not fails, "\n".join(fails[:20])
    check_importance_bound(r, ref)
    pu.assert_output_close(O, ref, cfg.dtype == "f32")
    if "topk_ratio" in dict(opts):
        mask = r.mask.cpu().numpy().reshape(-1, cfg.NQ, cfg.NK)
        for bh, h in enumerate(ref):
            live = int((h["k_counts"] > 0).sum())
            want = max(1, int(np.ceil(_RATIO * live)))
            rows = h["q_counts"] > 0
            assert np.all(mask[bh][rows].sum(axis=1) == want)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_sip_matches_oracle(park, name):
    """SIP selection (caller-given uniforms) and the weighted attention: masks
    bit-exact, weights within the float32 / fast-path bound, outputs within the
    attention tolerance."""
    from synth.generator import gen_uniform
    cfg = CONFIGS[name]
    ratio = float(np.float32(0.4))
    Q, K, V = pu.inputs(name)
    U = gen_uniform(cfg)
    ref = po.layer(Q.astype(np.float64), K.astype(np.float64), V.astype(np.float64), cfg.NQ, cfg.NK, ratio,
                   cfg.iters, cfg.dtype, sip_ratio=ratio, sip_u=U.astype(np.float64))
    dt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    shape = park.Shape.of(cfg, dt)
    q, k, v = (pu.to_device(x, dt) for x in (Q, K, V))
    out = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, q.device, sip_uniform=torch.from_numpy(U).to(q.device))
    O, r = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, ratio, cfg.iters, out=out)
    torch.cuda.synchronize()
    assert r.status_code() == 0, f"device status {r.status_code()}"
    fails = pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK)
    assert not fails, "\n".join(fails[:20])
    W = r.block_weight.cpu().numpy().astype(np.float64).reshape(-1, cfg.NQ, cfg.NK)
    for bh, h in enumerate(ref):
        assert np.array_equal(W[bh] > 0, h["mask"])
        assert np.allclose(W[bh], h["weight"], rtol=1e-4, atol=0)
    pu.assert_output_close(O, ref, cfg.dtype == "f32")


def test_per_step_injection_small(park):
    """Feed the oracle's iteration-t centroids as a warm start and run one
    iteration: labels and updated centroids must match the oracle's step t."""
    cfg = CONFIGS["small"]
    Q, K, V = pu.inputs("small")
    dt = torch.bfloat16
    shape = park.Shape.of(cfg, dt)
    q, k = pu.to_device(Q, dt), pu.to_device(K, dt)
    heads = [(0, h) for h in range(cfg.H)]
    for t in (0, 3, 9):
        out = park.alloc_retrieval(shape, cfg.NQ, cfg.NK, q.device)
        qc = np.zeros((1, cfg.H, cfg.NQ, cfg.D))
        kc = np.zeros((1, cfg.H, cfg.NK, cfg.D))
        want = []
        for b, h in heads:
            x = Q[b, h].astype(np.float64)
            y = K[b, h].astype(np.float64)
            _, _, hq = po.kmeans(x, cfg.NQ, t + 1, None, "bf16", history=True)
            _, _, hk = po.kmeans(y, cfg.NK, t + 1, po.QueryMetric(x), "bf16", history=True)
            qc[0, h], kc[0, h] = hq[t], hk[t]
            lq, cq = po.kmeans(x, cfg.NQ, 1, None, "bf16", init=hq[t])
            lk, ck = po.kmeans(y, cfg.NK, 1, po.QueryMetric(x), "bf16", init=hk[t])
            want.append((lq, cq, lk, ck))
        out.q_centroids.copy_(pu.to_device(qc, dt))
        out.k_centroids.copy_(pu.to_device(kc, dt))
        out.flags = park._lib.PARK_FLAG_WARM_START_Q | park._lib.PARK_FLAG_WARM_START_K
        park.retrieve(q, k, shape, cfg.NQ, cfg.NK, cfg.p, 1, out=out)
        torch.cuda.synchronize()
        assert out.status_code() == 0
        ql, kl = out.q_labels.cpu().numpy(), out.k_labels.cpu().numpy()
        cq, ck = pu.np64(out.q_centroids), pu.np64(out.k_centroids)
        for h, (lq, wq, lk, wk) in enumerate(want):
            assert np.array_equal(ql[0, h], lq), f"iter {t} head {h}: query labels"
            assert np.array_equal(kl[0, h], lk), f"iter {t} head {h}: key labels"
            assert np.array_equal(cq[0, h], wq), f"iter {t} head {h}: query centroids"
            assert np.array_equal(ck[0, h], wk), f"iter {t} head {h}: key centroids"


def test_all_blocks_kept_is_dense(park):
    cfg = CONFIGS["small"]
    Q, K, V = pu.inputs("small")
    O, r = run_layer(park, cfg, Q, K, V, p=1.0)
    mask = r.mask.cpu().numpy().astype(bool)
    klab = r.k_labels.cpu().numpy()
    for h in range(cfg.H):
        live = np.bincount(klab[0, h], minlength=cfg.NK) > 0
        qlive = np.bincount(r.q_labels.cpu().numpy()[0, h], minlength=cfg.NQ) > 0
        assert np.array_equal(mask[0, h], qlive[:, None] & live[None, :])
    got = pu.np64(O)
    for h in range(cfg.H):
        dense = po.dense_attention(Q[0, h], K[0, h], V[0, h], pu.scale_of(cfg.D))
        d = np.abs(got[0, h] - dense)
        assert d.max() <= pu.O_MAX_ABS and d.mean() <= pu.O_MEAN_ABS


RAGGED = LayerConfig("ragged", 2, 3, 3, 7, 11, 5, 128, "bf16", 9, 13, 4, 0.85, True, "normal")
RAGGED_F32 = LayerConfig("ragged32", 2, 2, 3, 5, 7, 3, 64, "f32", 6, 9, 3, 0.8, False, "positional")
# bf16 with D = 64: the float64 / SIMT kernels instead of the tensor-core ones
RAGGED_D64 = LayerConfig("ragged64", 2, 3, 3, 7, 11, 5, 64, "bf16", 9, 13, 4, 0.85, True, "normal")


@pytest.mark.parametrize("cfg", [RAGGED, RAGGED_F32, RAGGED_D64], ids=["bf16", "f32", "bf16_d64"])
def test_ragged_batch_shapes(park, cfg):
    """B = 2, ragged N (not a multiple of any tile), text tokens."""
    Q, K, V = gen_layer(cfg, seed=3)
    ref = po.layer(Q, K, V, cfg.NQ, cfg.NK, cfg.p, cfg.iters, cfg.dtype)
    O, r = run_layer(park, cfg, Q, K, V)
    fails = pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK)
    assert not fails, "\n".join(fails[:20])
    pu.assert_output_close(O, ref, cfg.dtype == "f32")


@pytest.mark.parametrize("NQ,NK", [(1, 1), (1, 7), (5, 1)])
def test_degenerate_cluster_counts(park, NQ, NK):
    cfg = RAGGED.replace(NQ=NQ, NK=NK)
    Q, K, V = gen_layer(cfg, seed=4)
    ref = po.layer(Q, K, V, NQ, NK, cfg.p, cfg.iters, cfg.dtype)
    O, r = run_layer(park, cfg, Q, K, V)
    fails = pu.compare_retrieval(r, ref, NQ, NK)
    assert not fails, "\n".join(fails[:20])
    pu.assert_output_close(O, ref, False)


def test_identity_clustering_pin(park):
    """NQ = NK = N: every token is its own cluster, importance is the exact
    attention matrix and p = 1 gives dense attention."""
    cfg = LayerConfig("ident", 1, 2, 2, 4, 6, 0, 128, "bf16", 48, 48, 2, 1.0, True, "normal")
    Q, K, V = gen_layer(cfg, seed=5)
    O, r = run_layer(park, cfg, Q, K, V)
    ql = r.q_labels.cpu().numpy()
    assert np.array_equal(ql[0, 0], np.arange(cfg.N)) and np.array_equal(ql[0, 1], np.arange(cfg.N))
    imp = r.importance.cpu().numpy().astype(np.float64)
    for h in range(cfg.H):
        q, k = Q[0, h].astype(np.float64), K[0, h].astype(np.float64)
        S = pu.scale_of(cfg.D) * q @ k.T
        A = np.exp(S - S.max(1, keepdims=True))
        A /= A.sum(1, keepdims=True)
        assert np.allclose(imp[0, h], A, rtol=1e-3, atol=1e-7)
        dense = po.dense_attention(Q[0, h], K[0, h], V[0, h], pu.scale_of(cfg.D))
        assert np.abs(pu.np64(O)[0, h] - dense).max() <= pu.O_MAX_ABS


def test_large_logits_many_key_tiles(park):
    """Queries scaled by 4 give logits whose row maxima keep growing across the
    ~12 key tiles of a query tile, so the attention kernel rescales its
    accumulator for some rows of a warp but not others."""
    cfg = LayerConfig("wide", 1, 2, 8, 16, 16, 0, 128, "bf16", 6, 8, 3, 0.95, True, "normal")
    Q, K, V = gen_layer(cfg, seed=12)
    Q = (Q * 4.0).astype(np.float32)  # a power of two: still exact in bf16
    ref = po.layer(Q, K, V, cfg.NQ, cfg.NK, cfg.p, cfg.iters, cfg.dtype)
    O, r = run_layer(park, cfg, Q, K, V)
    fails = pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK)
    assert not fails, "\n".join(fails[:20])
    assert int(r.counters.cpu()[6]) >= cfg.NQ  # several query tiles
    pu.assert_output_close(O, ref, False)


@pytest.mark.parametrize("where,value", [("Q", 2.0 ** -41), ("K", -(2.0 ** 40)), ("V", 2.0 ** -41)])
def test_range_precondition_reported(park, where, value):
    """One finite element outside 0 or 2^-40 <= |x| < 2^40 in any of Q, K, V
    sets PARK_ERR_RANGE; the extreme values inside it do not."""
    cfg = RAGGED
    Q, K, V = gen_layer(cfg, seed=6)
    X = {"Q": Q.copy(), "K": K.copy(), "V": V.copy()}
    X[where][0, 1, 7, 3] = value
    dt = torch.bfloat16
    shape = park.Shape.of(cfg, dt)
    q, k, v = (pu.to_device(X[t], dt) for t in "QKV")
    _, r = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, cfg.p, cfg.iters)
    torch.cuda.synchronize()
    assert r.status_code() == park._lib.PARK_ERR_RANGE
    for edge in (2.0 ** -40, -(2.0 ** 40 - 2.0 ** 32), 0.0):  # the ends of the range: accepted
        X[where][0, 1, 7, 3] = edge
        q, k, v = (pu.to_device(X[t], dt) for t in "QKV")
        _, r = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, cfg.p, cfg.iters)
        torch.cuda.synchronize()
        assert r.status_code() == 0, edge


def test_cached_retrieval_reused_on_new_inputs(park):
    """Mask reuse across denoising steps (PARK Appendix Table 9): a retrieval
    computed on one step's Q, K is kept, and park_sparse_attn alone runs on the
    next step's Q, K, V with it; the output equals the oracle's block-sparse
    attention of the new tensors under the cached labels and mask."""
    cfg = CONFIGS["small"]
    Q0, K0, _ = pu.inputs("small", 0)
    Q1, K1, V1 = pu.inputs("small", 1)
    dt = torch.bfloat16
    shape = park.Shape.of(cfg, dt)
    q0, k0 = pu.to_device(Q0, dt), pu.to_device(K0, dt)
    r = park.retrieve(q0, k0, shape, cfg.NQ, cfg.NK, cfg.p, cfg.iters)
    torch.cuda.synchronize()
    assert r.status_code() == 0
    ref = pu.oracle_layer("small", 0)
    assert not pu.compare_retrieval(r, ref, cfg.NQ, cfg.NK, Q0, K0, cfg.p)
    q1, k1, v1 = (pu.to_device(x, dt) for x in (Q1, K1, V1))
    O = park.sparse_attn(q1, k1, v1, shape, cfg.NQ, cfg.NK, r)
    torch.cuda.synchronize()
    assert r.status_code() == 0
    got = pu.np64(O)
    worst = 0.0
    for h, hr in enumerate(ref):
        want = po.sparse_attention(Q1[0, h], K1[0, h], V1[0, h], hr["q_labels"], hr["k_labels"], hr["mask"],
                                   pu.scale_of(cfg.D))
        d = np.abs(got[0, h] - want)
        assert d.max() <= pu.O_MAX_ABS and d.mean() <= pu.O_MEAN_ABS, (h, d.max(), d.mean())
        worst = max(worst, float(d.max()))
        # and it is not the output of the retrieval's own step
        same = po.sparse_attention(Q0[0, h], K0[0, h], V1[0, h], hr["q_labels"], hr["k_labels"], hr["mask"],
                                   pu.scale_of(cfg.D))
        assert np.abs(got[0, h] - same).max() > 10 * pu.O_MAX_ABS
    print(f"cached retrieval on new inputs: max abs {worst:.3g}")


def test_stream_and_repeat_determinism(park):
    """Two calls on a side stream give identical results (no order-dependent
    arithmetic anywhere on the path)."""
    cfg = CONFIGS["small"]
    Q, K, V = pu.inputs("small")
    dt = torch.bfloat16
    shape = park.Shape.of(cfg, dt)
    q, k, v = (pu.to_device(x, dt) for x in (Q, K, V))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        O1, r1 = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, cfg.p, cfg.iters, stream=s)
        O2, r2 = park.layer(q, k, v, shape, cfg.NQ, cfg.NK, cfg.p, cfg.iters, stream=s)
    s.synchronize()
    assert torch.equal(O1, O2)
    assert torch.equal(r1.importance, r2.importance) and torch.equal(r1.mask, r2.mask)
