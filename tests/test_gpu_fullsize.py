"""GPU parity at the sizes the benchmark runs: the CUDA path against the float64
oracle on whole heads of the Wan- and HunyuanVideo-shaped layers and of the
granularity sweep (NK = 3721), and on moderate shapes whose cluster counts
take every multi-chunk path of the kernels (several 128-centroid chunks in the
assign and PAMA GEMMs, both PAMA epilogue groups, the 64-row float64 PAMA tiles
and 2048-wide top-p sorts when NK > 1024).

Three comparisons per case:
* the whole 10-iteration trajectory (cold start), labels, centroids,
  permutations, masks and CSR bit for bit with ties counted (parity_util);
* per-step injection: the oracle's centroids entering iteration t given as a
  warm start, one iteration run, labels and updated centroids compared
  (t = 0 and the last iteration; at the last one also masks, importance and
  outputs, which then follow the oracle's own clustering);
* attention outputs on sampled whole query clusters against the oracle's
  block-sparse attention of those rows.
"""
import functools
import math

import numpy as np
import pytest
import torch

from oracle import park_oracle as po
from synth import CONFIGS
from synth.generator import LayerConfig, gen_tensor

import parity_util as pu

pytestmark = pytest.mark.gpu

HUN = CONFIGS["hunyuan"]
WAN = CONFIGS["wan"]
SMALL = CONFIGS["small"]

# name -> (config, heads of the full layer to take, NQ, NK, p)
CASES = {
    "hunyuan": (HUN, ((0, 0), (0, 23)), HUN.NQ, HUN.NK, 0.9),
    "wan": (WAN, ((0, 0), (0, 39)), WAN.NQ, WAN.NK, 0.9),
    "hunyuan_nk32": (HUN, ((0, 5),), HUN.NQ, 3721, 0.9),
    # small grid, cluster counts above one 128-wide chunk: NQ = NK = 300 (three
    # chunks: the centroid rings wrap, both PAMA epilogue groups work) and
    # NK = 1100 (64-row float64 PAMA tiles, 2048-wide top-p sort)
    "small_300": (SMALL, ((0, 0), (0, 7)), 300, 300, 0.9),
    "small_1100": (SMALL, ((0, 1), (0, 6)), 300, 1100, 0.9),
}
FULL = ("hunyuan", "wan", "hunyuan_nk32")


@functools.lru_cache(maxsize=None)
def case_inputs(name):
    cfg, heads, NQ, NK, p = CASES[name]
    Q, K, V = (gen_tensor(cfg, t, heads=list(heads)) for t in ("Q", "K", "V"))
    sub = cfg.replace(B=1, H=len(heads), NQ=NQ, NK=NK, p=p)
    return sub, Q[None], K[None], V[None]


@functools.lru_cache(maxsize=None)
def case_oracle(name):
    sub, Q, K, V = case_inputs(name)
    return [po.retrieve_head(Q[0, h], K[0, h], sub.NQ, sub.NK, sub.p, sub.iters, sub.dtype) for h in range(sub.H)]


@pytest.fixture(scope="module")
def park():
    import block_sparse_attention_means_b200 as park
    return park


def run_gpu(park, sub, Q, K, V, iters, q_init=None, k_init=None):
    dt = torch.bfloat16
    shape = park.Shape.of(sub, dt)
    q, k, v = (pu.to_device(x, dt) for x in (Q, K, V))
    out = park.alloc_retrieval(shape, sub.NQ, sub.NK, q.device, with_metric=True)
    if q_init is not None:
        out.q_centroids.copy_(pu.to_device(q_init, dt))
        out.k_centroids.copy_(pu.to_device(k_init, dt))
        out.flags = park._lib.PARK_FLAG_WARM_START_Q | park._lib.PARK_FLAG_WARM_START_K
    O, r = park.layer(q, k, v, shape, sub.NQ, sub.NK, sub.p, iters, out=out)
    torch.cuda.synchronize()
    assert r.status_code() == 0, f"device status {r.status_code()}"
    return O, r


def check_bound(r, refs):
    imp = r.importance.cpu().numpy().astype(np.float64)[0]
    bound = r.importance_bound.cpu().numpy().astype(np.float64)[0]
    for h, ref in enumerate(refs):
        want = ref["importance"]
        slack = (bound[h][:, None] + 2.0 ** -23) * want + 1e-30
        bad = np.abs(imp[h] - want) > slack
        assert not bad.any(), f"head {h}: {int(bad.sum())} importance entries outside their bound"


def check_sampled_outputs(O, sub, Q, K, V, refs, n_clusters=8, seed=0):
    """Outputs of every row of n_clusters whole query clusters (seeded choice)
    against the oracle's block-sparse attention of those rows."""
    got = pu.np64(O)[0]
    rng = np.random.default_rng(seed)
    worst, acc, n = 0.0, 0.0, 0
    for h, ref in enumerate(refs):
        live = np.nonzero(ref["q_counts"] > 0)[0]
        for r in rng.choice(live, size=min(n_clusters, live.size), replace=False):
            rows = np.nonzero(ref["q_labels"] == r)[0]
            want = po.sparse_attention(Q[0, h], K[0, h], V[0, h], ref["q_labels"], ref["k_labels"], ref["mask"],
                                       1.0 / math.sqrt(sub.D), rows=rows)
            d = np.abs(got[h][rows] - want)
            worst = max(worst, float(d.max()))
            acc += float(d.sum())
            n += d.size
    print(f"sampled outputs: {n // sub.D} rows, max abs {worst:.3g}, mean abs {acc / n:.3g}")
    assert worst <= pu.O_MAX_ABS and acc / n <= pu.O_MEAN_ABS


def check_counters(r, refs):
    cnt = r.counters.cpu().numpy()
    pairs = sum(int(np.sum(ref["q_counts"][:, None] * ref["mask"] * ref["k_counts"][None, :])) for ref in refs)
    assert int(cnt[5]) == pairs
    assert int(cnt[4]) == sum(int(ref["mask"].sum()) for ref in refs)
    print(f"counters {cnt.tolist()}")


@pytest.mark.parametrize("name", list(CASES))
def test_trajectory_matches_oracle(park, name):
    """Cold start, every iteration on the GPU: the final clustering, selection
    and outputs against the oracle's, ties counted."""
    sub, Q, K, V = case_inputs(name)
    refs = case_oracle(name)
    O, r = run_gpu(park, sub, Q, K, V, sub.iters)
    rep = {}
    fails = pu.compare_retrieval(r, refs, sub.NQ, sub.NK, Q, K, sub.p, rep)
    assert not fails, "\n".join(fails[:20])
    M = pu.np64(r.metric)[0]
    for h, ref in enumerate(refs):
        assert np.abs(M[h] - ref["M"]).max() / np.abs(ref["M"]).max() < 1e-13
    if rep["cascaded_heads"] == 0:
        check_bound(r, refs)
        check_counters(r, refs)
        check_sampled_outputs(O, sub, Q, K, V, refs)


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("step", ["first", "last"])
def test_step_injection_matches_oracle(park, name, step):
    """One GPU iteration from the oracle's centroids entering iteration t (t =
    0: the strided initialisation, cold start; t = iters - 1: a warm start):
    labels and updated centroids against the oracle's iteration t; after the
    last iteration also masks, importance bounds and sampled outputs."""
    sub, Q, K, V = case_inputs(name)
    refs = case_oracle(name)
    if step == "first":
        O, r = run_gpu(park, sub, Q, K, V, 1)
        want = []
        for h, ref in enumerate(refs):
            x, y = Q[0, h].astype(np.float64), K[0, h].astype(np.float64)
            ql = po.assign(x, ref["q_hist"][0])
            kl = po.assign(y, ref["k_hist"][0], ref["k_metric"])
            want.append(dict(ref, q_labels=ql, k_labels=kl, q_centroids=ref["q_hist"][1],
                             k_centroids=ref["k_hist"][1], q_hist=ref["q_hist"][:1], k_hist=ref["k_hist"][:1]))
        ql, kl = r.q_labels.cpu().numpy()[0], r.k_labels.cpu().numpy()[0]
        qc, kc = pu.np64(r.q_centroids)[0], pu.np64(r.k_centroids)[0]
        ties = 0
        for h, w in enumerate(want):
            for side, got, cen, X, M in (("q", ql[h], qc[h], Q[0, h], None),
                                         ("k", kl[h], kc[h], K[0, h], w["k_metric"])):
                bad, exc = pu.label_ties(X, w[f"{side}_hist"][0], M, got, w[f"{side}_labels"])
                assert np.setdiff1d(bad, exc).size == 0, f"head {h} {side}: labels differ not at a tie"
                ties += exc.size
                touched = np.union1d(got[bad], w[f"{side}_labels"][bad])
                keep = np.setdiff1d(np.arange(cen.shape[0]), touched)
                assert np.array_equal(cen[keep], w[f"{side}_centroids"][keep]), f"head {h} {side}: centroids"
        print(f"first iteration: {ties} label ties")
        return
    t = sub.iters - 1
    q_init = np.stack([ref["q_hist"][t] for ref in refs])[None]
    k_init = np.stack([ref["k_hist"][t] for ref in refs])[None]
    O, r = run_gpu(park, sub, Q, K, V, 1, q_init, k_init)
    rep = {}
    fails = pu.compare_retrieval(r, refs, sub.NQ, sub.NK, Q, K, sub.p, rep)
    assert not fails, "\n".join(fails[:20])
    if rep["cascaded_heads"] == 0:
        check_bound(r, refs)
        check_counters(r, refs)
        check_sampled_outputs(O, sub, Q, K, V, refs, seed=1)
