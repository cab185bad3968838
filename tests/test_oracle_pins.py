"""Pins for the float64 oracle: checks against closed forms, library routines,
brute force on tiny inputs and the invariants the PARK pages fix.  CPU only."""
import itertools
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import park_oracle as po
from synth import CONFIGS, gen_layer
from synth.generator import gen_integer_blobs

GOLDEN = __import__("os").path.join(__import__("os").path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(f"{GOLDEN}/{name}") as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            rows.append(line.split())
    return rows


# --------------------------------------------------------------------------- rounding


def test_round_bf16_matches_torch_on_f32_values():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 8, 20000),
                        rng.standard_normal(2000) * 2.0 ** -127,      # bf16 subnormals: fixed ulp 2^-133
                        [0.0, -0.0, 1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 2.0 ** -130]]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = po.round_to_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_round_bf16_direct_not_via_f32():
    # 1 + 2^-8 + 2^-40 lies above the bf16 tie point 1 + 2^-8: direct rounding
    # goes up; rounding to float32 first would land on the tie and go to even (1.0).
    x = 1.0 + 2.0 ** -8 + 2.0 ** -40
    assert po.round_to_bf16(np.array([x]))[0] == 1.0 + 2.0 ** -7
    assert po.round_to_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0          # tie -> even
    assert po.round_to_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2 * 2.0 ** -7


def test_round_f32():
    x = np.array([1.0 + 2.0 ** -24, 1.0 + 3 * 2.0 ** -24, 0.1])
    assert list(po.round_to(x, "f32")) == [1.0, 1.0 + 2.0 ** -22, float(np.float32(0.1))]


# --------------------------------------------------------------------------- exact mean


@pytest.mark.parametrize("seed", range(5))
def test_exact_mean_against_fractions(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 300))
    rows = po.round_to_bf16(rng.standard_normal((n, 6)) * 2.0 ** rng.integers(-18, 12, (n, 6)))
    for dtype in ("bf16", "f32", None):
        got = po.exact_mean(rows, dtype)
        want = [float(sum((Fraction(v) for v in rows[:, j]), Fraction(0))) / n for j in range(6)]
        assert np.array_equal(got, po.round_to(np.array(want), dtype))


def test_exact_mean_cancellation():
    # naive float64 summation loses the 1.0 here; the exact sum keeps it
    rows = np.array([[2.0 ** 60], [1.0], [-(2.0 ** 60)]])
    assert po.exact_mean(rows, None)[0] == 1.0 / 3.0


# --------------------------------------------------------------------------- metric


def test_metric_is_mean_squared_qk_difference():
    rng = np.random.default_rng(3)
    Q = rng.standard_normal((500, 16))
    k, c = rng.standard_normal(16), rng.standard_normal(16)
    M = po.metric(Q)
    lhs = (k - c) @ M @ (k - c)
    rhs = np.mean((Q @ k - Q @ c) ** 2)
    assert abs(lhs - rhs) <= 1e-12 * rhs
    # and the transformed-key distance is the same quadratic form
    D = po.distances(k[None], c[None], M)[0, 0]
    assert abs(D - rhs) <= 1e-12 * rhs


def test_metric_distance_matches_quadratic_form():
    rng = np.random.default_rng(4)
    Q = rng.standard_normal((300, 8)) * np.array([5, 1, 1, 0.1, 2, 3, 1, 1])
    X, C = rng.standard_normal((40, 8)), rng.standard_normal((7, 8))
    M = po.metric(Q)
    D = po.distances(X, C, M)
    U = X[:, None, :] - C[None, :, :]
    want = np.einsum("ika,ab,ikb->ik", U, M, U)
    assert np.allclose(D, want, rtol=1e-12, atol=0)


def test_qrkc_identity_and_power_of_two_scaling():
    X = gen_integer_blobs(64, 5, 4, seed=7)
    lab_e, C_e = po.kmeans(X, 4, 5, None, None)
    lab_i, C_i = po.kmeans(X, 4, 5, np.eye(5), None)
    lab_4, C_4 = po.kmeans(X, 4, 5, 4.0 * np.eye(5), None)
    assert np.array_equal(lab_e, lab_i) and np.array_equal(C_e, C_i)
    assert np.array_equal(lab_e, lab_4) and np.array_equal(C_e, C_4)
    Dx = po.distances(X, C_e, None)
    assert np.array_equal(po.distances(X, C_e, np.eye(5)), Dx)
    assert np.array_equal(po.distances(X, C_e, 4.0 * np.eye(5)), 4.0 * Dx)


def test_qrkc_changes_clustering_when_metric_is_anisotropic():
    # Queries live along axis 0 only: the QK score ignores axis 1, so QRKC must
    # group keys by their axis-0 coordinate even when axis 1 separates them more.
    Q = np.zeros((10, 2))
    Q[:, 0] = np.arange(1, 11)
    K = np.array([[0, 0], [0, 100], [10, 0], [10, 100]], dtype=np.float64)
    lab_q, _ = po.kmeans(K, 2, 3, po.metric(Q), None, init=K[[0, 1]])
    lab_e, _ = po.kmeans(K, 2, 3, None, None, init=K[[0, 1]])
    assert lab_e.tolist() == [0, 1, 0, 1]        # Euclidean: split along axis 1
    assert lab_q.tolist() == [0, 0, 1, 1] or lab_q.tolist() == [1, 1, 0, 0]


def test_retrieval_clusters_queries_euclidean_and_keys_under_the_query_metric():
    # PARK Figure 2 caption: standard K-means on the queries, the query-derived metric
    # on the keys.  Anisotropic inputs on which the two metrics give different
    # clusterings on both sides, so swapping or dropping the metric is visible.
    rng = np.random.default_rng(4)
    Q = rng.standard_normal((40, 4)) * np.array([20, 1, 1, 1])
    K = rng.standard_normal((40, 4)) * np.array([1, 1, 5, 1])
    M = po.metric(Q)
    qe, _ = po.kmeans(Q, 4, 3, None, None)
    ke, _ = po.kmeans(K, 4, 3, None, None)
    km, _ = po.kmeans(K, 4, 3, M, None)
    assert (qe != po.kmeans(Q, 4, 3, M, None)[0]).any() and (ke != km).any()
    r = po.retrieve_head(Q, K, 4, 4, 0.9, 3, None)
    assert np.array_equal(r["q_labels"], qe) and np.array_equal(r["k_labels"], km)
    assert np.array_equal(po.retrieve_head(Q, K, 4, 4, 0.9, 3, None, qrkc=False)["k_labels"], ke)


# --------------------------------------------------------------------------- K-means brute force


def _brute_min(X, K):
    best = math.inf
    for lab in itertools.product(range(K), repeat=X.shape[0]):
        lab = np.array(lab)
        obj = 0.0
        for k in range(K):
            pts = X[lab == k]
            if len(pts):
                obj += float(np.sum((pts - pts.mean(0)) ** 2))
        best = min(best, obj)
    return best


@pytest.mark.parametrize("seed", range(6))
def test_kmeans_bruteforce_tiny(seed):
    n, K = 8 + seed % 3, 2 + seed % 2
    X = gen_integer_blobs(n, 2, K, seed=seed, spread=1)
    labels, C, hist = po.kmeans(X, K, 12, None, None, history=True)
    # Lloyd fixed point: re-assigning and re-averaging changes nothing
    assert np.array_equal(po.assign(X, C), labels)
    assert np.array_equal(po.update(X, labels, C, None), C)
    # objective never below the global minimum over all K^n labelings
    best = _brute_min(X, K)
    obj = po.objective(X, labels, C)
    assert obj >= best - 1e-9
    # objective non-increasing over iterations (unrounded centroids)
    objs = []
    for Ct in hist[1:] + [C]:
        lab_t = po.assign(X, Ct)
        objs.append(po.objective(X, lab_t, Ct))
    assert all(objs[i + 1] <= objs[i] + 1e-9 for i in range(len(objs) - 1))


def test_kmeans_well_separated_reaches_global_minimum():
    X = np.array([[0, 0], [1, 0], [0, 1], [50, 50], [51, 50], [50, 51], [-40, 60], [-41, 60], [-40, 61]],
                 dtype=np.float64)
    labels, C = po.kmeans(X, 3, 10, None, None)
    assert abs(po.objective(X, labels, C) - _brute_min(X, 3)) < 1e-9


def test_kmeans_worked_example_1d():
    # x = 0, 1, 10, 11 ; K = 2 ; strided init picks x0 = 0 and x2 = 10.
    # assign: {0, 1} -> 0, {10, 11} -> 1 ; update: c = 0.5, 10.5 ; stable after.
    X = np.array([[0.0], [1.0], [10.0], [11.0]])
    labels, C = po.kmeans(X, 2, 3, None, None)
    assert labels.tolist() == [0, 0, 1, 1]
    assert C[:, 0].tolist() == [0.5, 10.5]


def test_kmeans_exact_tie_goes_to_lowest_index():
    X = np.array([[0.0, 0.0], [2.0, 0.0], [1.0, 0.0]])   # x2 equidistant from c0 = x0 and c1 = x1
    C = X[:2]
    assert po.assign(X, C).tolist() == [0, 1, 0]
    # with the centroids swapped the tie still goes to index 0
    assert po.assign(X, C[::-1]).tolist() == [1, 0, 0]


def test_empty_cluster_keeps_previous_centroid():
    X = np.array([[0.0], [0.5], [1.0]])
    C = np.array([[0.5], [100.0]])
    labels = po.assign(X, C)
    assert labels.tolist() == [0, 0, 0]
    C2 = po.update(X, labels, C, None)
    assert C2[1, 0] == 100.0 and C2[0, 0] == 0.5


def test_strided_init_and_bf16_centroids():
    cfg = CONFIGS["small"]
    Q, _, _ = gen_layer(cfg)
    X = Q[0, 0].astype(np.float64)
    C0 = po.strided_init(X, 7)
    assert np.array_equal(C0, X[[0, 292, 585, 877, 1170, 1462, 1755]])
    _, C = po.kmeans(X, 7, 2, None, "bf16")
    assert np.array_equal(po.round_to_bf16(C), C)


# --------------------------------------------------------------------------- permutation


def test_stable_permutation_matches_numpy_argsort():
    rng = np.random.default_rng(5)
    lab = rng.integers(0, 17, 1000)
    lab[lab == 3] = 4                         # an empty cluster
    perm, off = po.stable_permutation(lab, 17)
    assert np.array_equal(perm, np.argsort(lab, kind="stable"))
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(lab, minlength=17))]))


# --------------------------------------------------------------------------- PAMA / top-p


def _tiny_case(seed=0, N=48, d=8, NQ=5, NK=6):
    rng = np.random.default_rng(seed)
    Q, K, V = (rng.standard_normal((N, d)) for _ in range(3))
    ql, CQ = po.kmeans(Q, NQ, 3, None, None)
    kl, CK = po.kmeans(K, NK, 3, po.metric(Q), None)
    return Q, K, V, ql, CQ, kl, CK


def test_pama_against_per_query_loop():
    Q, K, V, ql, CQ, kl, CK = _tiny_case()
    NQ, NK = CQ.shape[0], CK.shape[0]
    kc = np.bincount(kl, minlength=NK)
    s = 1 / math.sqrt(Q.shape[1])
    I = po.pama(Q, ql, NQ, CK, kc, s)
    want = np.zeros((NQ, NK))
    for r in range(NQ):
        members = [i for i in range(Q.shape[0]) if ql[i] == r]
        for i in members:
            z = [s * sum(Q[i, j] * CK[m, j] for j in range(Q.shape[1])) for m in range(NK) if kc[m]]
            zmax = max(z)
            e = [math.exp(v - zmax) for v in z]
            tot = sum(e)
            live = [m for m in range(NK) if kc[m]]
            for t, m in enumerate(live):
                want[r, m] += e[t] / tot / len(members)
    assert np.allclose(I, want, rtol=1e-12, atol=1e-15)
    qc = np.bincount(ql, minlength=NQ)
    assert np.allclose(I[qc > 0].sum(1), 1.0, atol=1e-12)


def test_pama_ignores_empty_key_clusters():
    # an empty key cluster stands for no keys (PAMA over non-empty clusters only): its
    # column is 0, and its centroid, however strongly it would score, changes nothing
    Q, K, V, ql, CQ, kl, CK = _tiny_case(seed=3)
    NQ, NK = CQ.shape[0], CK.shape[0]
    kc = np.bincount(kl, minlength=NK)
    kc[2] = 0
    s = 1 / math.sqrt(Q.shape[1])
    I = po.pama(Q, ql, NQ, CK, kc, s)
    CK2 = CK.copy()
    CK2[2] = 50.0 * Q.mean(axis=0)
    I2 = po.pama(Q, ql, NQ, CK2, kc, s)
    qc = np.bincount(ql, minlength=NQ)
    assert np.all(I[:, 2] == 0.0) and np.array_equal(I, I2)
    assert np.allclose(I[qc > 0].sum(1), 1.0, atol=1e-12)


def test_identity_clustering_gives_exact_attention_mass():
    rng = np.random.default_rng(8)
    N, d = 24, 8
    Q, K, V = (rng.standard_normal((N, d)) for _ in range(3))
    s = 1 / math.sqrt(d)
    res = po.layer_head(Q, K, V, N, N, 1.0, 2, None)
    assert res["q_labels"].tolist() == list(range(N)) and res["k_labels"].tolist() == list(range(N))
    S = s * Q @ K.T
    A = np.exp(S - S.max(1, keepdims=True))
    A /= A.sum(1, keepdims=True)
    assert np.allclose(res["importance"], A, rtol=1e-12, atol=1e-15)
    assert np.allclose(res["O"], po.dense_attention(Q, K, V, s), rtol=0, atol=1e-12)


def test_all_blocks_kept_equals_dense_and_torch_sdpa():
    Q, K, V, ql, CQ, kl, CK = _tiny_case(seed=2)
    s = 1 / math.sqrt(Q.shape[1])
    mask = np.ones((CQ.shape[0], CK.shape[0]), dtype=bool)
    O = po.sparse_attention(Q, K, V, ql, kl, mask, s)
    O_dense = po.dense_attention(Q, K, V, s)
    t = [torch.from_numpy(a)[None, None] for a in (Q, K, V)]
    O_sdpa = torch.nn.functional.scaled_dot_product_attention(*t, scale=s)[0, 0].numpy()
    assert np.allclose(O, O_dense, rtol=0, atol=1e-12)
    assert np.allclose(O, O_sdpa, rtol=0, atol=1e-12)


def test_sparse_attention_against_per_query_loop():
    Q, K, V, ql, CQ, kl, CK = _tiny_case(seed=3)
    s = 1 / math.sqrt(Q.shape[1])
    rng = np.random.default_rng(0)
    mask = rng.random((CQ.shape[0], CK.shape[0])) < 0.4
    mask[np.arange(CQ.shape[0]), np.bincount(kl).argmax()] = True
    O = po.sparse_attention(Q, K, V, ql, kl, mask, s)
    for i in range(Q.shape[0]):
        js = [j for j in range(K.shape[0]) if mask[ql[i], kl[j]]]
        w = [math.exp(s * float(Q[i] @ K[j])) for j in js]
        want = sum(wt * V[j] for wt, j in zip(w, js)) / sum(w)
        assert np.allclose(O[i], want, rtol=1e-12, atol=1e-12)
    rows = np.array([5, 0, 17])
    assert np.allclose(po.sparse_attention(Q, K, V, ql, kl, mask, s, rows=rows), O[rows], rtol=0, atol=1e-14)


def test_top_p_rules():
    qc, kc = np.array([1, 1, 0, 1]), np.array([1, 1, 1, 0, 1])
    I = np.array([[0.1, 0.4, 0.4, 0.0, 0.1],      # tie 0.4/0.4: m=1 before m=2
                  [0.5, 0.25, 0.25, 0.0, 0.0],    # cumsum hits p = 0.75 exactly at m=1: crossing kept, stop
                  [0.2, 0.2, 0.2, 0.0, 0.4],      # empty query cluster: keeps nothing
                  [0.0, 0.0, 0.0, 0.0, 1.0]])
    m = po.top_p(I, 0.75, qc, kc)
    assert m[0].tolist() == [False, True, True, False, False]
    assert m[1].tolist() == [True, True, False, False, False]
    assert not m[2].any()
    assert m[3].tolist() == [False, False, False, False, True]
    m1 = po.top_p(I, 0.5, qc, kc)
    assert m1[0].tolist() == [False, True, True, False, False]   # 0.4 < 0.5: needs the tied second
    assert m1[1].tolist() == [True, False, False, False, False]  # 0.5 >= 0.5 with one block
    mall = po.top_p(I, 1.0, qc, kc)
    assert mall[0].tolist() == [True, True, True, False, True]
    # p = 1 keeps every non-empty block even when the running sum reaches 1 early
    assert po.top_p(np.array([[0.5, 0.5, 1e-20]]), 1.0, np.array([1]), np.array([1, 1, 1]))[0].all()
    # tiny p keeps exactly one block
    assert po.top_p(I, 1e-9, qc, kc).sum(1).tolist() == [1, 1, 0, 1]


def test_top_p_on_exact_mass_gives_recall_at_least_p():
    # PARK Table 1, Full/Full rows: worst-case recall >= 90.01 at p = 0.9.
    rows = _read_golden("park_table1_full_full.txt")
    assert all(float(r[3]) >= 90.0 for r in rows)
    cfg = CONFIGS["small"]
    Q, K, _ = gen_layer(cfg)
    s = 1 / math.sqrt(cfg.D)
    recalls = []
    for h in range(3):
        q, k = Q[0, h].astype(np.float64), K[0, h].astype(np.float64)
        ql, _ = po.kmeans(q, cfg.NQ, 3, None, "bf16")
        kl, _ = po.kmeans(k, cfg.NK, 3, po.metric(q), "bf16")
        I, _ = po.exact_block_mass(q, k, ql, cfg.NQ, kl, cfg.NK, s)
        mask = po.top_p(I, cfg.p, np.bincount(ql, minlength=cfg.NQ), np.bincount(kl, minlength=cfg.NK))
        recalls.append(po.block_recall(q, k, ql, kl, mask, s))
    assert min(recalls) >= cfg.p


def test_full_full_tv_is_zero():
    # PARK Appendix Table 4: Full query / full key has zero TV by definition.
    assert all(float(r[1]) == 0.0 for r in _read_golden("park_table4_full_full.txt"))
    rng = np.random.default_rng(9)
    Q, K = rng.standard_normal((20, 8)), rng.standard_normal((20, 8))
    tv = po.attention_tv(Q, K, np.arange(20), 20, K, 1 / math.sqrt(8))
    assert tv < 1e-12
    # and a real key clustering has a positive TV
    kl, CK = po.kmeans(K, 4, 3, None, None)
    assert po.attention_tv(Q, K, kl, 4, CK, 1 / math.sqrt(8)) > 1e-3


def test_recall_and_tv_hand_cases():
    # one query, two single-key clusters with equal scores: the dense attention is
    # (1/2, 1/2), so keeping one block recalls 1/2 and keeping both recalls 1
    Q, K = np.array([[1.0]]), np.array([[0.0], [0.0]])
    kl = np.array([0, 1])
    assert po.block_recall(Q, K, np.array([0]), kl, np.array([[True, False]]), 1.0) == 0.5
    assert po.block_recall(Q, K, np.array([0]), kl, np.array([[True, True]]), 1.0) == 1.0
    # centroids scoring ln 3 and 0 give P = (3/4, 1/4) against the block mass (1/2, 1/2):
    # total variation (1/2)(1/4 + 1/4) = 1/4
    CK = np.array([[math.log(3.0)], [0.0]])
    assert abs(po.attention_tv(Q, K, kl, 2, CK, 1.0) - 0.25) < 1e-15


def test_centroid_query_ablation_is_softmax_of_centroid():
    Q, K, V, ql, CQ, kl, CK = _tiny_case(seed=4)
    s = 1 / math.sqrt(Q.shape[1])
    qc, kc = np.bincount(ql, minlength=CQ.shape[0]), np.bincount(kl, minlength=CK.shape[0])
    I = po.pama_centroid_query(CQ, qc, CK, kc, s)
    r = int(np.argmax(qc))
    z = np.array([s * CQ[r] @ CK[m] for m in range(CK.shape[0])])
    e = np.exp(z - z.max()) * (kc > 0)
    assert np.allclose(I[r], e / e.sum(), rtol=1e-12, atol=1e-15)


def test_top_k_ratio():
    I = np.array([[0.1, 0.3, 0.2, 0.4]])
    m = po.top_k_ratio(I, 0.5, np.array([1]), np.array([1, 1, 1, 1]))
    assert m[0].tolist() == [False, True, False, True]
    # ties go to the lower index: k = 1 of two equal leaders, k = 3 of two equal last ones
    I = np.array([[0.2, 0.3, 0.3, 0.2]])
    assert po.top_k_ratio(I, 0.25, np.array([1]), np.ones(4, int))[0].tolist() == [False, True, False, False]
    assert po.top_k_ratio(I, 0.75, np.array([1]), np.ones(4, int))[0].tolist() == [True, True, True, False]


def test_size_prior_pama_is_exact_block_mass_for_tight_clusters():
    # Every key of cluster m equal to its centroid: the attention mass of block m
    # is |B_m| exp(s q.c_m) / sum_m' |B_m'| exp(s q.c_m'), which the size-weighted
    # PAMA must reproduce through the independently pinned exact block mass.
    rng = np.random.default_rng(11)
    d, NK = 8, 5
    protos = np.round(rng.standard_normal((NK, d)) * 4) / 4
    sizes = np.array([1, 3, 7, 2, 5])
    K = np.repeat(protos, sizes, axis=0)
    k_labels = np.repeat(np.arange(NK), sizes)
    Q = np.round(rng.standard_normal((12, d)) * 4) / 4
    q_labels = np.arange(12) % 3
    s = 1 / math.sqrt(d)
    I = po.pama(Q, q_labels, 3, protos, sizes, s, size_prior=True)
    A, _ = po.exact_block_mass(Q, K, q_labels, 3, k_labels, NK, s)
    assert np.allclose(I, A, rtol=1e-12, atol=1e-15)
    # without the prior the unequal sizes make it differ
    assert not np.allclose(po.pama(Q, q_labels, 3, protos, sizes, s), A, rtol=1e-3)


def test_size_prior_with_equal_sizes_changes_nothing():
    Q, K, V, ql, CQ, kl, CK = _tiny_case(seed=12)
    s = 1 / math.sqrt(Q.shape[1])
    counts = np.where(np.bincount(kl, minlength=CK.shape[0]) > 0, 6, 0)
    a = po.pama(Q, ql, CQ.shape[0], CK, counts, s)
    b = po.pama(Q, ql, CQ.shape[0], CK, counts, s, size_prior=True)
    assert np.allclose(a, b, rtol=1e-13, atol=1e-16)


def test_retrieve_topk_keeps_ceil_ratio_blocks():
    rng = np.random.default_rng(13)
    Q, K = rng.standard_normal((96, 16)), rng.standard_normal((96, 16))
    r = po.retrieve_head(Q, K, 6, 10, 0.9, 3, "bf16", topk_ratio=0.25)
    live = int((r["k_counts"] > 0).sum())
    k = max(1, math.ceil(0.25 * live))
    for q in range(6):
        if r["q_counts"][q] == 0:
            assert not r["mask"][q].any()
            continue
        kept = np.nonzero(r["mask"][q])[0]
        assert kept.size == k
        # every kept block is at least as important as every dropped live block
        dropped = [m for m in range(10) if r["k_counts"][m] > 0 and not r["mask"][q, m]]
        if dropped:
            assert r["importance"][q, kept].min() >= r["importance"][q, dropped].max()


def test_sip_probabilities_worked_examples():
    # budget 2 over [0.5, 0.3, 0.1, 0.1]: c = 2, nothing capped (c * 0.5 = 1)
    assert np.allclose(po.sip_probabilities([0.5, 0.3, 0.1, 0.1], 2), [1.0, 0.6, 0.2, 0.2], rtol=1e-15)
    # budget 2 over [0.7, 0.1, 0.1, 0.1]: 0.7 is certain, the rest share 1 -> 1/3 each
    assert np.allclose(po.sip_probabilities([0.7, 0.1, 0.1, 0.1], 2), [1.0, 1 / 3, 1 / 3, 1 / 3], rtol=1e-15)
    # budget >= count: everything is certain
    assert np.array_equal(po.sip_probabilities([0.2, 0.8], 2), [1.0, 1.0])


def test_sip_probabilities_sum_to_budget_and_are_proportional():
    rng = np.random.default_rng(14)
    for _ in range(50):
        L = int(rng.integers(2, 40))
        v = rng.random(L) ** 4 + 1e-6
        B = int(rng.integers(1, L))
        pi = po.sip_probabilities(v, B)
        assert abs(pi.sum() - B) < 1e-12 * B
        assert np.all(pi > 0) and np.all(pi <= 1.0)
        free = pi < 1.0
        if free.sum() > 1:
            ratio = pi[free] / v[free]
            assert np.allclose(ratio, ratio[0], rtol=1e-12)
        # certain blocks are the largest ones
        if (~free).any() and free.any():
            assert v[~free].min() >= v[free].max()


def test_sip_weighting_is_unbiased_by_enumeration():
    # E over independent draws of sum_{m drawn} X_m / pi_m equals sum_m X_m: enumerate
    # every inclusion pattern with its probability (a wrong weight, e.g. 1/pi^2, fails)
    rng = np.random.default_rng(15)
    v = rng.random(6) + 0.05
    X = rng.random(6)
    pi = po.sip_probabilities(v, 3)
    expect = 0.0
    for pattern in itertools.product([0, 1], repeat=6):
        prob = np.prod([p if z else 1 - p for z, p in zip(pattern, pi)])
        expect += prob * sum(X[m] / pi[m] for m in range(6) if pattern[m])
    assert abs(expect - X.sum()) < 1e-12


def test_sip_select_inclusion_thresholds_and_weights():
    # Block m is drawn exactly when its uniform lies below pi_m, so pi_m is the
    # threshold at which a constant uniform stops drawing m; found by bisection on
    # sip_select alone.  The thresholds must add up to the expected budget
    # ceil(0.3 * 7) = 3 (a fractional ratio * L), and every drawn block must carry
    # the inverse of its threshold as its weight.
    I = np.array([[0.5, 0.1, 0.1, 0.08, 0.07, 0.1, 0.05]])
    qc, kc = np.array([4]), np.ones(7, dtype=np.int64)

    def drawn(c):
        mask, w = po.sip_select(I, 0.3, np.full(I.shape, c), qc, kc)
        return mask[0], w[0]

    thr = np.zeros(7)
    for m in range(7):
        lo, hi = 0.0, 1.0
        for _ in range(60):
            mid = 0.5 * (lo + hi)
            if drawn(mid)[0][m]:
                lo = mid
            else:
                hi = mid
        thr[m] = lo
    assert abs(thr.sum() - 3.0) < 1e-9
    assert abs(thr[0] - 1.0) < 1e-12                        # the dominant block is certain
    assert np.allclose(thr[1:] / I[0, 1:], thr[1] / I[0, 1], rtol=1e-9)   # the rest in proportion
    for m in range(1, 7):
        mask, w = drawn(thr[m] * (1 - 1e-9))
        assert mask[m] and abs(w[m] * thr[m] - 1.0) < 1e-6


def test_integer_block_weights_equal_duplicated_keys():
    # A key block with weight n in both Softmax sums acts as if its keys were
    # present n times: the weighted sparse attention of one query cluster equals
    # plain attention over the kept keys, each repeated by its block's weight.
    Q, K, V, ql, CQ, kl, CK = _tiny_case(seed=17)
    NQ, NK = CQ.shape[0], CK.shape[0]
    s = 1 / math.sqrt(Q.shape[1])
    rng = np.random.default_rng(17)
    mask = rng.random((NQ, NK)) < 0.7
    mask[:, 0] = True
    weight = np.where(mask, rng.integers(1, 4, size=(NQ, NK)).astype(np.float64), 0.0)
    O = po.sparse_attention(Q, K, V, ql, kl, mask, s, weight=weight)
    for r in np.unique(ql):
        rows = np.nonzero(ql == r)[0]
        keys = [j for j in range(K.shape[0]) if mask[r, kl[j]] for _ in range(int(weight[r, kl[j]]))]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(Q[rows])[None], torch.from_numpy(K[keys])[None], torch.from_numpy(V[keys])[None],
            scale=s)[0].numpy()
        assert np.allclose(O[rows], ref, rtol=1e-10, atol=1e-12)


def test_sip_select_full_budget_is_dense_and_empty_draw_keeps_best():
    Q, K, V, ql, CQ, kl, CK = _tiny_case(seed=16)
    s = 1 / math.sqrt(Q.shape[1])
    qc, kc = np.bincount(ql, minlength=CQ.shape[0]), np.bincount(kl, minlength=CK.shape[0])
    I = po.pama(Q, ql, CQ.shape[0], CK, kc, s)
    u = np.random.default_rng(16).random(I.shape)
    mask, w = po.sip_select(I, 1.0, u, qc, kc)       # budget = every live block: all certain
    assert np.array_equal(mask, (qc[:, None] > 0) & (kc[None, :] > 0))
    assert np.all(w[mask] == 1.0)
    O = po.sparse_attention(Q, K, V, ql, kl, mask, s, weight=w)
    assert np.allclose(O, po.dense_attention(Q, K, V, s), rtol=1e-12, atol=1e-12)
    # uniforms that draw nothing: the most important block is kept alone
    mask, w = po.sip_select(I, 0.1, np.full(I.shape, 0.999999), qc, kc)
    for r in np.nonzero(qc)[0]:
        live = np.nonzero(kc)[0]
        best = live[np.argmax(I[r, live])]
        assert mask[r].sum() == 1 and mask[r, best] and w[r, best] >= 1.0


def test_qrkc_trades_raw_key_error_for_qk_score_error():
    # PARK Appendix Table 5: clustering the keys under the query-derived metric lowers
    # the QK-score squared error and raises the raw-key MSE against Euclidean K-means
    # (there -36.6 % / -22.8 % and +8.5 % / +14.8 % on real activations).  A direction
    # check on every head of the small synthetic layer.
    from synth.generator import gen_tensor
    cfg = CONFIGS["small"]
    Q, K = (gen_tensor(cfg, t).astype(np.float64)[0] for t in "QK")
    for h in range(cfg.H):
        M = po.metric(Q[h])
        le, Ce = po.kmeans(K[h], cfg.NK, cfg.iters, None, cfg.dtype)
        lm, Cm = po.kmeans(K[h], cfg.NK, cfg.iters, M, cfg.dtype)
        raw_e, qk_e = po.key_errors(Q[h], K[h], le, Ce)
        raw_m, qk_m = po.key_errors(Q[h], K[h], lm, Cm)
        print(f"head {h}: raw-key MSE {100 * (raw_m / raw_e - 1):+.1f} %, QK-score error {100 * (qk_m / qk_e - 1):+.1f} %")
        assert qk_m < qk_e and raw_m > raw_e


def test_key_errors_qk_term_is_metric_distance():
    rng = np.random.default_rng(10)
    Q, K = rng.standard_normal((64, 8)), rng.standard_normal((50, 8))
    kl, CK = po.kmeans(K, 5, 3, po.metric(Q), None)
    raw, qk = po.key_errors(Q, K, kl, CK)
    D = po.distances(K, CK, po.metric(Q))[np.arange(50), kl]
    assert abs(qk - D.mean()) <= 1e-12 * qk
    Deu = po.distances(K, CK, None)[np.arange(50), kl]
    assert abs(raw - Deu.mean()) <= 1e-12 * raw


def test_c_assign_is_the_distance_argmin():
    """The oracle's C assign loop equals the argmin of the written-out distance
    matrix: on integer inputs (exact sums, real ties resolved to the lowest
    index) bit for bit, with and without a metric; on random floats up to
    rounding-order near-ties, of which there are none here."""
    rng = np.random.default_rng(5)
    for trial in range(30):
        N, K, D = int(rng.integers(1, 200)), int(rng.integers(1, 23)), int(rng.integers(1, 40))
        X = rng.integers(-2, 3, size=(N, D)).astype(float)
        C = rng.integers(-2, 3, size=(K, D)).astype(float)
        D_ = po.distances(X, C)
        want = np.array([min(range(K), key=lambda k: (D_[i, k], k)) for i in range(N)])
        assert np.array_equal(po.assign(X, C), want), trial
    X = rng.standard_normal((3000, 64))
    C = rng.standard_normal((70, 64))
    M = po.metric(rng.standard_normal((400, 64)))
    assert np.array_equal(po.assign(X, C), np.argmin(po.distances(X, C), axis=1))
    assert np.array_equal(po.assign(X, C, M), np.argmin(po.distances(X, C, M), axis=1))
