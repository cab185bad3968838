"""PARK oracle: a plain, slow, float64 CPU statement of what the hot path computes.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import this module:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code with the
CUDA library; the only module both sides import is ``synth`` (seeded inputs).

Source: "PARK: Accurate Block Retrieval for Sparse Attention in Video Diffusion
Transformers" (abstract, AI summary, Figure 1 and Figure 2 captions, Table 1
caption).  The pages give no equations; every step below is the plainest reading
of their words, and each reading that fills a gap is marked READING.

Notation, per (batch b, head h): Q, K, V in R^{N x d}; s = 1/sqrt(d); query
clusters r = 0..NQ-1, key clusters m = 0..NK-1.  All arithmetic is float64.
Values that the method stores in the input dtype (centroids) are rounded once,
round-to-nearest-even, from float64.
"""
from __future__ import annotations

import math

import numpy as np

# ----------------------------------------------------------------------------
# rounding to the storage dtype
# ----------------------------------------------------------------------------


def round_to_bf16(x):
    """Nearest bf16 (8 significant bits, ties to even) of float64 values, taken
    directly from float64 (no intermediate float32)."""
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)                      # |x| in [2^(e-1), 2^e)
    e = np.maximum(e, -125)                 # below 2^-126 the bf16 ulp is fixed at 2^-133
    return np.ldexp(np.rint(np.ldexp(x, 8 - e)), e - 8)


def round_to(x, dtype):
    """Round float64 values to the storage dtype ("bf16", "f32", or None = keep)."""
    if dtype is None:
        return np.asarray(x, dtype=np.float64)
    if dtype == "bf16":
        return round_to_bf16(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


# ----------------------------------------------------------------------------
# QRKC metric
# ----------------------------------------------------------------------------


def metric(Q):
    """M = (1/N) sum_i q_i q_i^T, the queries' second-moment matrix.

    READING of PARK's Figure 2 caption, where the keys are clustered under a
    metric computed from this layer's queries, which should put keys that get
    alike scores from those queries in one cluster: for any key k and centroid c,
    (k - c)^T M (k - c) = mean_i (q_i.k - q_i.c)^2, the mean squared QK-score
    difference under the current queries, which is what the pages want small
    inside a key cluster.  A library matmul forms the sum."""
    Q = np.asarray(Q, dtype=np.float64)
    return (Q.T @ Q) / Q.shape[0]


class QueryMetric:
    """The QRKC metric of a set of queries, M = Q^T Q / N, together with a
    factor F = R^T / sqrt(N) from the QR decomposition Q = Q_1 R (so that
    M = F F^T): keys are transformed by F^T before clustering, as the pages put
    it (PARK abstract).  Taking F from the queries themselves keeps every
    direction in which the queries are small; a factor of M from its
    eigendecomposition loses the directions whose eigenvalues fall below
    float64 rounding of the largest one, which inputs spanning many binades
    reach."""

    def __init__(self, Q):
        Q = np.asarray(Q, dtype=np.float64)
        self.M = metric(Q)
        R = np.linalg.qr(Q, mode="r")
        self.F = R.T / math.sqrt(Q.shape[0])


def metric_factor(M):
    """F with M = F F^T, so that (x - c)^T M (x - c) = ||F^T x - F^T c||^2.
    A QueryMetric carries its own factor; a plain matrix M is factored by its
    eigendecomposition (clipped at 0 for a PSD M)."""
    if isinstance(M, QueryMetric):
        return M.F
    lam, V = np.linalg.eigh(np.asarray(M, dtype=np.float64))
    return V * np.sqrt(np.clip(lam, 0.0, None))


# ----------------------------------------------------------------------------
# K-means (queries: Euclidean; keys: QRKC)
# ----------------------------------------------------------------------------


def strided_init(X, K):
    """READING (pages silent on initialisation): c_k = x_floor(k N / K)."""
    N = X.shape[0]
    return np.asarray(X, dtype=np.float64)[(np.arange(K) * N) // K].copy()


def distances(X, C, M=None, row_block=4096):
    """D[i, k] = (x_i - c_k)^T M (x_i - c_k); M = None means the identity
    (standard Euclidean K-means, PARK Figure 2 caption).  For a metric (a
    matrix or a QueryMetric) the keys and centroids are first transformed by
    F^T with M = F F^T."""
    X = np.asarray(X, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    if M is not None:
        F = metric_factor(M)
        X = X @ F
        C = C @ F
    D = np.empty((X.shape[0], C.shape[0]))
    for i0 in range(0, X.shape[0], row_block):
        diff = X[i0:i0 + row_block, None, :] - C[None, :, :]
        D[i0:i0 + row_block] = np.sum(diff * diff, axis=2)
    return D


_CLIB = None


def _clib():
    """The oracle's C part (oracle/assign.c), compiled on first use."""
    global _CLIB
    if _CLIB is None:
        import ctypes
        from . import build_oracle
        lib = ctypes.CDLL(build_oracle.build())
        lib.oracle_assign.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_int64, ctypes.c_void_p]
        lib.oracle_assign.restype = None
        _CLIB = lib
    return _CLIB


def assign(X, C, M=None):
    """a(i) = argmin_k D(x_i, c_k); ties go to the lowest k (READING).

    The same distances as `distances` (rows and centroids transformed by F^T
    for a metric, then sum_j (x_j - c_j)^2), each summed in j order by the C
    loop in assign.c, which keeps full-size heads within seconds."""
    X = np.asarray(X, dtype=np.float64)
    C = np.asarray(C, dtype=np.float64)
    if M is not None:
        F = metric_factor(M)
        X = X @ F
        C = C @ F
    X = np.ascontiguousarray(X)
    C = np.ascontiguousarray(C)
    labels = np.empty(X.shape[0], dtype=np.int64)
    _clib().oracle_assign(X.ctypes.data, C.ctypes.data, X.shape[0], C.shape[0], X.shape[1], labels.ctypes.data)
    return labels


def exact_mean(rows, dtype):
    """Centroid = round_dtype( fl64(exact sum of the rows) / n ).

    The column sums are exact and rounded once to float64 (math.fsum is
    correctly rounded), then divided by n in IEEE float64, then rounded to the
    storage dtype.  READING: the pages only say that a cluster is represented
    by the mean of its members (PARK abstract)."""
    n = rows.shape[0]
    sums = np.array([math.fsum(col) for col in np.asarray(rows, dtype=np.float64).T.tolist()])
    return round_to(sums / float(n), dtype)


def update(X, labels, C_prev, dtype):
    """Centroid update; an empty cluster keeps its previous centroid (READING)."""
    X = np.asarray(X, dtype=np.float64)
    C = np.array(C_prev, dtype=np.float64, copy=True)
    order = np.argsort(labels, kind="stable")
    counts = np.bincount(labels, minlength=C.shape[0])
    start = 0
    for k in range(C.shape[0]):
        n = counts[k]
        if n:
            C[k] = exact_mean(X[order[start:start + n]], dtype)
        start += n
    return C


def kmeans(X, K, iters, M=None, dtype="bf16", init=None, history=False):
    """Lloyd K-means: `iters` x (assign, update), no early stop (READING).

    Returns (labels of the last assign, centroids of the last update) and, with
    history=True, the list of centroids entering each iteration."""
    if iters < 1:
        raise ValueError("iters >= 1")
    C = strided_init(X, K) if init is None else np.array(init, dtype=np.float64, copy=True)
    hist = []
    labels = None
    for _ in range(iters):
        hist.append(C.copy())
        labels = assign(X, C, M)
        C = update(X, labels, C, dtype)
    return (labels, C, hist) if history else (labels, C)


def objective(X, labels, C, M=None):
    """sum_i D(x_i, c_a(i))."""
    D = distances(X, C, M)
    return float(np.sum(D[np.arange(X.shape[0]), labels]))


# ----------------------------------------------------------------------------
# blocks: stable permutation by cluster
# ----------------------------------------------------------------------------


def stable_permutation(labels, K):
    """Counting sort: perm[pos] = original token index, cluster by cluster,
    original order inside a cluster; offsets[k] = first position of cluster k.
    READING: the query/key "blocks" are the clusters (PARK Figure 2)."""
    labels = np.asarray(labels)
    counts = [0] * K
    for a in labels.tolist():
        counts[a] += 1
    offsets = [0] * (K + 1)
    for k in range(K):
        offsets[k + 1] = offsets[k] + counts[k]
    cursor = offsets[:-1].copy()
    perm = [0] * len(labels)
    for i, a in enumerate(labels.tolist()):
        perm[cursor[a]] = i
        cursor[a] += 1
    return np.array(perm, dtype=np.int64), np.array(offsets, dtype=np.int64)


# ----------------------------------------------------------------------------
# PAMA block importance
# ----------------------------------------------------------------------------


def pama(Q, q_labels, NQ, CK, k_counts, scale, row_block=8192, size_prior=False):
    """Block-importance map I[r, m].

    PARK (abstract; Figure 2 caption): every original query keeps its own
    Softmax over the key centroids, and these distributions are averaged within
    each query block:
        P_im = softmax_m(s q_i . c_m),   I_rm = mean_{i in Q_r} P_im.
    READING: only non-empty key clusters take part (an empty cluster stands for
    no keys); rows of empty query clusters are 0.
    size_prior: a variant that is not on the pages, P_im proportional to
    |B_m| exp(s q_i . c_m) (the Softmax with a log |B_m| prior); when every key of
    cluster m equals c_m it is the exact attention mass of the cluster."""
    Q = np.asarray(Q, dtype=np.float64)
    CK = np.asarray(CK, dtype=np.float64)
    live = np.nonzero(np.asarray(k_counts) > 0)[0]
    NK = CK.shape[0]
    sums = np.zeros((NQ, live.size))
    q_labels = np.asarray(q_labels)
    prior = np.log(np.asarray(k_counts, dtype=np.float64)[live]) if size_prior else 0.0
    for i0 in range(0, Q.shape[0], row_block):
        Z = scale * (Q[i0:i0 + row_block] @ CK[live].T) + prior
        Z -= Z.max(axis=1, keepdims=True)
        P = np.exp(Z)
        P /= P.sum(axis=1, keepdims=True)
        np.add.at(sums, q_labels[i0:i0 + row_block], P)
    q_counts = np.bincount(q_labels, minlength=NQ)
    I = np.zeros((NQ, NK))
    nz = q_counts > 0
    I[np.ix_(nz, live)] = sums[nz] / q_counts[nz, None]
    return I


def pama_centroid_query(CQ, q_counts, CK, k_counts, scale, size_prior=False):
    """"w/o PAMA" ablation (PARK Table 3; Figure 1(a)): the query centroid is
    scored instead of every query, i.e. queries are averaged before Softmax:
    I_rm = softmax_m(s c_r^Q . c_m) for non-empty r, m (size_prior as in pama)."""
    live = np.nonzero(np.asarray(k_counts) > 0)[0]
    I = np.zeros((CQ.shape[0], CK.shape[0]))
    prior = np.log(np.asarray(k_counts, dtype=np.float64)[live]) if size_prior else 0.0
    for r in range(CQ.shape[0]):
        if q_counts[r] == 0:
            continue
        z = scale * (np.asarray(CK, dtype=np.float64)[live] @ np.asarray(CQ[r], dtype=np.float64)) + prior
        z -= z.max()
        e = np.exp(z)
        I[r, live] = e / e.sum()
    return I


# ----------------------------------------------------------------------------
# top-p selection
# ----------------------------------------------------------------------------


def top_p(I, p, q_counts, k_counts):
    """Keep, per non-empty query cluster r, the shortest prefix of the key
    clusters sorted by I[r, m] descending (ties: lower m first) whose float64
    running sum reaches p; the crossing block is kept (PARK Table 1 caption:
    top-p block retrieval, p = 0.9).  READING: p >= 1 keeps every non-empty key
    cluster; empty query clusters keep nothing."""
    NQ, NK = I.shape
    mask = np.zeros((NQ, NK), dtype=bool)
    live = [m for m in range(NK) if k_counts[m] > 0]
    for r in range(NQ):
        if q_counts[r] == 0:
            continue
        if p >= 1.0:
            mask[r, live] = True
            continue
        order = sorted(live, key=lambda m: (-I[r, m], m))
        acc = 0.0
        for m in order:
            mask[r, m] = True
            acc += I[r, m]
            if acc >= p:
                break
    return mask


def top_k_ratio(I, rho, q_counts, k_counts):
    """Top-k at a fixed retrieval ratio rho (PARK Table 10): keep the
    ceil(rho * NK_live) most important key clusters (ties: lower m)."""
    NQ, NK = I.shape
    mask = np.zeros((NQ, NK), dtype=bool)
    live = [m for m in range(NK) if k_counts[m] > 0]
    k = max(1, int(math.ceil(rho * len(live))))
    for r in range(NQ):
        if q_counts[r] == 0:
            continue
        order = sorted(live, key=lambda m: (-I[r, m], m))
        mask[r, order[:k]] = True
    return mask


# ----------------------------------------------------------------------------
# sampling with inclusion-probability weighting
# ----------------------------------------------------------------------------


def sip_probabilities(values, budget):
    """Inclusion probabilities proportional to importance, capped at 1, with
    expected sample size `budget` ("AB-Attention Brings More Accurate Sparse
    Attention to Video Diffusion", paragraph on SIP: blocks are sampled according
    to their estimated importance).  READING: pi_m = min(1, c v_m) with c such
    that sum_m pi_m = budget; the blocks whose c v_m would exceed 1 are taken with
    certainty, found in descending order of v (ties: lower index first).
    values: importances of the candidate blocks (> 0); returns pi in their order."""
    v = np.asarray(values, dtype=np.float64)
    L = v.size
    if budget >= L:
        return np.ones(L)
    order = sorted(range(L), key=lambda m: (-v[m], m))
    sv = v[order]
    tail = np.cumsum(sv[::-1])[::-1]           # tail[t] = sum of sv[t:]
    t = 0
    while (budget - t) * sv[t] > tail[t]:      # c_t v_(t) > 1: the t-th largest is certain
        t += 1
    c = (budget - t) / tail[t]
    pi = np.empty(L)
    for pos, m in enumerate(order):
        pi[m] = 1.0 if pos < t else c * sv[pos]
    return pi


def sip_select(I, ratio, u, q_counts, k_counts):
    """SIP selection ("AB-Attention ...", paragraph on SIP).  READING: per
    non-empty query cluster r, expected budget B = ceil(ratio L_r) (L_r
    non-empty key clusters); pi from sip_probabilities(I_r., B); block m is kept
    when u[r, m] < pi_m (independent draws, u uniform on [0, 1) given as input);
    kept blocks get the weight 1 / pi_m (the inverse inclusion probability).  If no
    block is drawn, the most important block is kept (with its weight).  Returns
    (mask, weight), weight 0 where not kept."""
    NQ, NK = I.shape
    mask = np.zeros((NQ, NK), dtype=bool)
    weight = np.zeros((NQ, NK))
    live = [m for m in range(NK) if k_counts[m] > 0]
    B = max(1, int(math.ceil(ratio * len(live))))
    for r in range(NQ):
        if q_counts[r] == 0:
            continue
        pi = sip_probabilities(I[r, live], B)
        for m, pm in zip(live, pi):
            if u[r, m] < pm:
                mask[r, m] = True
                weight[r, m] = 1.0 / pm
        if not mask[r].any():
            best = min(live, key=lambda m: (-I[r, m], m))
            mask[r, best] = True
            weight[r, best] = 1.0 / pi[live.index(best)]
    return mask, weight


# ----------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------


def dense_attention(Q, K, V, scale):
    """Textbook attention softmax(s Q K^T) V, row by row block."""
    Q, K, V = (np.asarray(a, dtype=np.float64) for a in (Q, K, V))
    O = np.empty((Q.shape[0], V.shape[1]))
    for i0 in range(0, Q.shape[0], 2048):
        S = scale * (Q[i0:i0 + 2048] @ K.T)
        S -= S.max(axis=1, keepdims=True)
        P = np.exp(S)
        O[i0:i0 + 2048] = (P @ V) / P.sum(axis=1, keepdims=True)
    return O


def sparse_attention(Q, K, V, q_labels, k_labels, mask, scale, rows=None, weight=None):
    """Block-sparse attention: query i attends, with a renormalised Softmax,
    only to keys whose cluster is kept for its query cluster a(i) (PARK
    abstract: attention is computed inside the retrieved blocks alone).  Returns
    float64 [N, d] in original token order (or only the listed rows).
    weight[r, m] (SIP): every exp term of key cluster m is multiplied by it, in
    the numerator and in the normaliser (a ratio of two inverse-probability
    weighted sums, each an unbiased estimate of its dense counterpart)."""
    Q, K, V = (np.asarray(a, dtype=np.float64) for a in (Q, K, V))
    q_labels = np.asarray(q_labels)
    k_labels = np.asarray(k_labels)
    want = np.arange(Q.shape[0]) if rows is None else np.asarray(rows)
    O = np.zeros((want.size, V.shape[1]))
    lab = q_labels[want]
    for r in np.unique(lab):
        sel = np.nonzero(lab == r)[0]
        keys = np.nonzero(mask[r][k_labels])[0]
        S = scale * (Q[want[sel]] @ K[keys].T)
        if weight is not None:
            S += np.log(weight[r][k_labels[keys]])[None, :]
        S -= S.max(axis=1, keepdims=True)
        P = np.exp(S)
        O[sel] = (P @ V[keys]) / P.sum(axis=1, keepdims=True)
    return O


# ----------------------------------------------------------------------------
# one layer
# ----------------------------------------------------------------------------


def retrieve_head(Q, K, NQ, NK, p, iters, dtype, qrkc=True, pama_mode="full", topk_ratio=None,
                  size_prior=False, sip_ratio=None, sip_u=None, grid=None, window=None, merge=False,
                  merge_rounds=8, q_init=None, k_init=None):
    """PARK retrieval for one (b, h): query K-means (Euclidean), key K-means
    with the query-derived metric (QRKC), PAMA importance, top-p mask
    (PARK Figure 2).  qrkc=False is the "w/o QRKC" ablation (M = I);
    pama_mode="centroid" is "w/o PAMA" (PARK Table 3); topk_ratio selects the
    top-k at that retrieval ratio instead of top-p (PARK Table 10);
    size_prior adds log |B_m| to the PAMA logits (a variant, see pama);
    sip_ratio with the uniforms sip_u [NQ, NK] selects by SIP (see sip_select)
    and adds the weights to the result.  window = (wt, wh, ww) with grid =
    (T, Hg, W) runs both K-means with HVA's local-window assign, and merge=True
    merges query clusters after the selection (hva_oracle); importance stays
    the one the selection used.  q_init / k_init: centroids to start K-means
    from instead of the strided initialisation (a warm start).  The result also
    holds q_hist / k_hist, the centroids entering each K-means iteration."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    d = Q.shape[1]
    scale = 1.0 / math.sqrt(d)
    qm = QueryMetric(Q)
    M = qm.M
    km = qm if qrkc else None
    q_hist = k_hist = None
    if window is None:
        q_labels, CQ, q_hist = kmeans(Q, NQ, iters, None, dtype, init=q_init, history=True)
        k_labels, CK, k_hist = kmeans(K, NK, iters, km, dtype, init=k_init, history=True)
    else:
        from . import hva_oracle as hva
        q_labels, CQ = hva.local_kmeans(Q, NQ, iters, grid, window, None, dtype)
        k_labels, CK = hva.local_kmeans(K, NK, iters, grid, window, km, dtype)
    q_counts = np.bincount(q_labels, minlength=NQ)
    k_counts = np.bincount(k_labels, minlength=NK)
    if pama_mode == "full":
        I = pama(Q, q_labels, NQ, CK, k_counts, scale, size_prior=size_prior)
    else:
        I = pama_centroid_query(CQ, q_counts, CK, k_counts, scale, size_prior=size_prior)
    weight = None
    if sip_ratio is not None:
        mask, weight = sip_select(I, sip_ratio, sip_u, q_counts, k_counts)
    elif topk_ratio is None:
        mask = top_p(I, p, q_counts, k_counts)
    else:
        mask = top_k_ratio(I, topk_ratio, q_counts, k_counts)
    if merge:
        if weight is not None:
            raise ValueError("merging is not defined for SIP weights")
        from . import hva_oracle as hva
        root = hva.merge_clusters(q_counts, mask, k_counts, merge_rounds)
        q_labels, CQ, mask = hva.apply_merge(Q, q_labels, CQ, mask, root, dtype)
        q_counts = np.bincount(q_labels, minlength=NQ)
    q_perm, q_off = stable_permutation(q_labels, NQ)
    k_perm, k_off = stable_permutation(k_labels, NK)
    return dict(M=M, q_labels=q_labels, k_labels=k_labels, q_centroids=CQ, k_centroids=CK,
                q_counts=q_counts, k_counts=k_counts, importance=I, mask=mask, weight=weight,
                q_perm=q_perm, q_offsets=q_off, k_perm=k_perm, k_offsets=k_off, q_hist=q_hist, k_hist=k_hist,
                qrkc=qrkc, k_metric=km)


def layer_head(Q, K, V, NQ, NK, p, iters, dtype, **kw):
    """Retrieval followed by block-sparse attention for one (b, h)."""
    r = retrieve_head(Q, K, NQ, NK, p, iters, dtype, **kw)
    scale = 1.0 / math.sqrt(np.asarray(Q).shape[1])
    r["O"] = sparse_attention(Q, K, V, r["q_labels"], r["k_labels"], r["mask"], scale, weight=r["weight"])
    return r


def layer(Q, K, V, NQ, NK, p, iters, dtype, **kw):
    """All (b, h) of [B, H, N, d] inputs; returns a list (row-major over b, h)."""
    B, H = Q.shape[:2]
    u = kw.pop("sip_u", None)  # [B, H, NQ, NK] uniforms for SIP, one slice per head
    return [layer_head(Q[b, h], K[b, h], V[b, h], NQ, NK, p, iters, dtype,
                       **kw, **({} if u is None else {"sip_u": np.asarray(u)[b, h]}))
            for b in range(B) for h in range(H)]


# ----------------------------------------------------------------------------
# diagnostics (PARK Tables 1, 4, 5)
# ----------------------------------------------------------------------------


def block_recall(Q, K, q_labels, k_labels, mask, scale, rows=None):
    """Attention recall of the kept blocks: (1/|rows|) sum_i sum_{j in J_a(i)} A_ij
    with A the dense float64 softmax(s Q K^T) (PARK Table 1)."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    want = np.arange(Q.shape[0]) if rows is None else np.asarray(rows)
    q_labels = np.asarray(q_labels)
    k_labels = np.asarray(k_labels)
    tot = 0.0
    for i0 in range(0, want.size, 2048):
        idx = want[i0:i0 + 2048]
        S = scale * (Q[idx] @ K.T)
        S -= S.max(axis=1, keepdims=True)
        A = np.exp(S)
        A /= A.sum(axis=1, keepdims=True)
        keep = mask[q_labels[idx]][:, k_labels]
        tot += float(np.sum(A * keep))
    return tot / want.size


def exact_block_mass(Q, K, q_labels, NQ, k_labels, NK, scale):
    """Full-query / full-key block importance: I_rm = mean_{i in Q_r} sum_{j in B_m} A_ij."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    S = scale * (Q @ K.T)
    S -= S.max(axis=1, keepdims=True)
    A = np.exp(S)
    A /= A.sum(axis=1, keepdims=True)
    mass = np.zeros((Q.shape[0], NK))
    np.add.at(mass.T, np.asarray(k_labels), A.T)
    q_counts = np.bincount(q_labels, minlength=NQ)
    I = np.zeros((NQ, NK))
    np.add.at(I, np.asarray(q_labels), mass)
    nz = q_counts > 0
    I[nz] /= q_counts[nz, None]
    return I, mass


def attention_tv(Q, K, k_labels, NK, CK, scale):
    """PARK Table 4, full-query / centroid-key row: mean_i (1/2) sum_m |P_im - sum_{j in B_m} A_ij|."""
    Q = np.asarray(Q, dtype=np.float64)
    k_counts = np.bincount(k_labels, minlength=NK)
    live = np.nonzero(k_counts > 0)[0]
    Z = scale * (Q @ np.asarray(CK, dtype=np.float64)[live].T)
    Z -= Z.max(axis=1, keepdims=True)
    P = np.exp(Z)
    P /= P.sum(axis=1, keepdims=True)
    _, mass = exact_block_mass(Q, K, np.zeros(Q.shape[0], dtype=np.int64), 1, k_labels, NK, scale)
    return float(np.mean(0.5 * np.sum(np.abs(P - mass[:, live]), axis=1)))


def key_errors(Q, K, k_labels, CK):
    """PARK Table 5: raw-key MSE mean_j ||k_j - c_a(j)||^2 / d ... reported as the
    mean over keys of the squared distance, and the QK-score squared error
    mean_{i,j} (q_i.k_j - q_i.c_a(j))^2, computed directly over queries."""
    Q = np.asarray(Q, dtype=np.float64)
    R = np.asarray(K, dtype=np.float64) - np.asarray(CK, dtype=np.float64)[np.asarray(k_labels)]
    raw = float(np.mean(np.sum(R * R, axis=1)))
    qk = float(np.mean((Q @ R.T) ** 2))
    return raw, qk
