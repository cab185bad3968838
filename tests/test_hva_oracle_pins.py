"""Pins of the HVA oracle (local-window K-means and CTA-aligned cluster
merging) to facts that do not come from the oracle itself: worked examples
computed by hand, reductions to the global K-means (already pinned against its
own worked examples), the independence of the windows, and a brute-force search
of the merged groups for any remaining profitable merge."""
import itertools
import math

import numpy as np
import pytest

from oracle import hva_oracle as hva
from oracle import park_oracle as po


def _bf16(x):
    return po.round_to_bf16(np.asarray(x, dtype=np.float64))


# ----------------------------------------------------------------------------- local windows


def test_local_window_worked_example():
    # grid 1 x 2 x 4 in (t, y, w) order, windows of 1 x 2 x 2 tokens: window 0 holds
    # tokens 0, 1, 4, 5 (values 0..3), window 1 tokens 2, 3, 6, 7 (values 10..13);
    # one centroid per window, initialised at the window's first token.
    X = np.array([0, 1, 10, 11, 2, 3, 12, 13], dtype=np.float64)[:, None]
    labels, C = hva.local_kmeans(X, 2, 3, (1, 2, 4), (1, 2, 2))
    assert labels.tolist() == [0, 0, 1, 1, 0, 0, 1, 1]
    assert C[:, 0].tolist() == [1.5, 11.5]
    # after one iteration the global K-means (started at tokens 0 and 4, values 0
    # and 2; value 1 ties and goes to centroid 0) still differs
    assert hva.local_kmeans(X, 2, 1, (1, 2, 4), (1, 2, 2))[0].tolist() == [0, 0, 1, 1, 0, 0, 1, 1]
    assert po.kmeans(X, 2, 1)[0].tolist() == [0, 0, 1, 1, 1, 1, 1, 1]


def test_text_token_joins_the_nearest_centroid_anywhere():
    # the same grid plus one text token of value 11: it has no window and joins
    # centroid 1 (value 10 at the first assign); centroid 1 becomes bf16(57 / 5)
    X = np.array([0, 1, 10, 11, 2, 3, 12, 13, 11], dtype=np.float64)[:, None]
    labels, C = hva.local_kmeans(X, 2, 3, (1, 2, 4), (1, 2, 2))
    assert labels.tolist() == [0, 0, 1, 1, 0, 0, 1, 1, 1]
    assert C[1, 0] == _bf16(57.0 / 5.0) == 11.375
    assert C[0, 0] == 1.5


def _grid_data(T, Hg, W, n_text, d, seed):
    rng = np.random.default_rng(seed)
    return _bf16(rng.normal(size=(T * Hg * W + n_text, d)))


@pytest.mark.parametrize("metric", [False, True])
def test_whole_grid_window_is_the_global_kmeans(metric):
    T, Hg, W, d, K = 3, 4, 5, 8, 7
    X = _grid_data(T, Hg, W, 0, d, 1)
    M = po.metric(_grid_data(T, Hg, W, 0, d, 2)) if metric else None
    l1, c1 = hva.local_kmeans(X, K, 4, (T, Hg, W), (T, Hg, W), M)
    l2, c2 = po.kmeans(X, K, 4, M)
    assert np.array_equal(l1, l2)
    assert np.array_equal(c1, c2)


def test_windows_are_independent_kmeans():
    # without text tokens every window is its own K-means over its members with
    # its share of the centroids
    T, Hg, W, d, K = 4, 6, 6, 8, 13
    window = (2, 3, 4)
    X = _grid_data(T, Hg, W, 0, d, 3)
    labels, C = hva.local_kmeans(X, K, 5, (T, Hg, W), window)
    nW = int(np.prod(hva.window_counts(T, Hg, W, window)))
    assert nW == 2 * 2 * 2
    k0 = [(w * K) // nW for w in range(nW + 1)]
    for w in range(nW):
        # the members of window w in token order, from the grid coordinates
        members = [(t * Hg + y) * W + x for t in range(T) for y in range(Hg) for x in range(W)
                   if ((t // 2) * 2 + y // 3) * 2 + x // 4 == w]
        lw, cw = po.kmeans(X[members], k0[w + 1] - k0[w], 5)
        assert np.array_equal(labels[members], lw + k0[w])
        assert np.array_equal(C[k0[w]:k0[w + 1]], cw)


def test_local_assign_candidates():
    T, Hg, W, n_text, d, K = 2, 4, 4, 5, 4, 6
    window = (1, 2, 4)
    X = _grid_data(T, Hg, W, n_text, d, 4)
    labels, C, hist = hva.local_kmeans(X, K, 3, (T, Hg, W), window, history=True)
    win = hva.token_windows(T, Hg, W, n_text, window)
    k0 = hva.window_starts(K, 4)
    Cl = hist[-1]
    for i in range(X.shape[0]):
        dist = [float(np.sum((X[i] - Cl[k]) ** 2)) for k in range(K)]
        if win[i] < 0:                 # text: the nearest of all centroids
            assert labels[i] == int(np.argmin(dist))
        else:                          # grid: the nearest centroid of its own window
            lo, hi = k0[win[i]], k0[win[i] + 1]
            assert lo <= labels[i] < hi
            assert labels[i] == lo + int(np.argmin(dist[lo:hi]))


def test_too_few_centroids_for_the_windows():
    X = _grid_data(2, 2, 2, 0, 4, 5)
    with pytest.raises(ValueError):
        hva.local_kmeans(X, 3, 2, (2, 2, 2), (1, 1, 2))   # 4 windows, 3 centroids


# ----------------------------------------------------------------------------- merging


def test_tile_cost_worked_values():
    assert hva.tile_cost(100, 256) == 2
    assert hva.tile_cost(129, 128) == 2
    assert hva.tile_cost(256, 257) == 6
    assert hva.padded_rows([1, 8, 9, 0]).tolist() == [8, 8, 16, 0]


def test_merge_worked_example():
    # cluster 0: 100 rows keeping blocks {0, 1}; cluster 1: 140 rows keeping {0, 1};
    # cluster 2: 20 rows keeping {3}; four key blocks of 128 rows.
    # costs 1*2, 2*2, 1*1; merging 0+1: 2 query tiles x 2 key tiles = 4 (gain 2);
    # 0+2: 1 x 3 = 3 (gain 0, not taken); 1+2: 2 x 3 = 6 (gain -1).
    n = [100, 140, 20]
    mask = np.array([[1, 1, 0, 0], [1, 1, 0, 0], [0, 0, 0, 1]], dtype=bool)
    k = [128, 128, 128, 128]
    root = hva.merge_clusters(n, mask, k)
    assert root.tolist() == [0, 0, 2]
    assert hva.total_tile_cost(n, mask, k) == 7
    n2 = np.bincount(root, weights=n, minlength=3).astype(int)
    m2 = np.zeros_like(mask)
    for r in range(3):
        m2[root[r]] |= mask[r]
    assert hva.total_tile_cost(n2, m2, k) == 5


def test_merge_ties_and_round_cap():
    # three 10-row clusters keeping the same 128-row block: every pair gains 1;
    # the first merge round pairs 0 with 1 (lowest partner on ties), the second adds 2
    n = [10, 10, 10]
    mask = np.ones((3, 1), dtype=bool)
    assert hva.merge_clusters(n, mask, [128]).tolist() == [0, 0, 0]
    assert hva.merge_clusters(n, mask, [128], rounds=1).tolist() == [0, 0, 2]


def test_merge_pairs_only_mutual_choices():
    # three 40-row clusters over five 128-row key blocks, A {0,1}, B {0,1,2,3},
    # C {1,2,3,4}: the gain of a pair is the number of shared blocks (a second query
    # tile never arises: 40 + 40 + 40 <= 128), so A -> B (2), B -> C (3), C -> B (3).
    # Only the mutual pair B, C merges in the first round; A joins in the second.
    n = [40, 40, 40]
    mask = np.array([[1, 1, 0, 0, 0], [1, 1, 1, 1, 0], [0, 1, 1, 1, 1]], dtype=bool)
    k = [128] * 5
    assert hva.merge_clusters(n, mask, k, rounds=1).tolist() == [0, 1, 1]
    assert hva.merge_clusters(n, mask, k).tolist() == [0, 0, 0]


def _gain_bruteforce(na, Sa, nb, Sb, wk):
    # the tile cost written with Python sets, independent of merge_clusters
    def cost(n, S):
        L = sum(int(wk[m]) for m in S)
        return math.ceil(n / 128) * math.ceil(L / 128)
    return cost(na, Sa) + cost(nb, Sb) - cost(na + nb, Sa | Sb)


@pytest.mark.parametrize("seed", range(6))
def test_merge_ends_in_a_local_optimum(seed):
    rng = np.random.default_rng(seed)
    NQ, NK = 11, 9
    n = rng.integers(0, 300, NQ)
    n[rng.integers(0, NQ)] = 0                      # an empty cluster stays alone
    k = rng.integers(1, 200, NK)
    mask = rng.random((NQ, NK)) < 0.4
    mask[np.arange(NQ), rng.integers(0, NK, NQ)] = True
    mask[n == 0] = False
    root = hva.merge_clusters(n, mask, k, rounds=1000)
    wk = hva.padded_rows(k)
    groups = {}
    for r in range(NQ):
        groups.setdefault(int(root[r]), []).append(r)
        assert root[root[r]] == root[r]              # roots are final
        if n[r] == 0:
            assert root[r] == r
    gsize = {g: int(sum(n[r] for r in rs)) for g, rs in groups.items()}
    gset = {g: set(m for r in rs for m in np.nonzero(mask[r])[0].tolist()) for g, rs in groups.items()}
    for g in groups:
        assert g == min(groups[g])                   # a group is named by its lowest cluster
    live = [g for g in groups if gsize[g] > 0]
    for a, b in itertools.combinations(live, 2):
        assert _gain_bruteforce(gsize[a], gset[a], gsize[b], gset[b], wk) <= 0
    before = hva.total_tile_cost(n, mask, k)
    m2 = np.zeros_like(mask)
    for r in range(NQ):
        m2[root[r]] |= mask[r]
    n2 = np.bincount(root, weights=n, minlength=NQ).astype(int)
    assert hva.total_tile_cost(n2, m2, k) <= before
    for r in range(NQ):
        assert np.all(m2[root[r]] >= mask[r])        # no query loses a kept block


def test_apply_merge_recomputes_centroids_and_moves_labels():
    Q = np.array([[0.0], [2.0], [4.0], [8.0]])
    q_labels = np.array([0, 0, 1, 2])
    CQ = np.array([[1.0], [4.0], [8.0]])
    mask = np.array([[1, 0], [0, 1], [1, 0]], dtype=bool)
    root = np.array([0, 0, 2])
    labels, C, m = hva.apply_merge(Q, q_labels, CQ, mask, root, "bf16")
    assert labels.tolist() == [0, 0, 0, 2]
    assert C[:, 0].tolist() == [2.0, 4.0, 8.0]       # (0+2+4)/3; cluster 1 is empty and keeps 4
    assert m.tolist() == [[True, True], [False, False], [True, False]]
