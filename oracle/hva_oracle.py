"""HVA oracle: 3D local-window K-means and CTA-aligned query-cluster merging,
as plain float64 / integer CPU code.

TEST INFRASTRUCTURE ONLY, like park_oracle (whose K-means steps it reuses):
nothing in the product path may import it.

Source: "HyperVAttention: Efficient Sparse Attention with Spatio-Temporal
Clustering for Video Diffusion" (abstract).  The page names two of the method's
parts that touch this hot path and gives no equations for either:

* 3D local-window clustering: the centroid search is restricted to fixed local
  neighbourhoods of the video grid, which lowers the clustering cost;
* hardware-aware cluster merging: clusters are merged by parallel agglomerative
  merging so as to lower the tile-aligned (CTA-aligned) execution cost, which
  fills idle tile capacity, raises block density and, because a merged cluster
  attends to the union of its members' blocks, fidelity.

Every step below is the plainest reading of those sentences; each reading that
fills a gap is marked READING.
"""
from __future__ import annotations

import math

import numpy as np

from . import park_oracle as po

# ----------------------------------------------------------------------------
# 3D local windows
# ----------------------------------------------------------------------------


def window_counts(T, Hg, W, window):
    """Number of windows along (t, y, w) for a window of (wt, wh, ww) tokens;
    the last window of an axis may be shorter (READING: fixed, non-overlapping
    boxes tiling the grid)."""
    wt, wh, ww = window
    return -(-T // wt), -(-Hg // wh), -(-W // ww)


def token_windows(T, Hg, W, n_text, window):
    """Window id of every token, (a * nWh + b) * nWw + c for the box (a, b, c)
    holding grid position (t, y, w); text tokens (after the grid) get -1."""
    wt, wh, ww = window
    _, nWh, nWw = window_counts(T, Hg, W, window)
    t, y, w = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(W), indexing="ij")
    win = ((t // wt) * nWh + (y // wh)) * nWw + (w // ww)
    return np.concatenate([win.reshape(-1), np.full(n_text, -1, dtype=np.int64)]).astype(np.int64)


def window_starts(K, nW):
    """READING: the K centroids are split over the windows as evenly as integer
    division allows, window w owning centroids floor(w K / nW) .. floor((w+1) K / nW) - 1
    (every window owns at least one when K >= nW)."""
    return np.array([(w * K) // nW for w in range(nW + 1)], dtype=np.int64)


def local_init(X, K, win, nW):
    """READING (the global initialisation applied inside each window): centroid j
    of window w is the window's member floor(j n_w / K_w), members taken in token
    order."""
    X = np.asarray(X, dtype=np.float64)
    k0 = window_starts(K, nW)
    C = np.empty((K, X.shape[1]))
    for w in range(nW):
        members = np.nonzero(win == w)[0]
        Kw = k0[w + 1] - k0[w]
        for j in range(Kw):
            C[k0[w] + j] = X[members[(j * len(members)) // Kw]]
    return C


def local_assign(X, C, win, nW, M=None):
    """Each grid token searches only the centroids of its own window (READING of
    the abstract's centroid search limited to a fixed neighbourhood around each
    token: that neighbourhood is the token's window); a text token has no grid position and searches
    every centroid.  Distances and ties as in the global assign (lowest index)."""
    K = C.shape[0]
    k0 = window_starts(K, nW)
    labels = np.empty(X.shape[0], dtype=np.int64)
    for w in range(nW):
        rows = np.nonzero(win == w)[0]
        if len(rows):
            labels[rows] = k0[w] + po.assign(X[rows], C[k0[w]:k0[w + 1]], M)
    text = np.nonzero(win < 0)[0]
    if len(text):
        labels[text] = po.assign(X[text], C, M)
    return labels


def local_kmeans(X, K, iters, grid, window, M=None, dtype="bf16", init=None, history=False):
    """Lloyd K-means with the local assign: `iters` x (local assign, update), the
    update being the global exact-mean update (empty clusters keep their
    centroid).  grid = (T, Hg, W); the tokens past T*Hg*W are text tokens."""
    T, Hg, W = grid
    X = np.asarray(X, dtype=np.float64)
    n_text = X.shape[0] - T * Hg * W
    if n_text < 0 or iters < 1:
        raise ValueError("bad grid or iters")
    nWt, nWh, nWw = window_counts(T, Hg, W, window)
    nW = nWt * nWh * nWw
    if K < nW:
        raise ValueError("K must be at least the number of windows")
    win = token_windows(T, Hg, W, n_text, window)
    C = local_init(X, K, win, nW) if init is None else np.array(init, dtype=np.float64, copy=True)
    hist, labels = [], None
    for _ in range(iters):
        hist.append(C.copy())
        labels = local_assign(X, C, win, nW, M)
        C = po.update(X, labels, C, dtype)
    return (labels, C, hist) if history else (labels, C)


# ----------------------------------------------------------------------------
# CTA-aligned cluster merging
# ----------------------------------------------------------------------------

TILE_ROWS = 128   # query rows of one attention work item, key rows of one key tile
KEY_GROUP = 8     # key clusters are stored in whole groups of 8 rows


def padded_rows(k_counts):
    """Key rows a key cluster occupies in the attention's key tiles: its size
    rounded up to whole 8-row groups."""
    k_counts = np.asarray(k_counts, dtype=np.int64)
    return KEY_GROUP * ((k_counts + KEY_GROUP - 1) // KEY_GROUP)


def tile_cost(n, L):
    """(query tile, key tile) pairs the attention computes for a query group of
    n rows whose kept key clusters fill L padded key rows: ceil(n/128) query
    tiles, each streaming ceil(L/128) key tiles.  READING of "CTA-aligned
    execution cost" for this library's attention kernel (128-row query tiles,
    kept key clusters packed into 128-row key tiles)."""
    return -(-n // TILE_ROWS) * -(-L // TILE_ROWS)


def merge_clusters(q_counts, mask, k_counts, rounds=8):
    """Parallel agglomerative merging of query clusters (READING):

    * groups start as the non-empty query clusters, each with its kept set S_g
      (mask row), its size n_g and L_g = padded key rows of S_g;
    * one round: every group g picks the partner h != g with the largest gain
      cost(g) + cost(h) - cost(g u h) (tile_cost; the merged group keeps the
      union of the kept sets), only a strictly positive gain, ties to the lowest
      h; every mutual pair (g picks h, h picks g) merges into the lower index;
    * rounds repeat until one merges nothing, at most `rounds` times (the pages
      give no count).

    Returns root[r]: the group cluster r ended in (r itself if it was not
    merged away; empty clusters stay their own roots)."""
    mask = np.asarray(mask).astype(bool)
    NQ = mask.shape[0]
    wk = padded_rows(k_counts)
    n = np.asarray(q_counts, dtype=np.int64).copy()
    S = mask.astype(np.int64)
    alive = n > 0
    root = np.arange(NQ)
    for _ in range(rounds):
        L = S @ wk
        cost = np.array([tile_cost(n[g], L[g]) for g in range(NQ)])
        inter = (S * wk) @ S.T                      # padded rows kept by both g and h
        best = np.full(NQ, -1)
        for g in np.nonzero(alive)[0]:
            top = 0
            for h in np.nonzero(alive)[0]:
                if h == g:
                    continue
                gain = cost[g] + cost[h] - tile_cost(n[g] + n[h], L[g] + L[h] - inter[g, h])
                if gain > top:
                    top, best[g] = gain, h
        merged = False
        for g in np.nonzero(alive)[0]:
            h = best[g]
            if h > g and best[h] == g:
                S[g] = np.maximum(S[g], S[h])
                n[g] += n[h]
                n[h] = 0
                S[h] = 0
                alive[h] = False
                root[h] = g
                merged = True
        if not merged:
            break
    for r in range(NQ):                             # follow merges to the final group
        g = r
        while root[g] != g:
            g = root[g]
        root[r] = g
    return root


def apply_merge(Q, q_labels, CQ, mask, root, dtype):
    """The merged query clustering: every token moves to its cluster's root; a
    root's kept set is the union of its members' (so no query loses a block);
    merged-away clusters become empty (no kept blocks, centroid kept, as for any
    empty cluster); centroids are recomputed as exact means of the new members.
    Returns (labels, centroids, mask)."""
    labels = np.asarray(root)[np.asarray(q_labels)]
    new_mask = np.zeros_like(np.asarray(mask, dtype=bool))
    for r in range(len(root)):
        new_mask[root[r]] |= np.asarray(mask[r], dtype=bool)
    C = po.update(Q, labels, CQ, dtype)
    return labels, C, new_mask


def total_tile_cost(q_counts, mask, k_counts):
    """Sum over query clusters of tile_cost: the attention's (query tile, key
    tile) pairs."""
    wk = padded_rows(k_counts)
    L = np.asarray(mask, dtype=np.int64) @ wk
    return int(sum(tile_cost(int(n), int(l)) for n, l in zip(np.asarray(q_counts), L) if n > 0))
