"""Helpers shared by the GPU parity tests: run the oracle on seeded inputs,
run the CUDA path through the binding, and compare element by element."""
from __future__ import annotations

import functools
import math

import numpy as np
import torch

from oracle import park_oracle as po
from synth import CONFIGS, gen_layer

# Attention output tolerance for bf16 inputs with fp32 accumulation.
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
# float32 inputs: fp32 Softmax and accumulation on float32 values.
O_MAX_ABS_F32 = 1e-5


@functools.lru_cache(maxsize=None)
def inputs(name: str, seed: int = 0):
    return gen_layer(CONFIGS[name], seed)


@functools.lru_cache(maxsize=None)
def oracle_layer(name: str, seed: int = 0, p: float | None = None, NQ: int | None = None, NK: int | None = None,
                 iters: int | None = None):
    cfg = CONFIGS[name]
    Q, K, V = inputs(name, seed)
    return po.layer(Q.astype(np.float64), K.astype(np.float64), V.astype(np.float64), NQ or cfg.NQ, NK or cfg.NK,
                    cfg.p if p is None else p, iters or cfg.iters, cfg.dtype)



@functools.lru_cache(maxsize=None)
def oracle_layer_variant(name: str, p: float, variant: tuple):
    """The oracle layer with retrieval options (qrkc, pama_mode, topk_ratio,
    size_prior) given as a sorted tuple of (key, value) pairs."""
    cfg = CONFIGS[name]
    Q, K, V = inputs(name)
    return po.layer(Q.astype(np.float64), K.astype(np.float64), V.astype(np.float64), cfg.NQ, cfg.NK, p, cfg.iters,
                    cfg.dtype, **dict(variant))


def to_device(x: np.ndarray, dtype: torch.dtype, device="cuda:0") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(device=device).to(dtype).contiguous()


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def csr_from_mask(mask: np.ndarray):
    """CSR (row pointers, ascending column lists) of a boolean [NQ, NK] mask."""
    cnt = mask.sum(1)
    ptr = np.concatenate([[0], np.cumsum(cnt)])
    idx = np.concatenate([np.nonzero(row)[0] for row in mask]) if mask.any() else np.zeros(0, dtype=np.int64)
    return ptr, idx


# Where several results are correct: a label or a mask entry may differ from the
# oracle's only at a tie, i.e. where the oracle's own two distances (or the two
# importances at the top-p cut) differ by less than 1e-6 relative, or where the
# oracle's running sum at the cut is within 1e-6 of p.  Such mismatches are
# counted and reported; any other mismatch fails.
TIE_REL = 1e-6


def label_ties(X, C_enter, M, got, want):
    """(mismatched rows, excused rows) of a label vector: a row is excused when
    the oracle's distances to its own centroid and to the GPU's centroid (the
    centroids that entered the last assign) differ by < TIE_REL relative."""
    bad = np.nonzero(got != want)[0]
    if bad.size == 0:
        return bad, bad
    D = po.distances(np.asarray(X, dtype=np.float64)[bad], C_enter, M)
    d_want = D[np.arange(bad.size), want[bad]]
    d_got = D[np.arange(bad.size), got[bad]]
    ok = np.abs(d_got - d_want) <= TIE_REL * np.maximum(np.maximum(np.abs(d_want), np.abs(d_got)), 1e-300)
    return bad, bad[ok]


def mask_row_tie(I_row, live, got_row, want_row, p):
    """True when the mask rows differ only at a top-p tie (see TIE_REL)."""
    order = sorted(np.nonzero(live)[0].tolist(), key=lambda m: (-I_row[m], m))
    vals = np.array([I_row[m] for m in order])
    S = np.cumsum(vals)
    kept = int(np.sum(want_row))
    cut = max(kept - 1, 0)
    edge = vals[cut]
    diff = np.nonzero(got_row != want_row)[0]
    close = np.all(np.abs(I_row[diff] - edge) <= TIE_REL * max(edge, 1e-300))
    near_p = abs(S[cut] - p) <= TIE_REL or (cut > 0 and abs(S[cut - 1] - p) <= TIE_REL)
    return bool(close or near_p)


def _stable_ok(labels, perm, offsets, K):
    want_perm = np.argsort(labels, kind="stable")
    want_off = np.concatenate([[0], np.cumsum(np.bincount(labels, minlength=K))])
    return np.array_equal(perm, want_perm) and np.array_equal(offsets, want_off)


def compare_retrieval(gpu, ref_heads, NQ: int, NK: int, Q=None, K=None, p=None, report=None):
    """Comparison of labels, centroids, permutations, masks and CSR against the
    oracle, bit for bit; importance within its float32 rounding.  With the
    inputs Q, K ([BH, N, D] or [B, H, N, D]) and p, mismatches at ties (see
    TIE_REL) are counted instead of failing: labels against the oracle's
    distances (then the permutation must be the stable sort of the GPU's labels
    and only clusters that gained or lost an excused row may differ), mask rows
    against the oracle's importances.  Downstream of an excused label the
    clusterings differ, so masks and importance are then not compared (counted
    as cascaded heads).  Returns a list of failure strings; tie counts go to
    `report` (a dict) and are printed."""
    fails = []
    rep = report if report is not None else {}
    for key in ("q_label_ties", "k_label_ties", "mask_row_ties", "cascaded_heads", "heads"):
        rep.setdefault(key, 0)
    B, H = gpu.q_labels.shape[:2]
    ql, kl = gpu.q_labels.cpu().numpy(), gpu.k_labels.cpu().numpy()
    qp, kp = gpu.q_perm.cpu().numpy(), gpu.k_perm.cpu().numpy()
    qo, ko = gpu.q_offsets.cpu().numpy(), gpu.k_offsets.cpu().numpy()
    qc, kc = np64(gpu.q_centroids), np64(gpu.k_centroids)
    imp, mask = gpu.importance.cpu().numpy().astype(np.float64), gpu.mask.cpu().numpy().astype(bool)
    kptr, kidx = gpu.kept_ptr.cpu().numpy(), gpu.kept_idx.cpu().numpy()
    ties = Q is not None and K is not None
    if ties:
        Qh = np.asarray(Q).reshape(-1, *np.asarray(Q).shape[-2:])
        Kh = np.asarray(K).reshape(-1, *np.asarray(K).shape[-2:])
    for bh, ref in enumerate(ref_heads):
        b, h = divmod(bh, H)
        rep["heads"] += 1
        same_clustering = True
        for side, lab, perm, off, cen, KK in (("q", ql, qp, qo, qc, NQ), ("k", kl, kp, ko, kc, NK)):
            got, want = lab[b, h], ref[f"{side}_labels"]
            bad = np.nonzero(got != want)[0]
            if bad.size and ties and ref.get(f"{side}_hist") is not None:
                M = ref.get("k_metric") if side == "k" else None
                X = Qh[bh] if side == "q" else Kh[bh]
                bad, excused = label_ties(X, ref[f"{side}_hist"][-1], M, got, want)
                rep[f"{side}_label_ties"] += int(excused.size)
                unexcused = np.setdiff1d(bad, excused)
                if unexcused.size:
                    fails.append(f"bh={bh} {side}_labels: {unexcused.size} mismatches not at a tie, first at "
                                 f"{unexcused[:3].tolist()}")
            elif bad.size:
                fails.append(f"bh={bh} {side}_labels: {bad.size} mismatches, first at {bad[:3].tolist()}")
            if bad.size == 0:
                for name, g, w in ((f"{side}_perm", perm[b, h], ref[f"{side}_perm"]),
                                   (f"{side}_offsets", off[b, h], ref[f"{side}_offsets"]),
                                   (f"{side}_centroids", cen[b, h], ref[f"{side}_centroids"])):
                    if not np.array_equal(g, w):
                        e = np.argwhere(np.asarray(g) != np.asarray(w))
                        fails.append(f"bh={bh} {name}: {len(e)} mismatches, first at {e[:3].tolist()}")
            else:
                same_clustering = False
                if not _stable_ok(got, perm[b, h], off[b, h], KK):
                    fails.append(f"bh={bh} {side}_perm/offsets are not the stable sort of the GPU's labels")
                touched = np.union1d(got[bad], want[bad])
                keep = np.setdiff1d(np.arange(KK), touched)
                if not np.array_equal(cen[b, h][keep], ref[f"{side}_centroids"][keep]):
                    fails.append(f"bh={bh} {side}_centroids differ on clusters without a tied row")
        if not same_clustering:
            rep["cascaded_heads"] += 1
            continue
        live = ref["k_counts"] > 0
        drows = np.nonzero(np.any(mask[b, h] != ref["mask"], axis=1))[0]
        if drows.size:
            if ties and p is not None:
                excused = [r for r in drows
                           if mask_row_tie(ref["importance"][r], live, mask[b, h][r], ref["mask"][r], p)]
                rep["mask_row_ties"] += len(excused)
                if len(excused) < drows.size:
                    fails.append(f"bh={bh} mask: {drows.size - len(excused)} rows differ not at a tie, first "
                                 f"{[r for r in drows if r not in excused][:3]}")
            else:
                fails.append(f"bh={bh} mask: {drows.size} rows differ, first {drows[:3].tolist()}")
        rel = np.abs(imp[b, h] - ref["importance"]) / np.maximum(ref["importance"], 1e-30)
        # importance is float32: the float64 path rounds once; the certified
        # float32 path is within its own bound (well below 1e-3 relative)
        if np.max(np.where(ref["importance"] > 1e-20, rel, 0.0)) > 1e-3:
            fails.append(f"bh={bh} importance: max rel err {rel.max():.3g}")
        ptr, idx = csr_from_mask(mask[b, h])  # the CSR must describe the GPU's own mask
        if not np.array_equal(kptr[b, h], ptr):
            fails.append(f"bh={bh} kept_ptr differs")
        elif not np.array_equal(kidx[b, h][:ptr[-1]], idx):
            fails.append(f"bh={bh} kept_idx differs")
    if ties:
        print(f"ties: {rep}")
    return fails


def compare_output(O_gpu: torch.Tensor, ref_heads, f32: bool):
    O = np64(O_gpu)
    B, H = O.shape[:2]
    worst, mean_acc, n = 0.0, 0.0, 0
    for bh, ref in enumerate(ref_heads):
        b, h = divmod(bh, H)
        d = np.abs(O[b, h] - ref["O"])
        worst = max(worst, float(d.max()))
        mean_acc += float(d.sum())
        n += d.size
    return worst, mean_acc / n


def assert_output_close(O_gpu, ref_heads, f32: bool):
    worst, mean = compare_output(O_gpu, ref_heads, f32)
    if f32:
        assert worst <= O_MAX_ABS_F32, f"max abs err {worst:.3g}"
    else:
        assert worst <= O_MAX_ABS and mean <= O_MEAN_ABS, f"max abs {worst:.3g}, mean abs {mean:.3g}"
    return worst, mean


def scale_of(D: int) -> float:
    return 1.0 / math.sqrt(D)
