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


def compare_retrieval(gpu, ref_heads, NQ: int, NK: int):
    """Bit-exact comparison of labels, centroids, permutations, masks and CSR;
    importance within its float32 rounding.  Returns a list of failure strings."""
    fails = []
    B, H = gpu.q_labels.shape[:2]
    ql, kl = gpu.q_labels.cpu().numpy(), gpu.k_labels.cpu().numpy()
    qp, kp = gpu.q_perm.cpu().numpy(), gpu.k_perm.cpu().numpy()
    qo, ko = gpu.q_offsets.cpu().numpy(), gpu.k_offsets.cpu().numpy()
    qc, kc = np64(gpu.q_centroids), np64(gpu.k_centroids)
    imp, mask = gpu.importance.cpu().numpy().astype(np.float64), gpu.mask.cpu().numpy().astype(bool)
    kptr, kidx = gpu.kept_ptr.cpu().numpy(), gpu.kept_idx.cpu().numpy()
    for bh, ref in enumerate(ref_heads):
        b, h = divmod(bh, H)
        for name, got, want in (("q_labels", ql[b, h], ref["q_labels"]), ("k_labels", kl[b, h], ref["k_labels"]),
                                ("q_perm", qp[b, h], ref["q_perm"]), ("k_perm", kp[b, h], ref["k_perm"]),
                                ("q_offsets", qo[b, h], ref["q_offsets"]), ("k_offsets", ko[b, h], ref["k_offsets"]),
                                ("q_centroids", qc[b, h], ref["q_centroids"]),
                                ("k_centroids", kc[b, h], ref["k_centroids"]), ("mask", mask[b, h], ref["mask"])):
            if not np.array_equal(got, want):
                bad = np.argwhere(np.asarray(got) != np.asarray(want))
                fails.append(f"bh={bh} {name}: {len(bad)} mismatches, first at {bad[:3].tolist()}")
        rel = np.abs(imp[b, h] - ref["importance"]) / np.maximum(ref["importance"], 1e-30)
        # importance is float32: the float64 path rounds once; the certified
        # float32 path is within its own bound (well below 1e-3 relative)
        if np.max(np.where(ref["importance"] > 1e-20, rel, 0.0)) > 1e-3:
            fails.append(f"bh={bh} importance: max rel err {rel.max():.3g}")
        ptr, idx = csr_from_mask(ref["mask"])
        if not np.array_equal(kptr[b, h], ptr):
            fails.append(f"bh={bh} kept_ptr differs")
        elif not np.array_equal(kidx[b, h][:ptr[-1]], idx):
            fails.append(f"bh={bh} kept_idx differs")
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
