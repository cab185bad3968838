"""Seeded synthetic Q/K/V for one video-DiT attention layer.

This module only *creates inputs*; it holds none of the retrieval or attention
arithmetic, so both the CPU oracle and the CUDA path may import it.

Recipe (the pages' HunyuanVideo / Wan layers are replaced by data of the same
shape; real activations are not available):

* Tokens are a T x Hg x W video grid in (t, y, w) order, w fastest, followed by
  ``n_text`` text tokens (HunyuanVideo only).
* Positional features, per (tensor, batch, head, channel):
  ``x(t,y,w) = sum_{s<8} a_s sin(2 pi (f_t t/T + f_h y/Hg + f_w w/W) + phi_s)``
  with ``a_s ~ N(0, 0.5^2)``, ``f ~ U{0..3}`` per axis, ``phi ~ U[0, 2 pi)``,
  plus ``N(0, 0.3^2)`` noise (0.3 read as a standard deviation).
* 3D rotary embedding on Q and K video tokens (configs with ``rope``): the D/2
  channel pairs (2j, 2j+1) are split over the (t, y, w) axes as
  (D/2 - 2*(D/2//3), D/2//3, D/2//3) = 22/21/21 for D = 128, with
  ``theta_j = 10000^(-j/n_axis)``. Text tokens get no rotary embedding.
* V is positional (tiny, small) or i.i.d. N(0, 1) (Wan- and HunyuanVideo-shaped).
  Text tokens are i.i.d. N(0, 1) in Q, K and V.
* Values are computed in float64, rounded to float32 and then, for bf16
  configs, to bf16 with round-to-nearest-even.  Nothing else is changed.
* Every (tensor, batch, head) slice has its own stream
  ``numpy.random.default_rng([seed, tensor_id, b, h])`` so slices can be made
  in any order, in parallel, and one at a time for large configs.
"""
from __future__ import annotations

import concurrent.futures as _fut
import dataclasses
import math
import os

import numpy as np

TENSOR_IDS = {"Q": 0, "K": 1, "V": 2, "U": 3}


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    B: int
    H: int
    T: int
    Hg: int
    W: int
    n_text: int
    D: int
    dtype: str          # "bf16" or "f32"
    NQ: int
    NK: int
    iters: int
    p: float
    rope: bool
    v_kind: str         # "positional" or "normal"

    @property
    def N(self) -> int:
        return self.T * self.Hg * self.W + self.n_text

    def replace(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)


def _nclusters(n: int, size: int) -> int:
    # "~591 / ~930 clusters of mean size 128": floor(N/size + 1/2)
    return int(math.floor(n / size + 0.5))


CONFIGS = {
    "tiny": LayerConfig("tiny", 1, 1, 4, 8, 8, 0, 64, "f32", 8, 16, 10, 0.9, False, "positional"),
    "small": LayerConfig("small", 1, 8, 8, 16, 16, 0, 128, "bf16", 32, 32, 10, 0.9, True, "positional"),
    "wan": LayerConfig("wan", 1, 40, 21, 45, 80, 0, 128, "bf16",
                       _nclusters(75600, 128), _nclusters(75600, 128), 10, 0.9, True, "normal"),
    "hunyuan": LayerConfig("hunyuan", 1, 24, 33, 45, 80, 256, 128, "bf16",
                           _nclusters(119056, 128), _nclusters(119056, 128), 10, 0.9, True, "normal"),
    # the PARK paper's own HunyuanVideo setting (its Table 7 row matching Table 3's PARK row):
    # 128 query centroids, 1024 key centroids; context beside the pages' PAMA timings
    "hunyuan_nq128_nk1024": LayerConfig("hunyuan_nq128_nk1024", 1, 24, 33, 45, 80, 256, 128, "bf16",
                                        128, 1024, 10, 0.9, True, "normal"),
}


def sweep_configs():
    """Granularity/sparsity sweep at the HunyuanVideo shape: key clusters of mean
    size 32/64/128 (NK = 3721/1860/930) x p in {0.8, 0.9, 0.95}."""
    base = CONFIGS["hunyuan"]
    out = []
    for size in (32, 64, 128):
        for p in (0.8, 0.9, 0.95):
            out.append(base.replace(name=f"hunyuan_nk{size}_p{p}", NK=_nclusters(base.N, size), p=p))
    return out


def round_bf16_from_f32(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    r = ((u + bias) & np.uint32(0xFFFF0000)).astype(np.uint32)
    return r.view(np.float32)


def _positional(rng: np.random.Generator, cfg: LayerConfig) -> np.ndarray:
    """Sum of 8 random sinusoids over (t, y, w) per channel, float64 [Nv, D]."""
    D, T, Hg, W = cfg.D, cfg.T, cfg.Hg, cfg.W
    a = rng.normal(0.0, 0.5, size=(D, 8))
    f = rng.integers(0, 4, size=(D, 8, 3))
    phi = rng.uniform(0.0, 2.0 * np.pi, size=(D, 8))
    # Group the 8 terms by their frequency triple: A[c, ft, fh, fw] (complex).
    A = np.zeros((D, 4, 4, 4), dtype=np.complex128)
    coef = a * np.exp(1j * phi)
    for s in range(8):
        np.add.at(A, (np.arange(D), f[:, s, 0], f[:, s, 1], f[:, s, 2]), coef[:, s])
    fr = np.arange(4)
    Et = np.exp(2j * np.pi * np.outer(fr, np.arange(T)) / T)    # [4, T]
    Eh = np.exp(2j * np.pi * np.outer(fr, np.arange(Hg)) / Hg)  # [4, Hg]
    Ew = np.exp(2j * np.pi * np.outer(fr, np.arange(W)) / W)    # [4, W]
    t1 = np.einsum("cabf,fw->cabw", A, Ew)
    t2 = np.einsum("cabw,by->cayw", t1, Eh)
    x = np.einsum("cayw,at->tywc", t2, Et)                      # [T, Hg, W, D]
    out = x.imag.reshape(T * Hg * W, D)
    out += rng.standard_normal(size=out.shape) * 0.3
    return out


def _rope_3d(x: np.ndarray, cfg: LayerConfig) -> np.ndarray:
    """Rotate channel pairs (2j, 2j+1) by position x theta_j, axes split t/y/w."""
    D, T, Hg, W = cfg.D, cfg.T, cfg.Hg, cfg.W
    npair = D // 2
    n_y = n_w = npair // 3
    n_t = npair - n_y - n_w
    t, y, w = np.meshgrid(np.arange(T), np.arange(Hg), np.arange(W), indexing="ij")
    pos = [t.reshape(-1), y.reshape(-1), w.reshape(-1)]
    angles = np.empty((x.shape[0], npair))
    col = 0
    for axis, n_axis in enumerate((n_t, n_y, n_w)):
        theta = 10000.0 ** (-np.arange(n_axis) / n_axis)
        angles[:, col:col + n_axis] = np.outer(pos[axis], theta)
        col += n_axis
    c, s = np.cos(angles), np.sin(angles)
    xe, xo = x[:, 0::2], x[:, 1::2]
    out = np.empty_like(x)
    out[:, 0::2] = xe * c - xo * s
    out[:, 1::2] = xe * s + xo * c
    return out


def _finish(x64: np.ndarray, dtype: str) -> np.ndarray:
    x32 = x64.astype(np.float32)
    if dtype == "bf16":
        x32 = round_bf16_from_f32(x32)
    return x32


def gen_slice(cfg: LayerConfig, tensor: str, b: int, h: int, seed: int = 0) -> np.ndarray:
    """One (tensor, batch, head) slice as float32 [N, D] holding values exactly
    representable in ``cfg.dtype``."""
    rng = np.random.default_rng([seed, TENSOR_IDS[tensor], b, h])
    nv = cfg.T * cfg.Hg * cfg.W
    if tensor == "V" and cfg.v_kind == "normal":
        x = rng.standard_normal(size=(nv, cfg.D))
    else:
        x = _positional(rng, cfg)
        if tensor in ("Q", "K") and cfg.rope:
            x = _rope_3d(x, cfg)
    if cfg.n_text:
        txt = rng.standard_normal(size=(cfg.n_text, cfg.D))
        x = np.concatenate([x, txt], axis=0)
    return _finish(x, cfg.dtype)


def gen_tensor(cfg: LayerConfig, tensor: str, seed: int = 0, heads=None, workers=None) -> np.ndarray:
    """Full [B, H, N, D] float32 tensor (or only the listed (b, h) heads, stacked
    as [len(heads), N, D])."""
    if heads is None:
        heads = [(b, h) for b in range(cfg.B) for h in range(cfg.H)]
        shape = (cfg.B, cfg.H, cfg.N, cfg.D)
    else:
        shape = (len(heads), cfg.N, cfg.D)
    out = np.empty((len(heads), cfg.N, cfg.D), dtype=np.float32)
    workers = workers or min(len(heads), os.cpu_count() or 1)

    def one(i):
        b, h = heads[i]
        out[i] = gen_slice(cfg, tensor, b, h, seed)

    if workers <= 1:
        for i in range(len(heads)):
            one(i)
    else:
        with _fut.ThreadPoolExecutor(workers) as ex:
            list(ex.map(one, range(len(heads))))
    return out.reshape(shape)


def gen_layer(cfg: LayerConfig, seed: int = 0, workers=None):
    """(Q, K, V), each float32 [B, H, N, D]."""
    return tuple(gen_tensor(cfg, t, seed, workers=workers) for t in ("Q", "K", "V"))


def gen_integer_blobs(n: int, d: int, k: int, seed: int, spread: int = 2, sep: int = 20) -> np.ndarray:
    """Small integer-valued point sets (well separated blobs) for brute-force
    K-means checks: exact arithmetic, exact ties possible. float64 [n, d]."""
    rng = np.random.default_rng([seed, 99])
    centers = rng.integers(-3, 4, size=(k, d)) * sep
    lab = rng.integers(0, k, size=n)
    return (centers[lab] + rng.integers(-spread, spread + 1, size=(n, d))).astype(np.float64)


def gen_uniform(cfg: LayerConfig, seed: int = 0) -> np.ndarray:
    """Uniforms on [0, 1) for randomised block selection, float32 [B, H, NQ, NK]
    (one stream per (b, h), like the tensors).  Values are float32 so that the
    oracle and the GPU compare against the same numbers."""
    out = np.empty((cfg.B, cfg.H, cfg.NQ, cfg.NK), dtype=np.float32)
    for b in range(cfg.B):
        for h in range(cfg.H):
            rng = np.random.default_rng([seed, TENSOR_IDS["U"], b, h])
            out[b, h] = rng.random((cfg.NQ, cfg.NK), dtype=np.float32)
    return out


def with_extreme_magnitudes(x: np.ndarray, dtype: str, seed: int, frac_small: float = 0.01,
                            frac_zero: float = 0.002, frac_large: float = 0.0, large_exp=(16.0, 39.9)) -> np.ndarray:
    """A copy of ``x`` with a seeded fraction of its elements replaced by values
    at the ends of the library's input range (0 or 2^-40 <= |x| < 2^40):
    magnitudes 2^u with u ~ U[-40, -20) (``frac_small``), exact zeros
    (``frac_zero``) and magnitudes 2^u with u ~ U[large_exp) (``frac_large``),
    random signs, rounded to ``dtype`` (a rounding that reaches 2^40 is pulled
    back one ulp).  Only an input generator: it holds none of the method's
    arithmetic."""
    rng = np.random.default_rng([seed, 7])
    out = np.array(x, dtype=np.float32, copy=True)
    flat = out.reshape(-1)
    n = flat.size
    pick = rng.random(n)
    sign = np.where(rng.random(n) < 0.5, -1.0, 1.0)
    u_small = rng.uniform(-40.0, -20.0, size=n)
    u_large = rng.uniform(large_exp[0], large_exp[1], size=n)
    small = pick < frac_small
    zero = (pick >= frac_small) & (pick < frac_small + frac_zero)
    large = (pick >= frac_small + frac_zero) & (pick < frac_small + frac_zero + frac_large)
    vals = np.where(small, sign * np.exp2(u_small), np.where(large, sign * np.exp2(u_large), 0.0))
    v32 = _finish(vals, dtype)
    top = np.float32(2.0 ** 40)
    v32 = np.where(np.abs(v32) >= top, np.nextafter(np.float32(np.abs(v32)), np.float32(0)) * np.sign(v32), v32)
    v32 = np.where(np.abs(v32) < np.float32(2.0 ** -40), np.sign(v32) * np.float32(2.0 ** -40), v32)
    v32 = _finish(v32.astype(np.float64), dtype)
    flat[small | zero | large] = v32[small | zero | large]
    flat[zero] = 0.0
    return out
