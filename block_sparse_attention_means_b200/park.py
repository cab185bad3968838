"""Thin PyTorch binding of libpark: device memory and streams come from torch,
every step of the computation runs in the library's CUDA kernels.

The names follow the C ABI: ``workspace_size``, ``retrieve``, ``sparse_attn``,
``layer``.  Tensors are [B, H, N, D], contiguous, on one CUDA device, in
torch.bfloat16 or torch.float32 with D a multiple of 32 up to 128 (bf16 with
D = 128 runs the tensor-core kernels).
"""
from __future__ import annotations

import ctypes
import dataclasses

import torch

from . import _lib

_DT = {torch.bfloat16: _lib.PARK_BF16, torch.float32: _lib.PARK_F32}


@dataclasses.dataclass(frozen=True)
class Shape:
    """Problem shape: N = T * Hg * W + n_text tokens (video grid first)."""
    B: int
    H: int
    T: int
    Hg: int
    W: int
    n_text: int
    D: int
    dtype: torch.dtype = torch.bfloat16

    @property
    def N(self) -> int:
        return self.T * self.Hg * self.W + self.n_text

    def c(self) -> _lib.ParkShape:
        if self.dtype not in _DT:
            raise TypeError(f"unsupported dtype {self.dtype}")
        return _lib.ParkShape(self.B, self.H, self.T, self.Hg, self.W, self.n_text, self.D, _DT[self.dtype])

    @staticmethod
    def of(cfg, dtype=None) -> "Shape":
        dt = dtype or (torch.bfloat16 if cfg.dtype == "bf16" else torch.float32)
        return Shape(cfg.B, cfg.H, cfg.T, cfg.Hg, cfg.W, cfg.n_text, cfg.D, dt)


@dataclasses.dataclass
class Retrieval:
    """Caller-owned retrieval result (see park_retrieval in include/park.h)."""
    q_labels: torch.Tensor
    k_labels: torch.Tensor
    q_perm: torch.Tensor
    k_perm: torch.Tensor
    q_offsets: torch.Tensor
    k_offsets: torch.Tensor
    q_centroids: torch.Tensor
    k_centroids: torch.Tensor
    importance: torch.Tensor
    mask: torch.Tensor
    kept_ptr: torch.Tensor
    kept_idx: torch.Tensor
    metric: torch.Tensor | None
    importance_bound: torch.Tensor | None
    counters: torch.Tensor
    status: torch.Tensor
    flags: int = 0
    sip_uniform: torch.Tensor | None = None   # float32 [B,H,NQ,NK], input with PARK_FLAG_SIP
    block_weight: torch.Tensor | None = None  # float32 [B,H,NQ,NK], output with PARK_FLAG_SIP
    window: tuple = (0, 0, 0)                 # (frames, rows, columns) of a box, with PARK_FLAG_LOCAL_WINDOW
    merge_rounds: int = 0                     # with PARK_FLAG_MERGE_Q (0 = the library's default)

    def c(self) -> _lib.ParkRetrieval:
        p = lambda t: ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)  # noqa: E731
        return _lib.ParkRetrieval(self.flags, p(self.q_labels), p(self.k_labels), p(self.q_perm), p(self.k_perm),
                                  p(self.q_offsets), p(self.k_offsets), p(self.q_centroids), p(self.k_centroids),
                                  p(self.importance), p(self.mask), p(self.kept_ptr), p(self.kept_idx),
                                  p(self.metric), p(self.importance_bound), p(self.counters), p(self.status),
                                  p(self.sip_uniform), p(self.block_weight), *[int(x) for x in self.window],
                                  int(self.merge_rounds))

    def status_code(self) -> int:
        return int(self.status.item())


def alloc_retrieval(shape: Shape, NQ: int, NK: int, device, with_metric: bool = False,
                    sip_uniform: torch.Tensor | None = None, window: tuple | None = None,
                    merge: bool = False, merge_rounds: int = 0) -> Retrieval:
    """Outputs of park_retrieve on `device`.  With sip_uniform (float32
    [B,H,NQ,NK] uniforms on the device) the result is set up for PARK_FLAG_SIP:
    the flag is set and block_weight is allocated.  window = (frames, rows,
    columns) sets PARK_FLAG_LOCAL_WINDOW with that box; merge sets
    PARK_FLAG_MERGE_Q."""
    B, H, N, D = shape.B, shape.H, shape.N, shape.D
    i32 = dict(dtype=torch.int32, device=device)
    sip = {}
    if sip_uniform is not None:
        if tuple(sip_uniform.shape) != (B, H, NQ, NK) or sip_uniform.dtype != torch.float32:
            raise ValueError("sip_uniform must be float32 [B, H, NQ, NK]")
        sip = dict(flags=_lib.PARK_FLAG_SIP, sip_uniform=sip_uniform.contiguous(),
                   block_weight=torch.empty(B, H, NQ, NK, dtype=torch.float32, device=device))
    flags = sip.pop("flags", 0)
    if window is not None:
        flags |= _lib.PARK_FLAG_LOCAL_WINDOW
        sip["window"] = tuple(int(x) for x in window)
    if merge:
        flags |= _lib.PARK_FLAG_MERGE_Q
        sip["merge_rounds"] = int(merge_rounds)
    return Retrieval(flags=flags, **sip,
        q_labels=torch.empty(B, H, N, **i32), k_labels=torch.empty(B, H, N, **i32),
        q_perm=torch.empty(B, H, N, **i32), k_perm=torch.empty(B, H, N, **i32),
        q_offsets=torch.empty(B, H, NQ + 1, **i32), k_offsets=torch.empty(B, H, NK + 1, **i32),
        q_centroids=torch.empty(B, H, NQ, D, dtype=shape.dtype, device=device),
        k_centroids=torch.empty(B, H, NK, D, dtype=shape.dtype, device=device),
        importance=torch.empty(B, H, NQ, NK, dtype=torch.float32, device=device),
        mask=torch.empty(B, H, NQ, NK, dtype=torch.uint8, device=device),
        kept_ptr=torch.empty(B, H, NQ + 1, **i32), kept_idx=torch.empty(B, H, NQ * NK, **i32),
        metric=torch.empty(B, H, D, D, dtype=torch.float64, device=device) if with_metric else None,
        importance_bound=torch.empty(B, H, NQ, dtype=torch.float32, device=device),
        counters=torch.zeros(_lib.PARK_NUM_COUNTERS, dtype=torch.int64, device=device),
        status=torch.zeros(1, dtype=torch.int32, device=device))


def workspace_size(shape: Shape, NQ: int, NK: int) -> int:
    n = ctypes.c_size_t(0)
    s = shape.c()
    _lib.check(_lib.load().park_workspace_size(ctypes.byref(s), NQ, NK, ctypes.byref(n)), "park_workspace_size")
    return int(n.value)


def alloc_workspace(shape: Shape, NQ: int, NK: int, device) -> torch.Tensor:
    return torch.empty(workspace_size(shape, NQ, NK), dtype=torch.uint8, device=device)


def _check_inputs(shape: Shape, *ts):
    want = (shape.B, shape.H, shape.N, shape.D)
    for t in ts:
        if tuple(t.shape) != want or t.dtype != shape.dtype or not t.is_contiguous() or not t.is_cuda:
            raise ValueError(f"expected contiguous CUDA {shape.dtype} tensor of shape {want}, got "
                             f"{tuple(t.shape)} {t.dtype} contiguous={t.is_contiguous()} device={t.device}")


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def retrieve(Q, K, shape: Shape, NQ: int, NK: int, p: float, iters: int, out: Retrieval | None = None,
             ws: torch.Tensor | None = None, stream=None) -> Retrieval:
    _check_inputs(shape, Q, K)
    out = out or alloc_retrieval(shape, NQ, NK, Q.device)
    ws = ws if ws is not None else alloc_workspace(shape, NQ, NK, Q.device)
    s, r = shape.c(), out.c()
    rc = _lib.load().park_retrieve(ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()), ctypes.byref(s),
                                   NQ, NK, float(p), int(iters), ctypes.byref(r), ctypes.c_void_p(ws.data_ptr()),
                                   ws.numel(), _stream(stream))
    _lib.check(rc, "park_retrieve")
    return out


def sparse_attn(Q, K, V, shape: Shape, NQ: int, NK: int, r: Retrieval, O: torch.Tensor | None = None,
                ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _check_inputs(shape, Q, K, V)
    O = O if O is not None else torch.empty_like(Q)
    _check_inputs(shape, O)
    ws = ws if ws is not None else alloc_workspace(shape, NQ, NK, Q.device)
    s, rc_ = shape.c(), r.c()
    rc = _lib.load().park_sparse_attn(ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()),
                                      ctypes.c_void_p(V.data_ptr()), ctypes.byref(s), NQ, NK, ctypes.byref(rc_),
                                      ctypes.c_void_p(O.data_ptr()), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                                      _stream(stream))
    _lib.check(rc, "park_sparse_attn")
    return O


def layer(Q, K, V, shape: Shape, NQ: int, NK: int, p: float, iters: int, O: torch.Tensor | None = None,
          out: Retrieval | None = None, ws: torch.Tensor | None = None, stream=None):
    """Retrieval + block-sparse attention; returns (O, Retrieval)."""
    _check_inputs(shape, Q, K, V)
    O = O if O is not None else torch.empty_like(Q)
    out = out or alloc_retrieval(shape, NQ, NK, Q.device)
    ws = ws if ws is not None else alloc_workspace(shape, NQ, NK, Q.device)
    s, r = shape.c(), out.c()
    rc = _lib.load().park_layer(ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(K.data_ptr()),
                                ctypes.c_void_p(V.data_ptr()), ctypes.byref(s), NQ, NK, float(p), int(iters),
                                ctypes.c_void_p(O.data_ptr()), ctypes.byref(r), ctypes.c_void_p(ws.data_ptr()),
                                ws.numel(), _stream(stream))
    _lib.check(rc, "park_layer")
    return O, out


def launch_count() -> int:
    return int(_lib.load().park_launch_count())


def profile_enable(on: bool = True) -> None:
    """Record a CUDA event pair around every later kernel launch of the library."""
    _lib.check(_lib.load().park_profile_enable(1 if on else 0), "park_profile_enable")


def profile_collect() -> dict:
    """{kernel name: (total ms, launches)} of the recorded launches (call after a
    synchronize); clears the record."""
    cap = 64
    buf = (_lib.ParkKernelTime * cap)()
    n = ctypes.c_int(0)
    _lib.check(_lib.load().park_profile_collect(buf, cap, ctypes.byref(n)), "park_profile_collect")
    return {buf[i].name.decode(): (buf[i].total_ms, int(buf[i].launches)) for i in range(n.value)}


def set_wait_limit_ns(ns: int) -> None:
    """Limit of every bounded device wait inside the library's kernels (0 = the
    default, 2 s).  Only the tests of the timeout path change it."""
    _lib.check(_lib.load().park_set_wait_limit_ns(int(ns)), "park_set_wait_limit_ns")
