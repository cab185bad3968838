"""park_qrkc_metric_static: the QRKC metric for callers that cannot allocate
device memory where they need it -- code running while a CUDA graph is being
captured (cudaMalloc cannot be captured) or a plug-in whose host framework
hands it only input and output buffers.  Its scratch is an array compiled into
the library.  Checked through the C ABI against the metric park_retrieve
writes and against the oracle, on two calls in a row; this file is collected
last."""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_means_b200 import _lib
from block_sparse_attention_means_b200 import park as P
from oracle import park_oracle as po
from synth import CONFIGS
from synth.generator import gen_tensor

pytestmark = pytest.mark.gpu


def _static_metric(q: torch.Tensor, shape: P.Shape, M: torch.Tensor, stream=None) -> int:
    s = shape.c()
    st = stream if stream is not None else torch.cuda.current_stream()
    return _lib.load().park_qrkc_metric_static(ctypes.c_void_p(q.data_ptr()), ctypes.byref(s),
                                               ctypes.c_void_p(M.data_ptr()), ctypes.c_void_p(st.cuda_stream))


def _rel(a, b):
    return np.abs(a - b).max() / np.abs(b).max()


def test_static_metric_matches_retrieve_and_oracle_twice():
    cfg = CONFIGS["small"]
    shape = P.Shape.of(cfg)
    dev = torch.device("cuda", 0)
    Qh = gen_tensor(cfg, "Q")
    q = torch.from_numpy(Qh).to(dev).to(torch.bfloat16).contiguous()
    k = torch.from_numpy(gen_tensor(cfg, "K")).to(dev).to(torch.bfloat16).contiguous()
    out = P.alloc_retrieval(shape, cfg.NQ, cfg.NK, dev, with_metric=True)
    P.retrieve(q, k, shape, cfg.NQ, cfg.NK, cfg.p, 2, out=out)
    torch.cuda.synchronize()
    assert out.status_code() == 0
    ref = out.metric.cpu().numpy()
    Ms = [torch.full((cfg.B, cfg.H, cfg.D, cfg.D), float("nan"), dtype=torch.float64, device=dev) for _ in range(3)]
    # the first call on the device looks up the array's address (the CUDA runtime may
    # load the library's module then); later calls take no device memory at all
    assert _static_metric(q, shape, Ms[2]) == _lib.PARK_OK
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(dev)[0]
    for M in Ms[:2]:  # two calls in a row share the static scratch
        assert _static_metric(q, shape, M) == _lib.PARK_OK
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info(dev)[0] == free0
    Ms = Ms[:2]
    results = [M.cpu().numpy() for M in Ms]
    for got in results:
        assert np.all(np.isfinite(got))
        assert _rel(got, ref) < 1e-13
        for h in range(cfg.H):
            assert _rel(got[0, h], po.metric(Qh[0, h].astype(np.float64))) < 1e-13
    assert np.array_equal(results[0], results[1])


def test_static_metric_fewer_row_chunks_for_many_heads():
    """40 heads: the array holds 128 partials of 128 x 128 float64, so each head
    gets 3 row chunks instead of park_retrieve's 8 (the reduced-chunk branch)."""
    cfg = CONFIGS["small"].replace(H=40)
    shape = P.Shape.of(cfg)
    dev = torch.device("cuda", 0)
    Qh = gen_tensor(cfg, "Q")
    q = torch.from_numpy(Qh).to(dev).to(torch.bfloat16).contiguous()
    for _ in range(2):
        M = torch.full((cfg.B, cfg.H, cfg.D, cfg.D), float("nan"), dtype=torch.float64, device=dev)
        assert _static_metric(q, shape, M) == _lib.PARK_OK
        torch.cuda.synchronize()
        got = M.cpu().numpy()
        for h in (0, 17, 39):
            assert _rel(got[0, h], po.metric(Qh[0, h].astype(np.float64))) < 1e-13


def test_static_metric_rejects_too_many_heads():
    """129 heads need more than the array: the call fails before enqueuing
    anything (no launch counted, the stream stays idle)."""
    shape = P.Shape(1, 129, 2, 4, 8, 0, 128)
    M = torch.empty(1, dtype=torch.float64, device="cuda:0")
    q = torch.empty(1, dtype=torch.bfloat16, device="cuda:0")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    before = P.launch_count()
    assert _static_metric(q, shape, M, stream=s) == _lib.PARK_ERR_UNSUPPORTED
    assert P.launch_count() == before
    assert s.query()
