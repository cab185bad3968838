"""park_qrkc_metric_static: the QRKC metric for callers that cannot allocate
device memory (its scratch is an array compiled into the library).  Checked
through the C ABI against the metric park_retrieve writes, on two calls in a
row; this file is collected last."""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_means_b200 import _lib
from block_sparse_attention_means_b200 import park as P
from synth import CONFIGS
from synth.generator import gen_tensor

pytestmark = pytest.mark.gpu


def _static_metric(q: torch.Tensor, shape: P.Shape, M: torch.Tensor) -> int:
    s = shape.c()
    return _lib.load().park_qrkc_metric_static(ctypes.c_void_p(q.data_ptr()), ctypes.byref(s),
                                               ctypes.c_void_p(M.data_ptr()),
                                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_metric_matches_retrieve_twice():
    cfg = CONFIGS["small"]
    shape = P.Shape.of(cfg)
    dev = torch.device("cuda", 0)
    q = torch.from_numpy(gen_tensor(cfg, "Q")).to(dev).to(torch.bfloat16).contiguous()
    k = torch.from_numpy(gen_tensor(cfg, "K")).to(dev).to(torch.bfloat16).contiguous()
    out = P.alloc_retrieval(shape, cfg.NQ, cfg.NK, dev, with_metric=True)
    P.retrieve(q, k, shape, cfg.NQ, cfg.NK, cfg.p, 2, out=out)
    torch.cuda.synchronize()
    assert out.status_code() == 0
    ref = out.metric.cpu().numpy()
    results = []
    for _ in range(2):  # two calls in a row share the static scratch
        M = torch.full((cfg.B, cfg.H, cfg.D, cfg.D), float("nan"), dtype=torch.float64, device=dev)
        assert _static_metric(q, shape, M) == _lib.PARK_OK
        torch.cuda.synchronize()
        results.append(M.cpu().numpy())
    for got in results:
        assert np.all(np.isfinite(got))
        rel = np.abs(got - ref).max() / np.abs(ref).max()
        assert rel < 1e-13, rel
    assert np.array_equal(results[0], results[1])


def test_static_metric_rejects_too_many_heads():
    shape = P.Shape(1, 129, 2, 4, 8, 0, 128)  # 129 heads x 128 KiB partials > 16 MiB
    M = torch.empty(1, dtype=torch.float64, device="cuda:0")
    q = torch.empty(1, dtype=torch.bfloat16, device="cuda:0")
    assert _static_metric(q, shape, M) == _lib.PARK_ERR_UNSUPPORTED
