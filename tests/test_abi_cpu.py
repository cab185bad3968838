"""C ABI checks that need no GPU: the library loads, exports every function
include/park.h declares, and rejects bad arguments on the host before any
device work is enqueued."""
import ctypes
import os
import re

import pytest

from block_sparse_attention_means_b200 import _lib
from block_sparse_attention_means_b200 import park as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "park.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(park_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_function():
    lib = _lib.load()
    declared = header_functions()
    assert set(declared) == set(_lib.EXPORTS), declared
    for name in declared:
        assert hasattr(lib, name), name
    assert lib.park_version() >= 100


def test_struct_layout_matches_header():
    # park_shape: 8 ints; park_retrieval: uint32 flags + 18 pointers (padded) + 4 int32
    assert ctypes.sizeof(_lib.ParkShape) == 32
    assert ctypes.sizeof(_lib.ParkRetrieval) == 8 + 18 * 8 + 4 * 4
    text = open(os.path.join(ROOT, "include", "park.h")).read()
    assert re.search(r"#define PARK_NUM_COUNTERS 8", text)
    for name in ("PARK_OK", "PARK_ERR_INVALID_ARG", "PARK_ERR_UNSUPPORTED", "PARK_ERR_WORKSPACE", "PARK_ERR_CUDA",
                 "PARK_ERR_RANGE", "PARK_ERR_TIMEOUT", "PARK_BF16", "PARK_F32", "PARK_FLAG_WARM_START_Q",
                 "PARK_FLAG_WARM_START_K", "PARK_FLAG_NO_QRKC", "PARK_FLAG_CENTROID_QUERY", "PARK_FLAG_TOPK",
                 "PARK_FLAG_SIZE_PRIOR", "PARK_FLAG_SIP", "PARK_FLAG_MERGE_Q", "PARK_FLAG_LOCAL_WINDOW",
                 "PARK_FLAG_NO_TILE_PACKING",
                 "PARK_CNT_KEPT_PAIRS"):
        m = re.search(rf"#define {name} (\w+)", text)
        assert m and int(m.group(1).rstrip("u"), 0) == getattr(_lib, name), name


def test_status_strings():
    for code in range(7):
        assert _lib.status_string(code)
    assert _lib.status_string(99) == "unknown status"


def test_workspace_size_and_shape_validation():
    hy = P.Shape(1, 24, 33, 45, 80, 256, 128)
    n = P.workspace_size(hy, 930, 930)
    assert 2.0e9 < n < 4.0e9                     # the item-major Q image and the K/V tile images dominate
    # streamed PAMA: workspace does not grow with N * NK (PARK Appendix Table 6)
    n2 = P.workspace_size(P.Shape(1, 24, 66, 45, 80, 256, 128), 930, 930)
    assert n2 < 2.2 * n
    assert P.workspace_size(P.Shape(1, 8, 8, 16, 16, 0, 64), 32, 32) > 0         # bf16 with D = 64
    bad = [(P.Shape(1, 8, 8, 16, 16, 0, 48), 32, 32, _lib.PARK_ERR_UNSUPPORTED),    # D % 32 != 0
           (P.Shape(1, 8, 8, 16, 16, 0, 160), 32, 32, _lib.PARK_ERR_UNSUPPORTED),   # D > 128
           (P.Shape(1, 8, 8, 32, 32, 0, 128, dtype=__import__("torch").float32), 32, 5000,
            _lib.PARK_ERR_UNSUPPORTED),                                              # NK > 4096
           (P.Shape(1, 8, 8, 16, 16, 0, 128), 0, 32, _lib.PARK_ERR_INVALID_ARG),
           (P.Shape(1, 8, 8, 16, 16, 0, 128), 32, 2049, _lib.PARK_ERR_INVALID_ARG),  # NK > N
           (P.Shape(0, 8, 8, 16, 16, 0, 128), 32, 32, _lib.PARK_ERR_INVALID_ARG),
           (P.Shape(1, 1, 128, 128, 128, 0, 128), 8, 8, _lib.PARK_ERR_UNSUPPORTED)]  # N > 2^20
    for shape, nq, nk, code in bad:
        with pytest.raises(_lib.ParkError) as e:
            P.workspace_size(shape, nq, nk)
        assert e.value.code == code, (shape, nq, nk)


def _fake_retrieval():
    # non-null placeholders: every call below fails validation before touching them
    r = _lib.ParkRetrieval()
    for name, kind in _lib.ParkRetrieval._fields_[1:]:
        if kind is ctypes.c_void_p:
            setattr(r, name, ctypes.c_void_p(0x1000))
    return r


def test_host_argument_errors_enqueue_nothing():
    lib = _lib.load()
    shape = P.Shape(1, 2, 2, 4, 8, 0, 128).c()
    fake = ctypes.c_void_p(0x1000)
    r = _fake_retrieval()
    need = P.workspace_size(P.Shape(1, 2, 2, 4, 8, 0, 128), 4, 4)
    before = lib.park_launch_count()
    cases = [
        (lib.park_retrieve(fake, fake, ctypes.byref(shape), 4, 4, 0.9, 10, ctypes.byref(r), fake, need - 1, None),
         _lib.PARK_ERR_WORKSPACE),
        (lib.park_retrieve(fake, fake, ctypes.byref(shape), 4, 4, 0.0, 10, ctypes.byref(r), fake, need, None),
         _lib.PARK_ERR_INVALID_ARG),
        (lib.park_retrieve(fake, fake, ctypes.byref(shape), 4, 4, float("nan"), 10, ctypes.byref(r), fake, need,
                           None), _lib.PARK_ERR_INVALID_ARG),
        (lib.park_retrieve(fake, fake, ctypes.byref(shape), 4, 4, 0.9, 0, ctypes.byref(r), fake, need, None),
         _lib.PARK_ERR_INVALID_ARG),
        (lib.park_retrieve(None, fake, ctypes.byref(shape), 4, 4, 0.9, 10, ctypes.byref(r), fake, need, None),
         _lib.PARK_ERR_INVALID_ARG),
        (lib.park_retrieve(fake, fake, ctypes.byref(shape), 4, 4, 0.9, 10, None, fake, need, None),
         _lib.PARK_ERR_INVALID_ARG),
        (lib.park_sparse_attn(fake, fake, None, ctypes.byref(shape), 4, 4, ctypes.byref(r), fake, fake, need, None),
         _lib.PARK_ERR_INVALID_ARG),
        (lib.park_layer(fake, fake, fake, ctypes.byref(shape), 4, 65, 0.9, 10, fake, ctypes.byref(r), fake, need,
                        None), _lib.PARK_ERR_INVALID_ARG),
    ]
    r2 = _fake_retrieval()
    r2.mask = None
    cases.append((lib.park_retrieve(fake, fake, ctypes.byref(shape), 4, 4, 0.9, 10, ctypes.byref(r2), fake, need,
                                    None), _lib.PARK_ERR_INVALID_ARG))
    r3 = _fake_retrieval()
    r3.flags = 0x400                              # unknown flag bit
    cases.append((lib.park_retrieve(fake, fake, ctypes.byref(shape), 4, 4, 0.9, 10, ctypes.byref(r3), fake, need,
                                    None), _lib.PARK_ERR_INVALID_ARG))
    r4 = _fake_retrieval()
    r4.flags = _lib.PARK_FLAG_TOPK                # a top-k ratio above 1
    cases.append((lib.park_retrieve(fake, fake, ctypes.byref(shape), 4, 4, 1.5, 10, ctypes.byref(r4), fake, need,
                                    None), _lib.PARK_ERR_INVALID_ARG))
    r5 = _fake_retrieval()
    r5.flags = _lib.PARK_FLAG_SIP                 # SIP without its uniforms
    r5.sip_uniform = None
    cases.append((lib.park_retrieve(fake, fake, ctypes.byref(shape), 4, 4, 0.5, 10, ctypes.byref(r5), fake, need,
                                    None), _lib.PARK_ERR_INVALID_ARG))
    r6 = _fake_retrieval()
    r6.flags = _lib.PARK_FLAG_SIP | _lib.PARK_FLAG_TOPK
    r6.sip_uniform = r6.block_weight = 0x1000
    cases.append((lib.park_retrieve(fake, fake, ctypes.byref(shape), 4, 4, 0.5, 10, ctypes.byref(r6), fake, need,
                                    None), _lib.PARK_ERR_INVALID_ARG))
    # HVA options: merging with SIP, too many merging rounds, a box that is empty,
    # larger than the grid (2 x 4 x 8 here), or more boxes than centroids
    bad = [(_lib.PARK_FLAG_MERGE_Q | _lib.PARK_FLAG_SIP, dict(), 0.5),
           (_lib.PARK_FLAG_MERGE_Q, dict(merge_rounds=65), 0.9),
           (_lib.PARK_FLAG_MERGE_Q, dict(merge_rounds=-1), 0.9),
           (_lib.PARK_FLAG_LOCAL_WINDOW, dict(window_t=0, window_h=1, window_w=1), 0.9),
           (_lib.PARK_FLAG_LOCAL_WINDOW, dict(window_t=3, window_h=1, window_w=1), 0.9),
           (_lib.PARK_FLAG_LOCAL_WINDOW, dict(window_t=1, window_h=1, window_w=1), 0.9)]   # 16 boxes > 4
    for flags, fields, p in bad:
        rb = _fake_retrieval()
        rb.flags = flags
        for k, v in fields.items():
            setattr(rb, k, v)
        cases.append((lib.park_retrieve(fake, fake, ctypes.byref(shape), 4, 4, p, 10, ctypes.byref(rb), fake, need,
                                        None), _lib.PARK_ERR_INVALID_ARG))
        cases.append((lib.park_layer(fake, fake, fake, ctypes.byref(shape), 4, 4, p, 10, fake, ctypes.byref(rb),
                                     fake, need, None), _lib.PARK_ERR_INVALID_ARG))
    for got, want in cases:
        assert got == want
    assert lib.park_launch_count() == before
