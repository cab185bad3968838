"""PARK block retrieval + block-sparse attention for one video-DiT attention
layer, as hand-written CUDA for sm_100a behind a C ABI (include/park.h).

The Python side only marshals arguments; importing the package does not load
the library (``_lib.load()`` does, and raises if it has not been built)."""
from .park import (Retrieval, Shape, alloc_retrieval, alloc_workspace, layer, launch_count, profile_collect,  # noqa: F401
                   profile_enable, retrieve, set_wait_limit_ns, sparse_attn, workspace_size)
