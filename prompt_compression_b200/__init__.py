"""B200 (sm_100a) lookahead importance scoring: SpecKV / SpecPC scoring, pooling,
top-k selection and KV compaction.

This package is a thin binding over ``libspeckv.so`` (the C ABI declared in
``include/speckv.h``).  The functions below marshal torch tensors into raw
device pointers, sizes and a stream and call the C entry point of the same
name; every step of the computation runs in the library's CUDA kernels.
There is no CPU fallback: if the library is missing or cannot be loaded,
every call raises.

Method: "Draft-based Approximate Inference for LLMs" (paper notes, ICLR 2026),
section 关键设计 (SpecKV, SpecPC, SpecKV-PC) and section 损失函数 / 训练策略
(local pooling).
"""
from __future__ import annotations

from .binding import (  # noqa: F401
    SpeckvError, load_library, library_path,
    speckv_workspace_size, speckv_score, speckv_row_lse, speckv_row_offsets, speckv_colsum,
    speckv_prefill_attention, specpc_workspace_size, specpc_score, specpc_row_offsets, specpc_colsum,
    topk_workspace_size, topk_select, kv_compact, decode_attention,
    spk_device_error, spk_selftest_wait_timeout, spk_exp2_fma, mapped_host_pointer,
    SPK_POOL_MAX, SPK_POOL_AVG, vs_workspace_size, vs_sparse_attention,
)
from .pipeline import speckv_compress, specpc_select, cascade_compress  # noqa: F401

__all__ = [
    "SpeckvError", "load_library", "library_path",
    "speckv_workspace_size", "speckv_score", "speckv_row_lse", "speckv_row_offsets", "speckv_colsum",
    "speckv_prefill_attention", "specpc_workspace_size", "specpc_score", "specpc_row_offsets", "specpc_colsum",
    "topk_workspace_size", "topk_select", "kv_compact", "decode_attention",
    "spk_device_error", "spk_selftest_wait_timeout", "spk_exp2_fma", "mapped_host_pointer",
    "SPK_POOL_MAX", "SPK_POOL_AVG", "vs_workspace_size", "vs_sparse_attention", "speckv_compress", "specpc_select", "cascade_compress",
]
