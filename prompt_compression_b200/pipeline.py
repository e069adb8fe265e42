"""End-to-end compositions of the C entry points (allocation by torch only).

speckv_compress   scores -> pool + top-C_max + window -> compacted K/V
specpc_select     SpecPC scores -> pool + top-K prompt tokens
cascade_compress  SpecPC on the draft, gather the target K/V at the kept
                  tokens, then SpecKV on the gathered cache (SpecKV-PC)

"Draft-based Approximate Inference for LLMs" (paper notes), section 关键设计.
"""
from __future__ import annotations

from typing import Optional

import torch

from . import binding as B


class SpeckvBuffers:
    """Preallocated outputs and scratch for repeated speckv_compress calls."""

    def __init__(self, q, k, v, n_window: int, c_max: int, window_mass: bool = False,
                 with_pooled: bool = False):
        Bsz, L, hq, R, d = q.shape
        _, _, hkv, n_in, _ = k.shape
        units = Bsz * L * hkv
        n_pre = n_in - n_window
        keep = min(c_max, n_pre) + n_window
        dev = q.device
        shape = B.speckv_shape(q, k, n_window)
        self.units, self.n_pre, self.keep = units, n_pre, keep
        self.scores = torch.empty((units, n_pre), dtype=torch.float32, device=dev)
        self.window_mass = (torch.empty((units, n_window), dtype=torch.float32, device=dev)
                            if window_mass else None)
        self.pooled = torch.empty_like(self.scores) if with_pooled else None
        self.idx = torch.empty((units, keep), dtype=torch.int32, device=dev)
        self.k_out = torch.empty((Bsz, L, hkv, keep, d), dtype=k.dtype, device=dev)
        self.v_out = torch.empty((Bsz, L, hkv, keep, d), dtype=v.dtype, device=dev) if v is not None else None
        self.ws_score = torch.empty(max(B.speckv_workspace_size(shape), 256), dtype=torch.uint8, device=dev)
        self.ws_topk = torch.empty(max(B.topk_workspace_size(units, n_pre), 256), dtype=torch.uint8,
                                   device=dev)


def speckv_compress(q, k, v, n_window: int, c_max: int, pool: int = 7, scale: float = 1.0,
                    buffers: Optional[SpeckvBuffers] = None, window_mass: bool = False, stream=None,
                    pool_mode: int = B.SPK_POOL_MAX):
    """SpecKV on every unit: returns the buffers object (scores, idx, k_out, v_out).
    pool_mode: B.SPK_POOL_MAX (the workloads' max pool) or B.SPK_POOL_AVG."""
    buf = buffers or SpeckvBuffers(q, k, v, n_window, c_max, window_mass=window_mass)
    B.speckv_score(q, k, n_window, buf.scores, buf.window_mass, buf.ws_score, scale, stream)
    B.topk_select(buf.scores, c_max, n_window, buf.idx, pool, buf.pooled, buf.ws_topk, stream, pool_mode)
    B.kv_compact(k, v, buf.idx, buf.k_out, buf.v_out, 1, stream)
    return buf


def specpc_select(q, k, row_weights, l_skip: int, keep: int, pool: int = 7, n_lookahead: int = 1,
                  scale: float = 1.0, scores=None, idx=None, stream=None, pool_mode: int = B.SPK_POOL_MAX):
    """SpecPC prompt-token selection: (scores [B, n_in], idx [B, min(keep, n_in)])."""
    Bsz = q.shape[0]
    n_in = k.shape[3]
    if scores is None:
        scores = torch.empty((Bsz, n_in), dtype=torch.float32, device=q.device)
    if idx is None:
        idx = torch.empty((Bsz, min(keep, n_in)), dtype=torch.int32, device=q.device)
    B.specpc_score(q, k, row_weights, scores, l_skip, n_lookahead, None, scale, stream)
    B.topk_select(scores, keep, 0, idx, pool, None, None, stream, pool_mode)
    return scores, idx


def cascade_compress(draft_q, draft_k, row_weights, l_skip: int, keep: int, target_q, target_k, target_v,
                     n_window: int, c_max: int, pool: int = 7, stream=None):
    """SpecKV-PC: SpecPC keeps `keep` prompt tokens, the target K/V are gathered
    at them (one index row per batch element, shared by every layer and KV
    head), then SpecKV keeps c_max + n_window of the gathered tokens."""
    Bsz, L, hkv, n_full, d = target_k.shape
    pc_scores, pc_idx = specpc_select(draft_q, draft_k, row_weights, l_skip, keep, pool, stream=stream)
    n_keep = pc_idx.shape[1]
    k_g = torch.empty((Bsz, L, hkv, n_keep, d), dtype=target_k.dtype, device=target_k.device)
    v_g = torch.empty_like(k_g)
    B.kv_compact(target_k, target_v, pc_idx, k_g, v_g, L * hkv, stream)
    out = speckv_compress(target_q, k_g, v_g, n_window, c_max, pool, stream=stream)
    return pc_scores, pc_idx, k_g, v_g, out
