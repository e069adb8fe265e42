"""Shared helpers for the GPU parity tests: data movement and comparison rules.

Comparison rules (from the acceptance criteria of the scoring path):
  scores   |gpu - oracle| <= 1e-3 * max(|oracle|, 1e-6 * max_unit(oracle))
  indices  identical, except keys in the symmetric difference whose oracle
           pooled score lies within that tolerance of the C-th pooled score
  K/V      compacted rows are bit-exact copies of K/V at the GPU's indices
The selection kernel itself is checked bit-exactly: the oracle's pool + top-k
run on the GPU's own fp32 scores must give the GPU's indices.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

RTOL = 1e-3
FLOOR = 1e-6


def to_bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def assert_scores_close(gpu: np.ndarray, ref: np.ndarray, what="scores"):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    if ref.size == 0:
        return
    floor = FLOOR * np.abs(ref).max()
    tol = RTOL * np.maximum(np.abs(ref), floor)
    err = np.abs(gpu - ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst rel "
                           f"{(err / np.maximum(np.abs(ref), floor)).max():.3e} at {np.argmax(err / tol)}")


def assert_indices_match(gpu_idx: np.ndarray, ref_idx: np.ndarray, ref_pooled: np.ndarray, c: int):
    """Selected prefix indices (first c entries) equal up to near-threshold ties."""
    g = set(np.asarray(gpu_idx[:c]).tolist())
    r = set(np.asarray(ref_idx[:c]).tolist())
    assert len(g) == c and len(r) == c
    diff = g ^ r
    if diff:
        thr = np.sort(ref_pooled)[::-1][c - 1]
        floor = FLOOR * np.abs(ref_pooled).max()
        tol = RTOL * max(abs(thr), floor)
        far = [j for j in diff if abs(ref_pooled[j] - thr) > tol]
        assert not far, f"indices differ beyond the tie tolerance: {sorted(far)[:10]}"
    assert np.array_equal(gpu_idx[c:], ref_idx[c:]), "kept window differs"
    assert np.all(np.diff(gpu_idx[:c]) > 0), "selected indices must be ascending"


def oracle_unit(q_bits_unit: np.ndarray, k_bits_unit: np.ndarray, n_window: int, n_lookahead: int,
                c_max: int, pool: int, scale: float = 1.0):
    """Oracle scores, window mass, pooled scores and indices for one unit."""
    s, wm = oracle.speckv_unit(q_bits_unit, k_bits_unit, n_window, n_lookahead, scale)
    p = oracle.maxpool(s, pool) if s.size else s
    idx = oracle.topk_with_tail(p, c_max, n_window)
    return s, wm, p, idx
