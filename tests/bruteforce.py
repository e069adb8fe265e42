"""Brute-force NumPy/SciPy restatements used to pin the oracle.

These materialise what the pages describe literally -- the full causal
attention matrix of every query row (SpecKV), or the draft attention tensor
A[layer][head][query position][key] over all query positions (SpecPC) --
and reduce it with library routines (scipy.special.softmax,
scipy.ndimage.maximum_filter1d / uniform_filter1d, numpy.lexsort).  They are written
independently of oracle.c and only for tiny inputs.
"""
from __future__ import annotations

import numpy as np
from scipy.ndimage import maximum_filter1d, uniform_filter1d
from scipy.special import softmax


def causal_attention(q_rows, k, positions, scale=1.0):
    """P[i, j] = softmax over keys j <= positions[i] (input keys only)."""
    q_rows = np.asarray(q_rows, np.float64)
    k = np.asarray(k, np.float64)
    n_in = k.shape[0]
    logits = scale * q_rows @ k.T
    visible = np.arange(n_in)[None, :] <= np.asarray(positions)[:, None]
    logits = np.where(visible, logits, -np.inf)
    return softmax(logits, axis=1)


def speckv_unit(q, k, n_window, n_lookahead, scale=1.0):
    """q [g,R,d], k [n_in,d] -> (scores [n_pre], window_mass [n_window])."""
    g, R, d = q.shape
    n_in = k.shape[0]
    pos = np.concatenate([np.arange(n_in - n_window, n_in), n_in + np.arange(n_lookahead)])
    total = np.zeros(n_in)
    for h in range(g):
        total += causal_attention(q[h], k, pos, scale).sum(axis=0)
    n_pre = n_in - n_window
    return total[:n_pre], total[n_pre:]


def specpc_full_attention(q_all, k, scale=1.0):
    """The draft attention tensor for one layer and head: every query position
    t in [0, n_in + n_lookahead - 1) attends to the input keys j <= t."""
    positions = np.arange(q_all.shape[0])
    return causal_attention(q_all, k, positions, scale)


def specpc_batch(q_all, k, weights, l_skip, scale=1.0):
    """q_all [L,Hq,T,d] holds queries for ALL T = n_in + n_lookahead - 1 positions.
    Builds A[l][qh] over all positions, keeps the last W rows, takes the
    weighted mean over rows and the mean over layers >= l_skip, then the
    max over query heads."""
    L, hq, T, d = q_all.shape
    _, hkv, n_in, _ = k.shape
    g = hq // hkv
    W = len(weights)
    w = np.asarray(weights, np.float64)
    per_head = np.zeros((hq, n_in))
    for l in range(l_skip, L):
        for qh in range(hq):
            A = specpc_full_attention(q_all[l, qh], k[l, qh // g], scale)   # [T, n_in]
            per_head[qh] += (w[:, None] * A[T - W:]).sum(axis=0) / w.sum()
    per_head /= (L - l_skip)
    return per_head.max(axis=0)


def maxpool(s, kernel):
    # 'nearest' edge replication gives the same maximum as clipping the window
    return maximum_filter1d(np.asarray(s, np.float64), size=kernel, mode="nearest")


def avgpool(s, kernel):
    """Mean over the clipped window: a zero-padded box sum over a zero-padded
    box count (two uniform filters with constant-0 edges, whose 1/kernel
    factors cancel)."""
    s = np.asarray(s, np.float64)
    num = uniform_filter1d(s, size=kernel, mode="constant", cval=0.0)
    den = uniform_filter1d(np.ones_like(s), size=kernel, mode="constant", cval=0.0)
    return num / den


def topk_with_tail(pooled, k, n_tail):
    pooled = np.asarray(pooled, np.float64)
    n = pooled.size
    order = np.lexsort((np.arange(n), -pooled))      # value desc, index asc
    sel = np.sort(order[:min(k, n)])
    return np.concatenate([sel, n + np.arange(n_tail)]).astype(np.int32)
