"""Seeded synthetic workloads for lookahead importance scoring.

This module is shared by the oracle-side tests and the GPU path.  It holds
the workload shapes and the seeded input generators only: none of the
scoring, pooling, selection or compaction arithmetic lives here.

Workload shapes follow the model shapes named for SpecKV / SpecPC in
"Draft-based Approximate Inference for LLMs" (paper notes, ICLR 2026):
section "主实验" (Table 1: Qwen2.5-32B target, C_max = 256) and section
"关键设计" (SpecKV, SpecPC, SpecKV-PC).  The pages publish no kernel-level
workload, so the inputs are Gaussian stand-ins for the LongBench / RULER
contexts the pages evaluate on: Q, K, V ~ N(0, 1) with an attention sink at
key 0 and planted "heavy" keys that share a random unit direction u_h with
the queries of their KV head, so that importance has structure to recover.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

__all__ = [
    "SpecKVConfig", "SpecPCConfig", "CascadeConfig", "CONFIGS",
    "bf16_round", "bf16_bits", "bf16_decode",
    "tiny_speckv_numpy", "heavy_positions", "speckv_inputs", "specpc_inputs",
    "specpc_row_weights", "speckv_unit_numpy", "specpc_layer_numpy", "VSConfig", "vs_pattern",
]


@dataclasses.dataclass(frozen=True)
class SpecKVConfig:
    """Shape of one SpecKV scoring job.

    A unit is one (batch, layer, KV head).  Each unit scores the keys of its
    n_in input tokens with the queries of the last n_window input tokens
    plus the n_lookahead draft tokens, for every query head of the GQA group.
    """
    name: str
    batch: int
    layers: int
    hq: int
    hkv: int
    head_dim: int
    n_in: int
    n_window: int
    n_lookahead: int
    c_max: int
    pool: int = 7
    heavy_frac: float = 0.02
    heavy_spans: int = 0          # clustered heavy keys: number of spans
    span_len: int = 32
    q_offset: float = 1.5
    sink: float = 4.0
    heavy: float = 3.0

    @property
    def g(self) -> int:
        return self.hq // self.hkv

    @property
    def rows(self) -> int:            # R: query rows per query head
        return self.n_window + self.n_lookahead

    @property
    def n_pre(self) -> int:
        return self.n_in - self.n_window

    @property
    def units(self) -> int:
        return self.batch * self.layers * self.hkv

    @property
    def kv_head_tokens(self) -> int:
        return self.units * self.n_in

    @property
    def keep(self) -> int:             # rows kept per unit
        return min(self.c_max, self.n_pre) + self.n_window


@dataclasses.dataclass(frozen=True)
class SpecPCConfig:
    """Shape of one SpecPC scoring job (draft-model attention aggregation).

    Queries are the last n_rows (W) query positions of the draft; layers
    below l_skip are skipped; scores are per (batch, input token).
    """
    name: str
    batch: int
    layers: int
    l_skip: int
    hq: int
    hkv: int
    head_dim: int
    n_in: int
    n_rows: int
    n_lookahead: int
    keep: int
    pool: int = 7
    heavy_frac: float = 0.01
    q_offset: float = 1.5
    sink: float = 0.0
    heavy: float = 3.0

    @property
    def g(self) -> int:
        return self.hq // self.hkv

    @property
    def layers_used(self) -> int:
        return self.layers - self.l_skip

    @property
    def units(self) -> int:
        return self.batch * self.layers_used * self.hkv

    @property
    def kv_head_tokens(self) -> int:
        return self.units * self.n_in


@dataclasses.dataclass(frozen=True)
class CascadeConfig:
    """SpecPC on the draft selects prompt tokens; SpecKV then runs on the
    target K/V gathered at those tokens (section "关键设计", SpecKV-PC)."""
    name: str
    draft: SpecPCConfig
    target: SpecKVConfig          # n_in of target = draft.keep (gathered)
    n_in_full: int                # tokens before the SpecPC gather


@dataclasses.dataclass(frozen=True)
class DecodeConfig:
    """One decode step (one new query token per head) over the cache that
    SpecKV leaves (section "整体框架": the target then runs on the compressed
    cache), and, for contrast, over the full cache."""
    name: str
    batch: int
    layers: int
    hq: int
    hkv: int
    head_dim: int
    n_kv: int                     # kept rows per KV head (C_max + n_window)
    n_kv_full: int                # rows of the uncompressed cache

    @property
    def units(self) -> int:
        return self.batch * self.layers * self.hkv


@dataclasses.dataclass(frozen=True)
class VSConfig:
    """Vertical-Slash sparse prefill over an n-token sequence (section
    "损失函数 / 训练策略": SpecKV's target prefill is Vertical-Slash sparse).
    Query rows are the last n_q positions; per unit (batch, layer, KV head) the
    pattern has n_vertical key columns (the sink and random keys) and
    n_local + n_far diagonals (offsets 0 .. n_local-1 and random far ones)."""
    name: str
    batch: int
    layers: int
    hq: int
    hkv: int
    head_dim: int
    n: int
    n_q: int
    n_vertical: int
    n_local: int
    n_far: int

    @property
    def g(self) -> int:
        return self.hq // self.hkv

    @property
    def units(self) -> int:
        return self.batch * self.layers * self.hkv

    @property
    def n_slash(self) -> int:
        return self.n_local + self.n_far


TINY = SpecKVConfig("tiny_speckv", batch=1, layers=1, hq=4, hkv=2, head_dim=64,
                    n_in=512, n_window=16, n_lookahead=16, c_max=64, pool=7)
LLAMA8B_16K = SpecKVConfig("llama3.1-8b_speckv_16k", batch=1, layers=32, hq=32, hkv=8,
                           head_dim=128, n_in=16384, n_window=64, n_lookahead=64,
                           c_max=256, heavy_frac=0.02)
QWEN32B_64K = SpecKVConfig("qwen2.5-32b_speckv_64k", batch=1, layers=64, hq=40, hkv=8,
                           head_dim=128, n_in=65536, n_window=64, n_lookahead=128,
                           c_max=256, heavy_frac=0.01, heavy_spans=8, span_len=32)
QWEN05B_SPECPC_32K = SpecPCConfig("qwen2.5-0.5b_specpc_32k", batch=1, layers=24, l_skip=4,
                                  hq=14, hkv=2, head_dim=64, n_in=32768, n_rows=256,
                                  n_lookahead=1, keep=2048)
CASCADE_128K = CascadeConfig(
    "cascade_specpc_speckv_128k",
    draft=SpecPCConfig("cascade_draft_128k", batch=2, layers=24, l_skip=4, hq=14, hkv=2,
                       head_dim=64, n_in=131072, n_rows=256, n_lookahead=1, keep=2048),
    target=SpecKVConfig("cascade_target_2k", batch=2, layers=32, hq=32, hkv=8, head_dim=128,
                        n_in=2048, n_window=64, n_lookahead=64, c_max=256, heavy_frac=0.01),
    n_in_full=131072)

DECODE_QWEN32B = DecodeConfig("qwen2.5-32b_decode_compressed", batch=1, layers=64, hq=40, hkv=8,
                              head_dim=128, n_kv=320, n_kv_full=65536)

VS_LLAMA8B_16K = VSConfig("llama3.1-8b_vs_prefill_16k", batch=1, layers=32, hq=32, hkv=8, head_dim=128,
                          n=16384, n_q=16384, n_vertical=1024, n_local=64, n_far=16)

CONFIGS = {c.name: c for c in (TINY, LLAMA8B_16K, QWEN32B_64K, QWEN05B_SPECPC_32K, CASCADE_128K,
                               DECODE_QWEN32B, VS_LLAMA8B_16K)}


# ---------------------------------------------------------------------------
# bf16 encoding (round to nearest even), used to hand both sides the same bytes
# ---------------------------------------------------------------------------

def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 array -> uint16 bf16 bit patterns, round-to-nearest-even."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_decode(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> fp32 values (exact)."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    return bf16_decode(bf16_bits(x))


# ---------------------------------------------------------------------------
# generators
# ---------------------------------------------------------------------------

def _unit(v: np.ndarray) -> np.ndarray:
    return v / np.linalg.norm(v, axis=-1, keepdims=True)


def tiny_speckv_numpy(seed: int = 0, cfg: SpecKVConfig = TINY, heavy=(100, 101, 102, 103)):
    """The tiny SpecKV workload, in fp32, from np.random.default_rng(seed).

    Draw order: Q, K, V, then one unit vector u_h per KV head.  Key 0 gets
    +sink*u_h, the listed heavy keys +heavy*u_h, every query row of the
    group +q_offset*u_h; Q is then scaled by 1/sqrt(head_dim).
    Returns fp32 arrays q [B,L,Hq,R,d], k, v [B,L,Hkv,n_in,d].
    """
    rng = np.random.default_rng(seed)
    B, L, d = cfg.batch, cfg.layers, cfg.head_dim
    q = rng.standard_normal((B, L, cfg.hq, cfg.rows, d)).astype(np.float32)
    k = rng.standard_normal((B, L, cfg.hkv, cfg.n_in, d)).astype(np.float32)
    v = rng.standard_normal((B, L, cfg.hkv, cfg.n_in, d)).astype(np.float32)
    u = _unit(rng.standard_normal((B, L, cfg.hkv, d))).astype(np.float32)
    k[:, :, :, 0, :] += cfg.sink * u
    for j in heavy:
        k[:, :, :, j, :] += cfg.heavy * u
    q += cfg.q_offset * np.repeat(u, cfg.g, axis=2)[:, :, :, None, :]
    q *= np.float32(1.0 / math.sqrt(d))
    return q, k, v


def heavy_positions(n_cand: int, frac: float, spans: int, span_len: int, seed: int,
                    lo: int = 1) -> np.ndarray:
    """Planted heavy key positions in [lo, n_cand), shared by all layers and
    heads of a batch element.  With spans > 0, spans*span_len of them form
    non-overlapping clustered runs and the rest are uniform."""
    rng = np.random.default_rng(seed)
    total = max(1, int(round(frac * n_cand)))
    chosen = np.zeros(n_cand, dtype=bool)
    if spans > 0:
        n_slots = (n_cand - lo) // span_len
        slots = rng.choice(n_slots, size=min(spans, n_slots), replace=False)
        for s in slots:
            chosen[lo + s * span_len: lo + (s + 1) * span_len] = True
    rest = total - int(chosen.sum())
    if rest > 0:
        free = np.flatnonzero(~chosen[lo:]) + lo
        chosen[rng.choice(free, size=min(rest, free.size), replace=False)] = True
    return np.flatnonzero(chosen).astype(np.int64)


def _torch():
    import torch
    return torch


def speckv_inputs(cfg: SpecKVConfig, seed: int = 0, device="cpu", with_v: bool = True,
                  heavy_pos: Optional[np.ndarray] = None):
    """bf16 SpecKV inputs on `device`, generated layer by layer.

    Returns dict(q=[B,L,Hq,R,d], k=[B,L,Hkv,n_in,d], v=..., heavy=positions).
    Heavy positions are drawn in [1, n_pre) (the scored prefix), per batch
    element, unless heavy_pos gives them (one array per batch element); u_h
    is drawn per (batch, layer, KV head).
    """
    torch = _torch()
    B, L, Hq, Hkv, d = cfg.batch, cfg.layers, cfg.hq, cfg.hkv, cfg.head_dim
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = torch.empty((B, L, Hq, cfg.rows, d), dtype=torch.bfloat16, device=device)
    k = torch.empty((B, L, Hkv, cfg.n_in, d), dtype=torch.bfloat16, device=device)
    v = torch.empty_like(k) if with_v else None
    heavy = []
    for b in range(B):
        hp = heavy_pos[b] if heavy_pos is not None else heavy_positions(
            max(cfg.n_pre, 2), cfg.heavy_frac, cfg.heavy_spans, cfg.span_len, seed * 1000 + b)
        heavy.append(np.asarray(hp, dtype=np.int64))
    inv = 1.0 / math.sqrt(d)
    for l in range(L):
        kl = torch.randn((B, Hkv, cfg.n_in, d), generator=gen, device=device, dtype=torch.float32)
        ql = torch.randn((B, Hq, cfg.rows, d), generator=gen, device=device, dtype=torch.float32)
        u = torch.randn((B, Hkv, d), generator=gen, device=device, dtype=torch.float32)
        u = u / u.norm(dim=-1, keepdim=True)
        kl[:, :, 0, :] += cfg.sink * u
        for b in range(B):
            idx = torch.as_tensor(heavy[b], device=device)
            kl[b][:, idx, :] += cfg.heavy * u[b][:, None, :]
        ql += cfg.q_offset * u.repeat_interleave(cfg.g, dim=1)[:, :, None, :]
        ql *= inv
        k[:, l].copy_(kl)
        q[:, l].copy_(ql)
        if with_v:
            v[:, l].copy_(torch.randn((B, Hkv, cfg.n_in, d), generator=gen, device=device,
                                      dtype=torch.float32))
        del kl, ql
    return {"q": q, "k": k, "v": v, "heavy": heavy}


def specpc_row_weights(n_rows: int) -> np.ndarray:
    """Query-row weights of SpecPC: linear from 0.1 (oldest row) to 1 (last row).

    Section "关键设计" (SpecPC): rows further from the end weigh less.  The
    pages do not print the endpoints' formula; the linear 1 -> 0.1 ramp is
    the workload's own statement.  W = 1 gives the single weight 1.
    """
    if n_rows == 1:
        return np.ones(1, dtype=np.float64)
    i = np.arange(n_rows, dtype=np.float64)
    return 0.1 + 0.9 * i / (n_rows - 1)


def specpc_inputs(cfg: SpecPCConfig, seed: int = 0, device="cpu", heavy_pos=None):
    """bf16 SpecPC draft inputs: q [B,L,Hq,W,d], k [B,L,Hkv,n_in,d] (all layers
    are generated; scoring skips l < l_skip).  Heavy keys in [1, n_in)."""
    torch = _torch()
    B, L, Hq, Hkv, d = cfg.batch, cfg.layers, cfg.hq, cfg.hkv, cfg.head_dim
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = torch.empty((B, L, Hq, cfg.n_rows, d), dtype=torch.bfloat16, device=device)
    k = torch.empty((B, L, Hkv, cfg.n_in, d), dtype=torch.bfloat16, device=device)
    heavy = []
    for b in range(B):
        hp = heavy_pos[b] if heavy_pos is not None else heavy_positions(
            cfg.n_in, cfg.heavy_frac, 0, 32, seed * 1000 + b)
        heavy.append(np.asarray(hp, dtype=np.int64))
    inv = 1.0 / math.sqrt(d)
    for l in range(L):
        kl = torch.randn((B, Hkv, cfg.n_in, d), generator=gen, device=device, dtype=torch.float32)
        ql = torch.randn((B, Hq, cfg.n_rows, d), generator=gen, device=device, dtype=torch.float32)
        u = torch.randn((B, Hkv, d), generator=gen, device=device, dtype=torch.float32)
        u = u / u.norm(dim=-1, keepdim=True)
        if cfg.sink:
            kl[:, :, 0, :] += cfg.sink * u
        for b in range(B):
            idx = torch.as_tensor(heavy[b], device=device)
            kl[b][:, idx, :] += cfg.heavy * u[b][:, None, :]
        ql += cfg.q_offset * u.repeat_interleave(cfg.g, dim=1)[:, :, None, :]
        ql *= inv
        k[:, l].copy_(kl)
        q[:, l].copy_(ql)
        del kl, ql
    return {"q": q, "k": k, "heavy": heavy}


def speckv_unit_numpy(cfg: SpecKVConfig, seed: int, unit: int):
    """One unit's inputs (bf16 bit patterns) drawn on the host with numpy:
    q [g, R, d], k [n_in, d], v [n_in, d], same distribution as speckv_inputs
    (sink, heavy keys with the clustered layout of the config, query offset)."""
    rng = np.random.default_rng([seed, unit])
    d, g = cfg.head_dim, cfg.g
    q = rng.standard_normal((g, cfg.rows, d)).astype(np.float32)
    k = rng.standard_normal((cfg.n_in, d)).astype(np.float32)
    v = rng.standard_normal((cfg.n_in, d)).astype(np.float32)
    u = _unit(rng.standard_normal(d)).astype(np.float32)
    hp = heavy_positions(max(cfg.n_pre, 2), cfg.heavy_frac, cfg.heavy_spans, cfg.span_len, seed * 1000)
    k[0] += cfg.sink * u
    k[hp] += cfg.heavy * u
    q += cfg.q_offset * u
    q *= np.float32(1.0 / math.sqrt(d))
    return bf16_bits(q), bf16_bits(k), bf16_bits(v)


def specpc_layer_numpy(cfg: SpecPCConfig, seed: int, b: int, layer: int):
    """One (batch element, layer) of a SpecPC draft drawn on the host with
    numpy: q [Hq, W, d], k [Hkv, n_in, d] (bf16 bit patterns), with the
    distribution of specpc_inputs (heavy keys of the batch element, one u_h
    per KV head, query offset; its own random stream)."""
    rng = np.random.default_rng([seed, b, layer])
    d = cfg.head_dim
    q = rng.standard_normal((cfg.hq, cfg.n_rows, d)).astype(np.float32)
    k = rng.standard_normal((cfg.hkv, cfg.n_in, d)).astype(np.float32)
    u = _unit(rng.standard_normal((cfg.hkv, d))).astype(np.float32)
    hp = heavy_positions(cfg.n_in, cfg.heavy_frac, 0, 32, seed * 1000 + b)
    if cfg.sink:
        k[:, 0] += cfg.sink * u
    k[:, hp] += cfg.heavy * u[:, None, :]
    q += cfg.q_offset * np.repeat(u, cfg.g, axis=0)[:, None, :]
    q *= np.float32(1.0 / math.sqrt(d))
    return bf16_bits(q), bf16_bits(k)


def vs_pattern(cfg: VSConfig, seed: int = 0, device="cpu"):
    """Seeded Vertical-Slash pattern per unit: vertical = key 0 plus random
    distinct keys, slash = offsets 0 .. n_local-1 plus random distinct far
    offsets; both ascending int32 [units, count]."""
    torch = _torch()
    rng = np.random.default_rng(seed)
    vert = np.zeros((cfg.units, cfg.n_vertical), np.int32)
    sl = np.zeros((cfg.units, cfg.n_slash), np.int32)
    for u in range(cfg.units):
        if cfg.n_vertical:
            v = rng.choice(np.arange(1, cfg.n), size=cfg.n_vertical - 1, replace=False)
            vert[u] = np.sort(np.concatenate([[0], v]))
        far = rng.choice(np.arange(cfg.n_local, cfg.n), size=cfg.n_far, replace=False)
        sl[u] = np.sort(np.concatenate([np.arange(cfg.n_local), far]))
    return torch.from_numpy(vert).to(device), torch.from_numpy(sl).to(device)
