"""Seeded generators for K/V caches, queries and label-channel indices.

Every tensor is drawn from its own PCG64 stream keyed by
(config seed, tensor id, layer, batch row, KV head), so one (row, KV head)
slice can be regenerated alone for sampled checks.  Values are drawn in
float32, combined in float64 where a formula is involved, and rounded to bf16
with round-to-nearest-even.  bf16 tensors are returned as their uint16 bit
patterns; consumers reinterpret them (torch ``view(torch.bfloat16)``) or widen
them exactly (``f32_from_bf16_bits``).

Workload recipe (the pages fix none of it; each point is this generator's
reading of the workload descriptions):
  * K/V ~ N(0, kv_std^2); ``n_outlier`` seeded channels per KV head are scaled
    by ``outlier_scale`` in both K and V.
  * Planted tokens: keys = 0.8 * q_h/|q_h| * sqrt(qk_dim) + N(0, kv_std^2)
    noise, written after outlier scaling.  Positions are spread over
    ``planted_blocks`` seeded blocks (uniform over the context when 0); in
    position order, the planted tokens of a row are split into G contiguous
    runs, run h aligning to head h of the group.
  * Label channels per KV head: the outlier channels first (when the workload
    says so) topped up with seeded channels, sorted ascending.
  * Queries: q_0 ~ N(0,1); along a trajectory
    q_t = normalize(q_{t-1} + drift * N(0,1)) * sqrt(qk_dim), in float64.
"""

from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os

import numpy as np

from .configs import WorkloadConfig

# tensor ids used as the second element of every stream key
_T_K, _T_V, _T_Q, _T_OUTLIER, _T_LABEL, _T_PLANT, _T_QDRIFT = range(7)


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _bf16_from_f64(x: np.ndarray) -> np.ndarray:
    return bf16_bits_from_f32(np.asarray(x, dtype=np.float64).astype(np.float32))


def _rng(cfg: WorkloadConfig, *key: int) -> np.random.Generator:
    ss = np.random.SeedSequence(entropy=cfg.seed, spawn_key=tuple(int(k) for k in key))
    return np.random.Generator(np.random.PCG64(ss))


def gen_outlier_channels(cfg: WorkloadConfig, kvh: int, layer: int = 0) -> np.ndarray:
    if cfg.n_outlier <= 0:
        return np.zeros(0, dtype=np.int64)
    rng = _rng(cfg, _T_OUTLIER, layer, kvh)
    return np.sort(rng.choice(cfg.qk_dim, size=cfg.n_outlier, replace=False)).astype(np.int64)


def gen_label_channels(cfg: WorkloadConfig, layer: int = 0) -> np.ndarray:
    """Label-channel indices, int32 [n_kv_heads, n_label], ascending per head."""
    out = np.zeros((cfg.n_kv_heads, cfg.n_label), dtype=np.int32)
    for kvh in range(cfg.n_kv_heads):
        rng = _rng(cfg, _T_LABEL, layer, kvh)
        chosen = []
        if cfg.label_from_outliers:
            chosen = list(gen_outlier_channels(cfg, kvh, layer)[: cfg.n_label])
        rest = np.setdiff1d(np.arange(cfg.qk_dim), np.asarray(chosen, dtype=np.int64))
        fill = rng.choice(rest, size=cfg.n_label - len(chosen), replace=False)
        out[kvh] = np.sort(np.concatenate([np.asarray(chosen, dtype=np.int64), fill]))
    return out


def gen_query_trajectory(cfg: WorkloadConfig, steps: int | None = None, layer: int = 0) -> list[np.ndarray]:
    """bf16 bits [batch, n_q_heads, qk_dim] for steps 0..steps-1."""
    steps = cfg.steps if steps is None else steps
    shape = (cfg.batch, cfg.n_q_heads, cfg.qk_dim)
    state = _rng(cfg, _T_Q, layer).standard_normal(shape, dtype=np.float64)
    drift = _rng(cfg, _T_QDRIFT, layer)
    out = [_bf16_from_f64(state)]
    for _ in range(1, steps):
        nxt = state + cfg.q_drift * drift.standard_normal(shape, dtype=np.float64)
        nxt = nxt / np.linalg.norm(nxt, axis=-1, keepdims=True) * math.sqrt(cfg.qk_dim)
        state = nxt
        out.append(_bf16_from_f64(state))
    return out


def gen_queries(cfg: WorkloadConfig, layer: int = 0) -> np.ndarray:
    return gen_query_trajectory(cfg, 1, layer)[0]


@dataclasses.dataclass
class RowInputs:
    k: np.ndarray  # uint16 bf16 bits [ctx_len, qk_dim]
    v: np.ndarray | None  # uint16 bf16 bits [ctx_len, v_dim]; None when V is a slice of K
    planted_pos: np.ndarray  # int64 token positions, ascending
    planted_head: np.ndarray  # int64 head within the group each planted token aligns to


def _planted_positions(cfg: WorkloadConfig, rng: np.random.Generator) -> np.ndarray:
    n = cfg.planted_per_row
    if n <= 0:
        return np.zeros(0, dtype=np.int64)
    if cfg.planted_blocks <= 0:
        pos = rng.choice(cfg.ctx_len, size=n, replace=False)
    else:
        blocks = rng.choice(cfg.n_blocks, size=cfg.planted_blocks, replace=False)
        pool = (blocks[:, None] * cfg.block_size + np.arange(cfg.block_size)[None, :]).ravel()
        pos = rng.choice(pool, size=n, replace=False)
    return np.asarray(pos, dtype=np.int64)


def gen_row(cfg: WorkloadConfig, b: int, kvh: int, q_bits: np.ndarray, layer: int = 0) -> RowInputs:
    """K (and V) of one (batch row, KV head) slice; ``q_bits`` is the step-0 query [B, Hq, D]."""
    n, d = cfg.ctx_len, cfg.qk_dim
    outl = gen_outlier_channels(cfg, kvh, layer)

    k = _rng(cfg, _T_K, layer, b, kvh).standard_normal((n, d), dtype=np.float32)
    if cfg.kv_std != 1.0:
        k *= np.float32(cfg.kv_std)
    if outl.size:
        k[:, outl] *= np.float32(cfg.outlier_scale)

    prng = _rng(cfg, _T_PLANT, layer, b, kvh)
    pos = _planted_positions(cfg, prng)
    pos = np.sort(pos)
    heads = (np.arange(pos.size) * cfg.group) // max(pos.size, 1)
    if pos.size:
        g0 = kvh * cfg.group
        qh = f32_from_bf16_bits(q_bits[b, g0 + heads]).astype(np.float64)
        qhat = qh / np.linalg.norm(qh, axis=-1, keepdims=True)
        noise = prng.standard_normal((pos.size, d), dtype=np.float32).astype(np.float64) * cfg.kv_std
        k[pos] = (0.8 * math.sqrt(d) * qhat + noise).astype(np.float32)
    k_bits = bf16_bits_from_f32(k)
    del k

    v_bits = None
    if cfg.separate_v:
        v = _rng(cfg, _T_V, layer, b, kvh).standard_normal((n, cfg.v_dim), dtype=np.float32)
        if cfg.kv_std != 1.0:
            v *= np.float32(cfg.kv_std)
        vo = outl[outl < cfg.v_dim]
        if vo.size:
            v[:, vo] *= np.float32(cfg.outlier_scale)
        v_bits = bf16_bits_from_f32(v)
    return RowInputs(k=k_bits, v=v_bits, planted_pos=pos, planted_head=heads.astype(np.int64))


def gen_kv(cfg: WorkloadConfig, q_bits: np.ndarray, layer: int = 0, rows=None):
    """Full caches as uint16 bf16 bits: K [B, Hkv, N, Dqk], V [B, Hkv, N, Dv] (None for MLA)."""
    kk = np.empty((cfg.batch, cfg.n_kv_heads, cfg.ctx_len, cfg.qk_dim), dtype=np.uint16)
    vv = None
    if cfg.separate_v:
        vv = np.empty((cfg.batch, cfg.n_kv_heads, cfg.ctx_len, cfg.v_dim), dtype=np.uint16)
    planted = {}
    todo = [(b, h) for b in range(cfg.batch) for h in range(cfg.n_kv_heads) if rows is None or (b, h) in rows]

    def one(bh):
        b, h = bh
        r = gen_row(cfg, b, h, q_bits, layer)
        kk[b, h] = r.k
        if vv is not None:
            vv[b, h] = r.v
        return bh, (r.planted_pos, r.planted_head)

    # rows draw from independent streams, so threads change no value
    with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        for bh, pl in ex.map(one, todo):
            planted[bh] = pl
    return kk, vv, planted
