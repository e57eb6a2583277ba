"""Oracle: the AsyncTLS two-level sparse decode step, written out plainly.

TEST INFRASTRUCTURE.  Only tests/, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module.  It is numpy in float64, row by row, with no blocking, fusion or
reordering beyond what the definitions state, so that a reader can check each
function against the pages by eye.  It shares no code, constants or helpers
with the CUDA library.

Sources (five web pages on "AsyncTLS: Efficient Generative LLM Inference with
Asynchronous Two-level Sparse Attention"; cited by page and section):
  [EN 2A-1]  English summary, "2. Methodology", A. Hierarchical Two-Level Sparse
             Attention, Stage 1: Coarse-Grained Block Filtering (blocks, block
             index, GEMM reformulation of the Quest score, top-K_b).
  [EN 2A-2]  same section, Stage 2: Fine-Grained Token Selection (Double-Sparsity
             token selection, channel selection, INT4 keys, top-K_t).
  [EN 2B]    same page, B. Asynchronous Offloading Engine (temporal locality,
             staggered execution, incremental transfer T_t = M_t \\ C_t).
  [IT 2A.1]  Italian summary, "2. Metodologia", A.1 Filtraggio a Livello di
             Blocco: the block representation is the max/min of the keys.
  [IT 2A.2]  same page, A.2: attention is computed only on the selected tokens.
  [JA 2A/2B] Japanese summary, "2. 提案手法", A and B (same steps).

Readings where the pages are silent (each is listed in the design notes):
  * Block score: Quest's upper bound sum_c max(q_c*kmax_c, q_c*kmin_c).
  * Heads sharing a KV head combine by max, at both levels; the selection is
    per KV head and shared by the group.
  * INT4: symmetric per token, s = max_r |x_r| / 7 in float32 (IEEE division),
    code = round-half-even(x / s) in float32, clamped to [-7, 7]; s = 0 gives
    all-zero codes.  Packing: byte j holds channel 2j in the low nibble and
    2j+1 in the high nibble, two's complement.
  * Token score: max over the group's heads of s_t * sum_r q_h[label_r]*code_r
    (no softmax scale; it does not change the ranking).
  * Ties: higher score first, then lower index; index lists come out ascending.
  * Staggering: attend(t) uses blocks chosen with q_{t-1}, tokens and
    attention with q_t.
  * A sequence holds its first n tokens; its blocks are the ceil(n / bs)
    blocks those tokens fall in, the last one possibly partial, whose index
    is the max/min of the keys it holds.  Candidates are the held positions
    of the chosen blocks; a selection asked for more than there are takes
    them all.  Attention over no token gives a zero output and lse -inf.
  * Operator baselines [EN 4]: full attention (every held token), block
    selection alone (every token of the top-K_b blocks, Quest) and token
    selection alone (the top-k over every held token, Double Sparsity).

Pins (tests that tie each function to something other than itself) are in
tests/test_oracle_pins.py.  Parity of the *quality* of a selection (does it
find the tokens a real model needs?) is unpinned: the pages print no values.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "widen_bf16",
    "block_meta",
    "quant_label",
    "pack_codes",
    "unpack_codes",
    "block_scores",
    "group_max",
    "topk_ascending",
    "candidate_tokens",
    "token_scores",
    "attention",
    "decode_row",
    "staggered_row",
    "plan_transfer",
    "dense_row",
    "quest_row",
    "ds_row",
]


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# Index build  [EN 2A-1] blocks + block-level index; [IT 2A.1] max/min of keys
# --------------------------------------------------------------------------

def block_meta(k_bits: np.ndarray, block_size: int):
    """Per-block, per-channel max and min of the keys of one (row, KV head).

    k_bits: uint16 [N, D], the tokens the sequence holds.  Block j holds
    tokens j*bs .. min(N, (j+1)*bs) - 1, so the last block may be partial.
    Returns (kmax, kmin) as float64 [ceil(N/block_size), D]; both are bf16
    values (max/min selects an input, so no rounding happens).
    """
    k = widen_bf16(k_bits)
    n, d = k.shape
    nb = -(-n // block_size)
    kmax = np.empty((nb, d))
    kmin = np.empty((nb, d))
    for j in range(nb):
        rows = k[j * block_size:(j + 1) * block_size]
        kmax[j] = rows.max(axis=0)
        kmin[j] = rows.min(axis=0)
    return kmax, kmin


def quant_label(k_bits: np.ndarray, label_ch: np.ndarray):
    """INT4 label cache of one (row, KV head) [EN 2A-2: channel selection + INT4].

    Returns codes int8 [N, R] in [-7, 7] and scales float32 [N].
    """
    x = widen_bf16(k_bits)[:, np.asarray(label_ch, dtype=np.int64)].astype(np.float32)
    n = x.shape[0]
    codes = np.zeros(x.shape, dtype=np.int8)
    scales = np.zeros(n, dtype=np.float32)
    for t in range(n):
        m = np.float32(np.max(np.abs(x[t])))
        s = np.float32(m / np.float32(7.0))
        scales[t] = s
        if s == 0:
            continue
        q = np.rint(x[t] / s)  # float32 IEEE division, round half to even
        codes[t] = np.clip(q, -7, 7).astype(np.int8)
    return codes, scales


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """int8 [N, R] -> uint8 [N, R/2]; low nibble = even channel."""
    c = np.asarray(codes, dtype=np.int64) & 0xF
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.int64)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.int64)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    out[out >= 8] -= 16
    return out.astype(np.int8)


# --------------------------------------------------------------------------
# Level 1: block scores and top-K_b  [EN 2A-1], [IT 2A.1], [JA 2A]
# --------------------------------------------------------------------------

def block_scores(q: np.ndarray, kmax: np.ndarray, kmin: np.ndarray) -> np.ndarray:
    """Quest upper bound per head and block: S[h, j] = sum_c max(q_hc*kmax_jc, q_hc*kmin_jc).

    q: float64 [G, D] (the query heads that share this KV head).
    """
    g = q.shape[0]
    nb = kmax.shape[0]
    s = np.empty((g, nb))
    for h in range(g):
        s[h] = np.maximum(q[h][None, :] * kmax, q[h][None, :] * kmin).sum(axis=1)
    return s


def group_max(per_head: np.ndarray) -> np.ndarray:
    """Combine the heads that share a KV head: max over the group."""
    return per_head.max(axis=0)


def topk_ascending(scores: np.ndarray, k: int) -> np.ndarray:
    """The k best indices by (higher score, then lower index), returned ascending.

    NaN scores rank as -inf.
    """
    s = np.asarray(scores, dtype=np.float64).copy()
    s[np.isnan(s)] = -np.inf
    n = s.size
    order = sorted(range(n), key=lambda i: (-s[i], i))
    return np.sort(np.asarray(order[:k], dtype=np.int64))


# --------------------------------------------------------------------------
# Level 2: token scores inside the chosen blocks and top-k  [EN 2A-2], [JA 2A]
# --------------------------------------------------------------------------

def candidate_tokens(block_idx: np.ndarray, block_size: int, n_tokens: int | None = None) -> np.ndarray:
    """All token positions of the chosen blocks that the sequence holds
    (below n_tokens, when given), ascending."""
    b = np.sort(np.asarray(block_idx, dtype=np.int64))
    c = (b[:, None] * block_size + np.arange(block_size)[None, :]).ravel()
    return c if n_tokens is None else c[c < n_tokens]


def token_scores(q: np.ndarray, label_ch: np.ndarray, codes: np.ndarray,
                 scales: np.ndarray, cand: np.ndarray) -> np.ndarray:
    """Approximate score of each candidate token from its INT4 label keys.

    score(t) = max_h scale_t * sum_r q_h[label_r] * code_{t,r}.
    """
    ql = q[:, np.asarray(label_ch, dtype=np.int64)]  # [G, R]
    c = codes[cand].astype(np.float64)  # [n, R]
    dots = c @ ql.T  # [n, G]
    per_head = scales[cand].astype(np.float64)[:, None] * dots
    return per_head.max(axis=1)


# --------------------------------------------------------------------------
# Attention over the chosen tokens only  [IT 2A.2]
# --------------------------------------------------------------------------

def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, softmax_scale: float):
    """Softmax attention of G heads over n rows; returns (out [G, Dv], lse [G]).

    lse is the natural log of sum_t exp(scale * q.k_t).  With no row the
    output is zero and lse is -inf (an empty sum).
    """
    if k.shape[0] == 0:
        return np.zeros((q.shape[0], v.shape[1])), np.full(q.shape[0], -np.inf)
    logits = softmax_scale * (q @ k.T)  # [G, n]
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    l = p.sum(axis=1, keepdims=True)
    out = (p @ v) / l
    lse = (m + np.log(l))[:, 0]
    return out, lse


# --------------------------------------------------------------------------
# One decode step of one (batch row, KV head)
# --------------------------------------------------------------------------

def decode_row(q_bits_group: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray | None,
               label_ch: np.ndarray, block_size: int, K_b: int, k: int,
               softmax_scale: float, v_offset: int = -1, v_dim: int | None = None,
               meta=None, label=None, q_blocks_bits: np.ndarray | None = None,
               block_idx: np.ndarray | None = None, token_idx: np.ndarray | None = None):
    """Level 1, level 2 and attention for one row.

    q_bits_group: uint16 [G, D]; k_bits uint16 [N, D]; v_bits uint16 [N, Dv]
    or None when V is the K row slice [v_offset, v_offset + v_dim).
    q_blocks_bits: the query used for level 1 (default: the same query);
    passing q_{t-1} gives the staggered step.  ``block_idx`` / ``token_idx``
    override a level's choice (used to re-run later stages on another
    implementation's selection).
    """
    q = widen_bf16(q_bits_group)
    qb = q if q_blocks_bits is None else widen_bf16(q_blocks_bits)
    if meta is None:
        meta = block_meta(k_bits, block_size)
    kmax, kmin = meta
    if label is None:
        label = quant_label(k_bits, label_ch)
    codes, scales = label

    per_head = block_scores(qb, kmax, kmin)
    agg = group_max(per_head)
    if block_idx is None:
        block_idx = topk_ascending(agg, K_b)
    cand = candidate_tokens(block_idx, block_size, k_bits.shape[0])
    ts = token_scores(q, label_ch, codes, scales, cand)
    if token_idx is None:
        token_idx = cand[topk_ascending(ts, k)]
    kf = widen_bf16(k_bits[token_idx])
    if v_bits is None:
        vf = kf[:, v_offset:v_offset + v_dim]
    else:
        vf = widen_bf16(v_bits[token_idx])
    out, lse = attention(q, kf, vf, softmax_scale)
    return {
        "agg": agg,
        "block_idx": np.asarray(block_idx, dtype=np.int64),
        "cand": cand,
        "token_score": ts,
        "token_idx": np.asarray(token_idx, dtype=np.int64),
        "out": out,
        "lse": lse,
    }


def staggered_row(q_prev_bits: np.ndarray, q_cur_bits: np.ndarray, *args, **kw):
    """Step t of the staggered engine [EN 2B]: blocks from q_{t-1}, the rest from q_t."""
    return decode_row(q_cur_bits, *args, q_blocks_bits=q_prev_bits, **kw)


def plan_transfer(new_blocks, resident_blocks) -> np.ndarray:
    """Incremental transfer set T_t = M_t \\ C_t [EN 2B], ascending."""
    m = set(int(b) for b in new_blocks)
    c = set(int(b) for b in resident_blocks)
    return np.asarray(sorted(m - c), dtype=np.int64)


# --------------------------------------------------------------------------
# Operator baselines  [EN 4] (full attention, Quest alone, Double Sparsity alone)
# --------------------------------------------------------------------------

def dense_row(q_bits_group, k_bits, v_bits, softmax_scale, v_offset=-1, v_dim=None):
    """Full attention of the group's heads over every token the sequence holds."""
    kf = widen_bf16(k_bits)
    vf = kf[:, v_offset:v_offset + v_dim] if v_bits is None else widen_bf16(v_bits)
    return attention(widen_bf16(q_bits_group), kf, vf, softmax_scale)


def quest_row(q_bits_group, k_bits, v_bits, label_ch, block_size, K_b, softmax_scale, block_idx=None, **kw):
    """Block selection alone: level 1, then attention over every token of the
    K_b blocks (a token budget of K_b * bs takes every candidate)."""
    return decode_row(q_bits_group, k_bits, v_bits, label_ch, block_size, K_b, K_b * block_size, softmax_scale,
                      block_idx=block_idx, **kw)


def ds_row(q_bits_group, k_bits, v_bits, label_ch, block_size, k, softmax_scale, token_idx=None, **kw):
    """Token selection alone: level 2 over every block of the sequence, then attention."""
    nb = -(-k_bits.shape[0] // block_size)
    return decode_row(q_bits_group, k_bits, v_bits, label_ch, block_size, nb, k, softmax_scale,
                      block_idx=np.arange(nb), token_idx=token_idx, **kw)


def softmax_scale_for(qk_dim: int) -> float:
    return 1.0 / math.sqrt(qk_dim)
