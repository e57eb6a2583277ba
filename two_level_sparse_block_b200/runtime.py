"""Device-resident state for the decode step, built on the C ABI.

``DecodeState`` owns the device buffers of one attention layer (queries, K/V
cache, block metadata, INT4 label cache, index lists, output, workspace) and
calls libtls for every step of the path.  PyTorch is used only to allocate
device memory and to name the stream.
"""

from __future__ import annotations

import math

import numpy as np
import torch

from . import tls


def _bf16_from_bits(a: np.ndarray, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
    return t.to(device).view(torch.bfloat16)


class DecodeState:
    """One layer's KV cache and index, resident in HBM, with its step buffers.

    q_bits: uint16 [B, Hq, Dqk]; k_bits: uint16 [B, Hkv, N, Dqk];
    v_bits: uint16 [B, Hkv, N, Dv] or None (V is the K row slice at v_offset);
    label_ch: int32 [Hkv, R].  bf16 arrays are passed as their bit patterns.
    """

    def __init__(self, *, batch, n_q_heads, n_kv_heads, qk_dim, v_dim, v_offset, block_size, n_label, ctx_len,
                 K_b, k, q_bits, k_bits, v_bits, label_ch, softmax_scale=None, out_dtype=tls.TLS_OUT_F32,
                 device="cuda", build_index=True, kv_device=None, seq_lens=None):
        self.device = torch.device(device)
        scale = 1.0 / math.sqrt(qk_dim) if softmax_scale is None else softmax_scale
        # seq_lens: tokens present per sequence (int [B]); None: every sequence holds ctx_len
        self.seq_lens = (torch.as_tensor(np.asarray(seq_lens, dtype=np.int32)).to(self.device)
                         if seq_lens is not None else None)
        self.shape = tls.make_shape(batch, n_q_heads, n_kv_heads, qk_dim, v_dim, v_offset, block_size, n_label,
                                    ctx_len, scale, self.seq_lens)
        self._baseline_ws = {}
        self.K_b, self.k = int(K_b), int(k)
        self.rows = batch * n_kv_heads
        self.nb = ctx_len // block_size
        self.out_dtype = out_dtype
        dev = self.device
        self.q = _bf16_from_bits(q_bits, dev)
        self.kc = _bf16_from_bits(k_bits, kv_device or dev) if k_bits is not None else None
        self.vc = _bf16_from_bits(v_bits, kv_device or dev) if v_bits is not None else None
        self.label_ch = torch.from_numpy(np.ascontiguousarray(label_ch, dtype=np.int32)).to(dev)
        self.meta = torch.empty((batch, n_kv_heads, self.nb, 2 * qk_dim), dtype=torch.bfloat16, device=dev)
        self.codes = torch.empty((batch, n_kv_heads, ctx_len, n_label // 2), dtype=torch.uint8, device=dev)
        self.scales = torch.empty((batch, n_kv_heads, ctx_len), dtype=torch.float32, device=dev)
        self.block_idx = torch.empty((batch, n_kv_heads, self.K_b), dtype=torch.int32, device=dev)
        self.token_idx = torch.empty((batch, n_kv_heads, self.k), dtype=torch.int32, device=dev)
        self.block_score = torch.empty((batch, n_kv_heads, self.nb), dtype=torch.float32, device=dev)
        self.token_score = torch.empty((batch, n_kv_heads, self.K_b * block_size), dtype=torch.float32, device=dev)
        odt = torch.float32 if out_dtype == tls.TLS_OUT_F32 else torch.bfloat16
        self.out = torch.empty((batch, n_q_heads, v_dim), dtype=odt, device=dev)
        self.lse = torch.empty((batch, n_q_heads), dtype=torch.float32, device=dev)
        self.ws_bytes = tls.tls_workspace_bytes(self.shape, self.K_b, self.k)
        if self.ws_bytes == 0:
            raise tls.TlsError(tls.TLS_ERR_INVALID_ARG, "tls_workspace_bytes", "invalid shape / K_b / k")
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev)
        if self.kc is not None:
            v = self.vc if self.vc is not None else self.kc
            self.kv = tls.make_kv_view(self.kc, v, qk_dim, v_dim if self.vc is not None else qk_dim)
        if build_index and self.kc is not None:
            self.build_index()

    # index build (prefill) -------------------------------------------------
    def build_index(self, t0: int = 0, t1: int | None = None, stream=None):
        s = self.shape
        t1 = s.ctx_len if t1 is None else t1
        tls.tls_build_block_meta(s, self.kc, s.qk_dim, t0, t1, self.meta, stream)
        tls.tls_quant_label_cache(s, self.kc, s.qk_dim, self.label_ch, t0, t1, self.codes, self.scales, stream)

    # the per-step path -----------------------------------------------------
    def select_blocks(self, q=None, keep_scores=False, stream=None):
        tls.tls_select_blocks(self.shape, self.q if q is None else q, self.meta, self.K_b, self.block_idx,
                              self.block_score if keep_scores else None, self.ws, self.ws_bytes, stream)

    def select_tokens(self, q=None, block_idx=None, keep_scores=False, stream=None):
        tls.tls_select_tokens(self.shape, self.q if q is None else q, self.label_ch, self.codes, self.scales,
                              self.block_idx if block_idx is None else block_idx, self.K_b, self.k, self.token_idx,
                              self.token_score if keep_scores else None, self.ws, self.ws_bytes, stream)

    def select(self, q=None, stream=None):
        """Levels 1 and 2 (tls_select)."""
        tls.tls_select(self.shape, self.q if q is None else q, self.meta, self.label_ch, self.codes, self.scales,
                       self.K_b, self.k, self.block_idx, self.token_idx, self.ws, self.ws_bytes, stream)

    def attend(self, q=None, token_idx=None, kv=None, stream=None):
        tls.tls_sparse_decode_attn(self.shape, self.q if q is None else q, self.kv if kv is None else kv,
                                   self.token_idx if token_idx is None else token_idx, self.k, self.out_dtype,
                                   self.out, self.lse, self.ws, self.ws_bytes, stream)

    def step(self, q=None, stream=None):
        """One synchronous decode step (tls_select + attention)."""
        tls.tls_decode_step(self.shape, self.q if q is None else q, self.meta, self.label_ch, self.codes,
                            self.scales, self.kv, self.K_b, self.k, self.block_idx, self.token_idx, self.out_dtype,
                            self.out, self.lse, self.ws, self.ws_bytes, stream)

    def check_device_error(self, stream=None) -> int:
        return tls.tls_workspace_error(self.ws, True, stream)

    # per-token append ---------------------------------------------------------
    def append(self, k_new, v_new=None, stream=None):
        """Appends one decoded token to every sequence (tls_append_kv): device bf16 k_new [B, Hkv, Dqk],
        v_new [B, Hkv, Dv] (None for the MLA latent); needs seq_lens."""
        if self.seq_lens is None:
            raise ValueError("append needs a state created with seq_lens")
        v = self.vc if self.vc is not None else self.kc
        kv = tls.make_kv_view(self.kc, v, self.shape.qk_dim, self.shape.v_dim if self.vc is not None else self.shape.qk_dim)
        tls.tls_append_kv(self.shape, self.seq_lens, k_new, v_new, kv, self.meta, self.label_ch, self.codes,
                          self.scales, stream)

    # operator baselines (full attention, block selection alone, token selection alone)
    def _ws_for(self, K_b, k):
        key = (K_b, k)
        if key not in self._baseline_ws:
            n = tls.tls_workspace_bytes(self.shape, K_b, k)
            if n == 0:
                raise tls.TlsError(tls.TLS_ERR_INVALID_ARG, "tls_workspace_bytes", f"K_b {K_b}, k {k}")
            self._baseline_ws[key] = (torch.zeros(n, dtype=torch.uint8, device=self.device), n)
        return self._baseline_ws[key]

    def dense(self, q=None, stream=None):
        """Full attention over every token of each sequence (tls_dense_decode_attn) into out / lse."""
        ws, n = self._ws_for(self.nb, self.shape.ctx_len)
        tls.tls_dense_decode_attn(self.shape, self.q if q is None else q, self.kv, self.out_dtype, self.out, self.lse,
                                  ws, n, stream)

    def quest(self, q=None, K_b=None, block_idx=None, stream=None):
        """Block selection alone (tls_quest_decode_step): K_b blocks, every token of them attended."""
        K_b = self.K_b if K_b is None else K_b
        if block_idx is None:
            block_idx = self.block_idx if K_b == self.K_b else torch.empty(
                (self.shape.batch, self.shape.n_kv_heads, K_b), dtype=torch.int32, device=self.device)
        ws, n = self._ws_for(K_b, K_b * self.shape.block_size)
        tls.tls_quest_decode_step(self.shape, self.q if q is None else q, self.meta, self.kv, K_b, block_idx,
                                  self.out_dtype, self.out, self.lse, ws, n, stream)
        return block_idx

    def ds(self, q=None, k=None, token_idx=None, stream=None):
        """Token selection alone over every token (tls_ds_decode_step): k tokens attended."""
        k = self.k if k is None else k
        if token_idx is None:
            token_idx = self.token_idx if k == self.k else torch.empty(
                (self.shape.batch, self.shape.n_kv_heads, k), dtype=torch.int32, device=self.device)
        ws, n = self._ws_for(self.nb, k)
        tls.tls_ds_decode_step(self.shape, self.q if q is None else q, self.label_ch, self.codes, self.scales,
                               self.kv, k, token_idx, self.out_dtype, self.out, self.lse, ws, n, stream)
        return token_idx


class ResidentEngine:
    """The staggered schedule over a DecodeState's HBM-resident K/V and index
    (tls_engine_create_resident): step t selects tokens and attends within
    the blocks chosen at step t-1 while level 1 chooses M_t on a second
    stream.  Its own block lists (two), token list, output and workspace; the
    state's buffers are left alone.  A step never waits on the host and may be
    captured into a CUDA graph."""

    def __init__(self, st: DecodeState):
        self.st = st
        dev = st.device
        s = st.shape
        self.K_b, self.k = st.K_b, st.k
        self.block_idx = torch.empty((2, s.batch, s.n_kv_heads, self.K_b), dtype=torch.int32, device=dev)
        self.token_idx = torch.empty((s.batch, s.n_kv_heads, self.k), dtype=torch.int32, device=dev)
        self.out = torch.empty_like(st.out)
        self.lse = torch.empty_like(st.lse)
        self.out_dtype = st.out_dtype
        self.ws_bytes = tls.tls_workspace_bytes(s, self.K_b, self.k)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.engine = tls.tls_engine_create_resident(s, self.K_b, self.k, st.meta, st.label_ch, st.codes, st.scales,
                                                     st.kv, self.block_idx, self.token_idx, self.ws, self.ws_bytes)

    def step(self, q=None, stream=None, out=None):
        """One staggered step with q (default: the state's q); writes self.out (or `out`, a device
        buffer of the same shape and type) and self.lse."""
        tls.tls_engine_step(self.engine, self.st.q if q is None else q, self.out_dtype,
                            self.out if out is None else out, self.lse, stream)

    def steps_taken(self) -> int:
        return tls.tls_engine_steps(self.engine)

    def step_kernels(self) -> int:
        """Kernel launches of one step (tls_engine_step_kernels)."""
        return tls.tls_engine_step_kernels(self.engine)

    def blocks_of_step(self, t: int) -> torch.Tensor:
        """M_t (valid after step t, until step t + 2 overwrites it)."""
        return self.block_idx[t & 1]

    def check_device_error(self, stream=None) -> int:
        return tls.tls_workspace_error(self.ws, True, stream)

    def close(self):
        if getattr(self, "engine", None):
            tls.tls_engine_destroy(self.engine)
            self.engine = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def state_for_config(cfg, q_bits, k_bits, v_bits, label_ch, **kw) -> DecodeState:
    """DecodeState for a workload description with the fields of synth.WorkloadConfig."""
    return DecodeState(batch=cfg.batch, n_q_heads=cfg.n_q_heads, n_kv_heads=cfg.n_kv_heads, qk_dim=cfg.qk_dim,
                       v_dim=cfg.v_dim, v_offset=cfg.v_offset, block_size=cfg.block_size, n_label=cfg.n_label,
                       ctx_len=cfg.ctx_len, K_b=cfg.K_b, k=cfg.k, q_bits=q_bits, k_bits=k_bits, v_bits=v_bits,
                       label_ch=label_ch, softmax_scale=cfg.softmax_scale, **kw)


class OffloadedLayer:
    """One layer whose K/V live in pinned host memory behind an HBM block cache,
    decoded step by step by the staggered engine (tls_engine_*).

    q_bits are not needed to build it; k_bits / v_bits: uint16 [B, Hkv, N, D]
    bf16 bit patterns (v_bits None for the MLA latent).  The index (block
    meta, INT4 label cache) is built on the device from a temporary copy of K,
    which is released afterwards: only the n_slots-block pool holds K/V in HBM.
    """

    def __init__(self, *, batch, n_q_heads, n_kv_heads, qk_dim, v_dim, v_offset, block_size, n_label, ctx_len,
                 K_b, k, n_slots, k_bits, v_bits, label_ch, softmax_scale=None, out_dtype=tls.TLS_OUT_F32,
                 device="cuda", share_from=None):
        dev = torch.device(device)
        self.device = dev
        scale = 1.0 / math.sqrt(qk_dim) if softmax_scale is None else softmax_scale
        self.shape = tls.make_shape(batch, n_q_heads, n_kv_heads, qk_dim, v_dim, v_offset, block_size, n_label,
                                    ctx_len, scale)
        self.K_b, self.k, self.n_slots = int(K_b), int(k), int(n_slots)
        self.rows = batch * n_kv_heads
        self.nb = ctx_len // block_size
        self.out_dtype = out_dtype
        if share_from is not None:
            # another layer object over the same host K/V and index (its own
            # cache, block lists and engine): the pinned buffers and the index
            # are shared, read-only
            for name in ("host_k", "host_v", "label_ch", "meta", "codes", "scales"):
                setattr(self, name, getattr(share_from, name))
        else:
            # full K/V in pinned host memory
            self.host_k = torch.from_numpy(np.ascontiguousarray(k_bits).view(np.int16)).pin_memory()
            self.host_v = (torch.from_numpy(np.ascontiguousarray(v_bits).view(np.int16)).pin_memory()
                           if v_bits is not None else None)
            # resident index, built from a temporary device copy of K
            self.label_ch = torch.from_numpy(np.ascontiguousarray(label_ch, dtype=np.int32)).to(dev)
            self.meta = torch.empty((batch, n_kv_heads, self.nb, 2 * qk_dim), dtype=torch.bfloat16, device=dev)
            self.codes = torch.empty((batch, n_kv_heads, ctx_len, n_label // 2), dtype=torch.uint8, device=dev)
            self.scales = torch.empty((batch, n_kv_heads, ctx_len), dtype=torch.float32, device=dev)
            kd = self.host_k.to(dev).view(torch.bfloat16)
            tls.tls_build_block_meta(self.shape, kd, qk_dim, 0, ctx_len, self.meta, None)
            tls.tls_quant_label_cache(self.shape, kd, qk_dim, self.label_ch, 0, ctx_len, self.codes, self.scales,
                                      None)
            torch.cuda.synchronize(dev)
            del kd
        with_v = self.host_v is not None
        # the HBM block cache
        self.slot_k = torch.empty((n_slots, block_size, qk_dim), dtype=torch.bfloat16, device=dev)
        self.slot_v = (torch.empty((n_slots, block_size, v_dim), dtype=torch.bfloat16, device=dev)
                       if with_v else None)
        self.slot_table = torch.full((batch, n_kv_heads, self.nb), -1, dtype=torch.int32, device=dev)
        self.cache = tls.tls_block_cache_create(self.shape, self.host_k, self.host_v, qk_dim,
                                                v_dim if with_v else 0, n_slots, self.slot_k,
                                                self.slot_v, self.slot_table)
        self.block_idx = torch.empty((2, batch, n_kv_heads, self.K_b), dtype=torch.int32, device=dev)
        self.token_idx = torch.empty((batch, n_kv_heads, self.k), dtype=torch.int32, device=dev)
        odt = torch.float32 if out_dtype == tls.TLS_OUT_F32 else torch.bfloat16
        self.out = torch.empty((batch, n_q_heads, v_dim), dtype=odt, device=dev)
        self.lse = torch.empty((batch, n_q_heads), dtype=torch.float32, device=dev)
        self.ws_bytes = tls.tls_workspace_bytes(self.shape, self.K_b, self.k)
        self.ws = torch.zeros(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.engine = tls.tls_engine_create(self.shape, self.K_b, self.k, self.meta, self.label_ch, self.codes,
                                            self.scales, self.cache, self.block_idx, self.token_idx, self.ws,
                                            self.ws_bytes)

    def step(self, q, stream=None):
        """One staggered decode step with q (device bf16 [B, Hq, Dqk]); writes self.out / self.lse."""
        tls.tls_engine_step(self.engine, q, self.out_dtype, self.out, self.lse, stream)

    def steps_taken(self) -> int:
        return tls.tls_engine_steps(self.engine)

    def stats(self, step: int):
        return tls.tls_engine_stats(self.engine, step)

    def blocks_of_step(self, t: int) -> torch.Tensor:
        """M_t (valid after step t, until step t + 2 overwrites it)."""
        return self.block_idx[t & 1]

    def check_device_error(self, stream=None) -> int:
        return tls.tls_workspace_error(self.ws, True, stream)

    def close(self):
        if getattr(self, "engine", None):
            tls.tls_engine_destroy(self.engine)
            self.engine = None
        if getattr(self, "cache", None):
            tls.tls_block_cache_destroy(self.cache)
            self.cache = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def offloaded_layer_for_config(cfg, k_bits, v_bits, label_ch, n_slots=None, **kw) -> OffloadedLayer:
    """OffloadedLayer for a workload description with the fields of synth.WorkloadConfig.

    The pool is shared by all rows: cfg.n_slots (default 2 * K_b, which always
    holds M_{t-1} and M_t) slots per (batch row, KV head), unless n_slots
    gives the pool size itself."""
    pool = n_slots if n_slots is not None else (cfg.n_slots or 2 * cfg.K_b) * cfg.batch * cfg.n_kv_heads
    return OffloadedLayer(batch=cfg.batch, n_q_heads=cfg.n_q_heads, n_kv_heads=cfg.n_kv_heads, qk_dim=cfg.qk_dim,
                          v_dim=cfg.v_dim, v_offset=cfg.v_offset, block_size=cfg.block_size, n_label=cfg.n_label,
                          ctx_len=cfg.ctx_len, K_b=cfg.K_b, k=cfg.k, n_slots=pool,
                          k_bits=k_bits, v_bits=v_bits, label_ch=label_ch, softmax_scale=cfg.softmax_scale, **kw)
