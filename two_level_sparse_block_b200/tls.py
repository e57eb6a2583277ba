"""ctypes binding of libtls (include/tls.h), argument marshalling only.

Every function carries the C name and forwards to the library; tensors are
passed by their data pointers, streams as the raw cudaStream_t handle.  A
non-zero status raises ``TlsError`` with the library's message.  There is no
fallback: if libtls.so is missing, ``lib()`` raises.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtls.so")

TLS_OK, TLS_ERR_INVALID_ARG, TLS_ERR_UNSUPPORTED, TLS_ERR_CUDA, TLS_ERR_TIMEOUT, TLS_ERR_CAPACITY, TLS_ERR_COPY = range(7)
TLS_OUT_F32, TLS_OUT_BF16 = 0, 1

STATUS_NAMES = {
    0: "TLS_OK", 1: "TLS_ERR_INVALID_ARG", 2: "TLS_ERR_UNSUPPORTED", 3: "TLS_ERR_CUDA",
    4: "TLS_ERR_TIMEOUT", 5: "TLS_ERR_CAPACITY", 6: "TLS_ERR_COPY",
}


class TlsError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("qk_dim", ctypes.c_int32),
        ("v_dim", ctypes.c_int32),
        ("v_offset", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("n_label", ctypes.c_int32),
        ("ctx_len", ctypes.c_int64),
        ("softmax_scale", ctypes.c_float),
        ("seq_lens", ctypes.c_void_p),
    ]


class EngineStepStats(ctypes.Structure):
    _fields_ = [
        ("step", ctypes.c_int64),
        ("n_copied", ctypes.c_int32),
        ("bytes_copied", ctypes.c_int64),
        ("copy_ms", ctypes.c_float),
        ("exposed_ms", ctypes.c_float),
    ]


class KvView(ctypes.Structure):
    _fields_ = [
        ("k", ctypes.c_void_p),
        ("v", ctypes.c_void_p),
        ("k_row_stride", ctypes.c_int64),
        ("v_row_stride", ctypes.c_int64),
        ("slot_of_block", ctypes.c_void_p),
        ("n_slots", ctypes.c_int32),
    ]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_SIG = {
    "tls_last_error": (ctypes.c_char_p, []),
    "tls_version": (_I32, []),
    "tls_copy_from_host": (_I32, [_P, _P, _SZ, _P]),
    "tls_attn_kernel": (ctypes.c_char_p, [_P]),
    "tls_token_kernel": (ctypes.c_char_p, [_P, _I32, _I32, _I32, _P, _P]),
    "tls_workspace_bytes": (_SZ, [_P, _I32, _I32]),
    "tls_workspace_error": (_I32, [_P, _I32, _P, _P]),
    "tls_build_block_meta": (_I32, [_P, _P, _I64, _I64, _I64, _P, _P]),
    "tls_quant_label_cache": (_I32, [_P, _P, _I64, _P, _I64, _I64, _P, _P, _P]),
    "tls_select_blocks": (_I32, [_P, _P, _P, _I32, _P, _P, _P, _SZ, _P]),
    "tls_select_tokens": (_I32, [_P, _P, _P, _P, _P, _P, _I32, _I32, _P, _P, _P, _SZ, _P]),
    "tls_sparse_decode_attn": (_I32, [_P, _P, _P, _P, _I32, _I32, _P, _P, _P, _SZ, _P]),
    "tls_sparse_decode_attn_noalloc": (_I32, [_P, _P, _P, _P, _I32, _I32, _P, _P, _P]),
    "tls_dense_decode_attn": (_I32, [_P, _P, _P, _I32, _P, _P, _P, _SZ, _P]),
    "tls_quest_decode_step": (_I32, [_P, _P, _P, _P, _I32, _P, _I32, _P, _P, _P, _SZ, _P]),
    "tls_ds_decode_step": (_I32, [_P, _P, _P, _P, _P, _P, _I32, _P, _I32, _P, _P, _P, _SZ, _P]),
    "tls_append_kv": (_I32, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "tls_select": (_I32, [_P, _P, _P, _P, _P, _P, _I32, _I32, _P, _P, _P, _SZ, _P]),
    "tls_decode_step": (_I32, [_P, _P, _P, _P, _P, _P, _P, _I32, _I32, _P, _P, _I32, _P, _P, _P, _SZ, _P]),
    "tls_block_cache_create": (_I32, [_P, _P, _P, _I64, _I64, _I32, _P, _P, _P, _P]),
    "tls_block_cache_destroy": (None, [_P]),
    "tls_block_cache_plan": (_I32, [_P, _P, _P, _I32, _P, _P, _P, _P]),
    "tls_prefetch_diff": (_I32, [_P, _P, _P, _I32, _P, _P, _P]),
    "tls_prefetch_diff_device": (_I32, [_P, _P, _P, _I32, _P, _P, _P]),
    "tls_block_cache_table": (_I32, [_P, _P]),
    "tls_engine_create": (_I32, [_P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "tls_engine_create_resident": (_I32, [_P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "tls_engine_step": (_I32, [_P, _P, _I32, _P, _P, _P]),
    "tls_engine_steps": (_I64, [_P]),
    "tls_engine_step_kernels": (_I32, [_P]),
    "tls_engine_stats": (_I32, [_P, _I64, _P]),
    "tls_engine_destroy": (None, [_P]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Loads libtls.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libtls.so not built ({LIB_PATH}); run python -m two_level_sparse_block_b200.build")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIG.items():
            f = getattr(l, name)
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, torch.Tensor):
        return x.data_ptr()
    if isinstance(x, np.ndarray):
        if not x.flags["C_CONTIGUOUS"]:
            raise ValueError("host arrays passed to libtls must be C-contiguous")
        return x.ctypes.data
    if isinstance(x, ctypes.Array):
        return ctypes.addressof(x)
    return int(x)


def _stream(s):
    if s is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, torch.cuda.Stream):
        return s.cuda_stream
    return int(s)


def _check(status: int, where: str):
    if status != TLS_OK:
        raise TlsError(status, where, lib().tls_last_error().decode())


def make_shape(batch, n_q_heads, n_kv_heads, qk_dim, v_dim, v_offset, block_size, n_label, ctx_len,
               softmax_scale, seq_lens=None) -> Shape:
    """seq_lens: optional device int32 tensor [B] of tokens per sequence (the shape keeps its address)."""
    shape = Shape(batch, n_q_heads, n_kv_heads, qk_dim, v_dim, v_offset, block_size, n_label, ctx_len,
                  softmax_scale, _ptr(seq_lens))
    shape._keep = seq_lens  # the shape holds its address
    return shape


def make_kv_view(k, v, k_row_stride, v_row_stride, slot_of_block=None, n_slots=0) -> KvView:
    """The view holds device addresses; it also keeps the tensors it was made
    from alive, so a temporary (e.g. a slot table made inline) is not freed
    while the view may still be passed to a call."""
    view = KvView(_ptr(k), _ptr(v), int(k_row_stride), int(v_row_stride), _ptr(slot_of_block), int(n_slots))
    view._keep = (k, v, slot_of_block)
    return view


def tls_last_error() -> str:
    return lib().tls_last_error().decode()


def tls_version() -> int:
    return lib().tls_version()


def tls_copy_from_host(dst, src, nbytes=None, stream=None):
    """dst (device) <- src (pinned host), nbytes (default: src's size) by one kernel on `stream`."""
    if nbytes is None:
        nbytes = src.numel() * src.element_size() if isinstance(src, torch.Tensor) else src.nbytes
    _check(lib().tls_copy_from_host(_ptr(dst), _ptr(src), nbytes, _stream(stream)), "tls_copy_from_host")


def tls_token_kernel(shape: Shape, K_b: int, k: int, staggered: bool = False):
    """(name, CTAs per row, threads per CTA) of the level-2 kernel for this shape, K_b and k;
    staggered: as a resident engine's step launches it."""
    cl, nt = ctypes.c_int32(), ctypes.c_int32()
    r = lib().tls_token_kernel(ctypes.byref(shape), K_b, k, 1 if staggered else 0, ctypes.byref(cl), ctypes.byref(nt))
    if r is None:
        _check(TLS_ERR_INVALID_ARG, "tls_token_kernel")
    return r.decode(), cl.value, nt.value


def tls_attn_kernel(shape: Shape) -> str:
    """Name of the attention kernel the dispatch launches for this shape."""
    r = lib().tls_attn_kernel(ctypes.byref(shape))
    if r is None:
        _check(TLS_ERR_INVALID_ARG, "tls_attn_kernel")
    return r.decode()


def tls_workspace_bytes(shape: Shape, K_b: int, k: int) -> int:
    return lib().tls_workspace_bytes(ctypes.byref(shape), K_b, k)


def tls_workspace_error(ws, clear=True, stream=None) -> int:
    """Error word of a workspace, or (ws=None) of the scratch-free attention's array."""
    code = ctypes.c_int32(0)
    _check(lib().tls_workspace_error(_ptr(ws), int(bool(clear)), ctypes.byref(code), _stream(stream)),
           "tls_workspace_error")
    return code.value


def tls_build_block_meta(shape, k, k_row_stride, t0, t1, meta, stream=None):
    _check(lib().tls_build_block_meta(ctypes.byref(shape), _ptr(k), k_row_stride, t0, t1, _ptr(meta),
                                      _stream(stream)), "tls_build_block_meta")


def tls_quant_label_cache(shape, k, k_row_stride, label_ch, t0, t1, codes, scales, stream=None):
    _check(lib().tls_quant_label_cache(ctypes.byref(shape), _ptr(k), k_row_stride, _ptr(label_ch), t0, t1,
                                       _ptr(codes), _ptr(scales), _stream(stream)), "tls_quant_label_cache")


def tls_select_blocks(shape, q, meta, K_b, block_idx, block_score, ws, ws_bytes, stream=None):
    _check(lib().tls_select_blocks(ctypes.byref(shape), _ptr(q), _ptr(meta), K_b, _ptr(block_idx),
                                   _ptr(block_score), _ptr(ws), ws_bytes, _stream(stream)), "tls_select_blocks")


def tls_select_tokens(shape, q, label_ch, codes, scales, block_idx, K_b, k, token_idx, token_score, ws, ws_bytes,
                      stream=None):
    _check(lib().tls_select_tokens(ctypes.byref(shape), _ptr(q), _ptr(label_ch), _ptr(codes), _ptr(scales),
                                   _ptr(block_idx), K_b, k, _ptr(token_idx), _ptr(token_score), _ptr(ws), ws_bytes,
                                   _stream(stream)), "tls_select_tokens")


def tls_sparse_decode_attn(shape, q, kv: KvView, token_idx, k, out_dtype, out, lse, ws, ws_bytes, stream=None):
    _check(lib().tls_sparse_decode_attn(ctypes.byref(shape), _ptr(q), ctypes.byref(kv), _ptr(token_idx), k,
                                        out_dtype, _ptr(out), _ptr(lse), _ptr(ws), ws_bytes, _stream(stream)),
           "tls_sparse_decode_attn")


def tls_sparse_decode_attn_noalloc(shape, q, kv: KvView, token_idx, k, out_dtype, out, lse, stream=None):
    _check(lib().tls_sparse_decode_attn_noalloc(ctypes.byref(shape), _ptr(q), ctypes.byref(kv), _ptr(token_idx), k,
                                                out_dtype, _ptr(out), _ptr(lse), _stream(stream)),
           "tls_sparse_decode_attn_noalloc")


def tls_dense_decode_attn(shape, q, kv: KvView, out_dtype, out, lse, ws, ws_bytes, stream=None):
    _check(lib().tls_dense_decode_attn(ctypes.byref(shape), _ptr(q), ctypes.byref(kv), out_dtype, _ptr(out), _ptr(lse),
                                       _ptr(ws), ws_bytes, _stream(stream)), "tls_dense_decode_attn")


def tls_quest_decode_step(shape, q, meta, kv: KvView, K_b, block_idx, out_dtype, out, lse, ws, ws_bytes,
                          stream=None):
    _check(lib().tls_quest_decode_step(ctypes.byref(shape), _ptr(q), _ptr(meta), ctypes.byref(kv), K_b,
                                       _ptr(block_idx), out_dtype, _ptr(out), _ptr(lse), _ptr(ws), ws_bytes,
                                       _stream(stream)), "tls_quest_decode_step")


def tls_ds_decode_step(shape, q, label_ch, codes, scales, kv: KvView, k, token_idx, out_dtype, out, lse, ws, ws_bytes,
                       stream=None):
    _check(lib().tls_ds_decode_step(ctypes.byref(shape), _ptr(q), _ptr(label_ch), _ptr(codes), _ptr(scales),
                                    ctypes.byref(kv), k, _ptr(token_idx), out_dtype, _ptr(out), _ptr(lse), _ptr(ws),
                                    ws_bytes, _stream(stream)), "tls_ds_decode_step")


def tls_append_kv(shape, seq_lens, k_new, v_new, kv: KvView, meta, label_ch, codes, scales, stream=None):
    _check(lib().tls_append_kv(ctypes.byref(shape), _ptr(seq_lens), _ptr(k_new), _ptr(v_new), ctypes.byref(kv),
                               _ptr(meta), _ptr(label_ch), _ptr(codes), _ptr(scales), _stream(stream)),
           "tls_append_kv")


def tls_select(shape, q, meta, label_ch, codes, scales, K_b, k, block_idx, token_idx, ws, ws_bytes, stream=None):
    _check(lib().tls_select(ctypes.byref(shape), _ptr(q), _ptr(meta), _ptr(label_ch), _ptr(codes), _ptr(scales),
                            K_b, k, _ptr(block_idx), _ptr(token_idx), _ptr(ws), ws_bytes, _stream(stream)),
           "tls_select")


def tls_decode_step(shape, q, meta, label_ch, codes, scales, kv: KvView, K_b, k, block_idx, token_idx, out_dtype,
                    out, lse, ws, ws_bytes, stream=None):
    _check(lib().tls_decode_step(ctypes.byref(shape), _ptr(q), _ptr(meta), _ptr(label_ch), _ptr(codes),
                                 _ptr(scales), ctypes.byref(kv), K_b, k, _ptr(block_idx), _ptr(token_idx),
                                 out_dtype, _ptr(out), _ptr(lse), _ptr(ws), ws_bytes, _stream(stream)),
           "tls_decode_step")


def tls_block_cache_create(shape, host_k, host_v, host_k_row_stride, host_v_row_stride, n_slots, slot_k, slot_v,
                           slot_table_dev) -> int:
    h = ctypes.c_void_p(0)
    _check(lib().tls_block_cache_create(ctypes.byref(shape), _ptr(host_k), _ptr(host_v), host_k_row_stride,
                                        host_v_row_stride, n_slots, _ptr(slot_k), _ptr(slot_v),
                                        _ptr(slot_table_dev), ctypes.byref(h)), "tls_block_cache_create")
    return h.value


def tls_block_cache_destroy(handle: int):
    lib().tls_block_cache_destroy(handle)


def tls_block_cache_plan(handle, new_block_idx, in_use_block_idx, K_b, copy_row=None, copy_block=None,
                         copy_slot=None) -> int:
    n = ctypes.c_int32(0)
    _check(lib().tls_block_cache_plan(handle, _ptr(new_block_idx), _ptr(in_use_block_idx), K_b, _ptr(copy_row),
                                      _ptr(copy_block), _ptr(copy_slot), ctypes.byref(n)), "tls_block_cache_plan")
    return n.value


def tls_prefetch_diff(handle, new_block_idx_host, in_use_block_idx_host, K_b, copy_stream=None,
                      done_event=None) -> int:
    """done_event: optional torch.cuda.Event (or raw cudaEvent_t) recorded on copy_stream after the copies."""
    n = ctypes.c_int32(0)
    ev = getattr(done_event, "cuda_event", done_event)
    _check(lib().tls_prefetch_diff(handle, _ptr(new_block_idx_host), _ptr(in_use_block_idx_host), K_b,
                                   _stream(copy_stream), ev, ctypes.byref(n)), "tls_prefetch_diff")
    return n.value


def tls_prefetch_diff_device(handle, new_block_idx_dev, in_use_block_idx_dev, K_b, copy_stream=None,
                             done_event=None, n_copied_dev=None):
    """Device block lists (torch int32 tensors); n_copied_dev: optional device int32 tensor written with
    the number of copied blocks (-1: the plan failed)."""
    ev = getattr(done_event, "cuda_event", done_event)
    _check(lib().tls_prefetch_diff_device(handle, _ptr(new_block_idx_dev), _ptr(in_use_block_idx_dev), K_b,
                                          _stream(copy_stream), ev, _ptr(n_copied_dev)), "tls_prefetch_diff_device")


def tls_block_cache_table(handle, table):
    _check(lib().tls_block_cache_table(handle, _ptr(table)), "tls_block_cache_table")


def tls_engine_create(shape, K_b, k, meta, label_ch, codes, scales, cache, block_idx, token_idx, ws,
                      ws_bytes) -> int:
    h = ctypes.c_void_p()
    _check(lib().tls_engine_create(ctypes.byref(shape), K_b, k, _ptr(meta), _ptr(label_ch), _ptr(codes),
                                   _ptr(scales), cache, _ptr(block_idx), _ptr(token_idx), _ptr(ws), ws_bytes,
                                   ctypes.byref(h)), "tls_engine_create")
    return h.value


def tls_engine_create_resident(shape, K_b, k, meta, label_ch, codes, scales, kv: KvView, block_idx, token_idx, ws,
                               ws_bytes) -> int:
    h = ctypes.c_void_p()
    _check(lib().tls_engine_create_resident(ctypes.byref(shape), K_b, k, _ptr(meta), _ptr(label_ch), _ptr(codes),
                                            _ptr(scales), ctypes.byref(kv), _ptr(block_idx), _ptr(token_idx),
                                            _ptr(ws), ws_bytes, ctypes.byref(h)), "tls_engine_create_resident")
    return h.value


def tls_engine_step(engine, q, out_dtype, out, lse=None, stream=None):
    _check(lib().tls_engine_step(engine, _ptr(q), out_dtype, _ptr(out), _ptr(lse), _stream(stream)),
           "tls_engine_step")


def tls_engine_steps(engine) -> int:
    return lib().tls_engine_steps(engine)


def tls_engine_step_kernels(engine) -> int:
    return lib().tls_engine_step_kernels(engine)


def tls_engine_stats(engine, step: int) -> EngineStepStats:
    st = EngineStepStats()
    _check(lib().tls_engine_stats(engine, step, ctypes.byref(st)), "tls_engine_stats")
    return st


def tls_engine_destroy(engine):
    lib().tls_engine_destroy(engine)
