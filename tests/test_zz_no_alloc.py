"""The scratch-free attention entry point, through the C ABI.

tls_sparse_decode_attn_noalloc serves callers that cannot allocate device
memory (a plug-in inside a runtime that owns the whole HBM budget, or a decode
loop where cudaMalloc's possible device synchronisation is not allowed).  It
must give the same outputs as tls_sparse_decode_attn with a workspace, on two
calls in a row (the shared array keeps the previous call's contents), and must
refuse shapes whose scratch does not fit its fixed array.  This file is named
so that pytest collects it last.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import synth
from tests.parity import check_output

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def tls():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from two_level_sparse_block_b200 import build
    build.build()
    from two_level_sparse_block_b200 import tls as t
    return t


def _state(cfg):
    from two_level_sparse_block_b200 import runtime
    q = synth.gen_queries(cfg)
    K, V, _ = synth.gen_kv(cfg, q)
    lab = synth.gen_label_channels(cfg)
    st = runtime.state_for_config(cfg, q, K, V, lab)
    st.select_blocks()
    st.select_tokens()
    st.attend()
    torch.cuda.synchronize()
    return st


@pytest.mark.parametrize("name", ["c1", "c2"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(tls, name):
    st = _state(synth.get_config(name))
    ref_out = st.out.clone()
    ref_lse = st.lse.clone()
    for _ in range(2):
        out = torch.full_like(st.out, float("nan"))
        lse = torch.full_like(st.lse, float("nan"))
        tls.tls_sparse_decode_attn_noalloc(st.shape, st.q, st.kv, st.token_idx, st.k, st.out_dtype, out, lse)
        torch.cuda.synchronize()
        check_output(out.cpu().numpy(), ref_out.cpu().numpy(), f"{name} noalloc out")
        assert np.max(np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy())) <= 1e-4 * max(1.0, float(ref_lse.abs().max()))
        assert torch.equal(out, ref_out)
        # the array's error word (read through tls_workspace_error with no workspace) stays clear
        assert tls.tls_workspace_error(None) == 0


def test_noalloc_rejects_scratch_beyond_its_array(tls):
    # 512 rows x 8 heads x 2 splits x 130 floats = 4.26 MB > 4 MiB (256 tokens make two
    # 128-token splits); real buffers are allocated so that even a wrongly accepted call
    # would stay in bounds
    B, Hkv, G, D, N, bs, k = 64, 8, 8, 128, 256, 32, 256
    shape = tls.make_shape(B, Hkv * G, Hkv, D, D, -1, bs, 16, N, D ** -0.5)
    q = torch.zeros((B, Hkv * G, D), dtype=torch.bfloat16, device="cuda")
    kk = torch.zeros((B, Hkv, N, D), dtype=torch.bfloat16, device="cuda")
    vv = torch.zeros_like(kk)
    idx = torch.arange(k, dtype=torch.int32, device="cuda").repeat(B * Hkv, 1).contiguous()
    out = torch.zeros((B, Hkv * G, D), dtype=torch.float32, device="cuda")
    kv = tls.make_kv_view(kk, vv, D, D)
    with pytest.raises(tls.TlsError) as e:
        tls.tls_sparse_decode_attn_noalloc(shape, q, kv, idx, k, tls.TLS_OUT_F32, out, None)
    assert e.value.status == tls.TLS_ERR_CAPACITY
    torch.cuda.synchronize()
