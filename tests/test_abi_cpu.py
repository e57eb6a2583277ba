"""The C ABI without a GPU: the library loads, exports every declared entry
point, validates arguments, and its host-only block-cache planner follows the
incremental-transfer rule T_t = M_t \\ C_t (AsyncTLS English summary 2.B)."""

from __future__ import annotations

import ctypes
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def tls():
    from two_level_sparse_block_b200 import build
    build.build()
    from two_level_sparse_block_b200 import tls as t
    return t


def declared_functions():
    text = open(os.path.join(ROOT, "include", "tls.h")).read()
    return re.findall(r"^TLS_API\s+[\w\s\*]+?\b(tls_\w+)\s*\(", text, flags=re.M)


def test_library_exports_every_declared_symbol(tls):
    names = declared_functions()
    assert len(names) >= 15
    lib = ctypes.CDLL(tls.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/tls.h but not exported"
    # and the binding wraps each of them under the same name
    for n in names:
        assert hasattr(tls, n), f"binding lacks {n}"


def test_version_and_error_string(tls):
    assert tls.tls_version() >= 100
    assert isinstance(tls.tls_last_error(), str)


def test_copy_from_host_checks_its_arguments_before_anything(tls):
    # NULL pointers and sizes or addresses that are not multiples of 16 bytes
    # are rejected on the host (no CUDA call is reached)
    lib = tls.lib()
    buf = np.zeros(64, dtype=np.uint8)
    p = buf.ctypes.data + (-buf.ctypes.data) % 16
    assert lib.tls_copy_from_host(None, p, 16, None) == tls.TLS_ERR_INVALID_ARG
    assert lib.tls_copy_from_host(p, None, 16, None) == tls.TLS_ERR_INVALID_ARG
    assert lib.tls_copy_from_host(p, p, 24, None) == tls.TLS_ERR_INVALID_ARG
    assert lib.tls_copy_from_host(p + 8, p, 16, None) == tls.TLS_ERR_INVALID_ARG
    assert "16 bytes" in tls.tls_last_error()
    assert lib.tls_copy_from_host(p, p, 0, None) == tls.TLS_OK
    # memory that is not pinned (here: no device at all, or plain malloc'd
    # memory on a GPU machine) is refused before anything is launched
    assert lib.tls_copy_from_host(p, p, 16, None) == tls.TLS_ERR_INVALID_ARG
    assert "pinned" in tls.tls_last_error()


def c2_shape(tls, **kw):
    f = dict(batch=8, n_q_heads=32, n_kv_heads=8, qk_dim=128, v_dim=128, v_offset=-1, block_size=64, n_label=16,
             ctx_len=32768, softmax_scale=128 ** -0.5)
    f.update(kw)
    return tls.make_shape(**f)


def test_attention_dispatch_names_the_kernel_per_shape(tls):
    # 128-wide heads: one cluster of CTAs per (row, head group of <= 16 heads) while the grid
    # fits two CTAs per SM; more rows than that: the persistent form
    assert tls.tls_attn_kernel(c2_shape(tls)) == "sparse_attn_mma_cluster_kernel"              # 64 rows x 4
    assert tls.tls_attn_kernel(c2_shape(tls, n_q_heads=128)) == "sparse_attn_mma_cluster_kernel"  # G = 16
    assert tls.tls_attn_kernel(c2_shape(tls, batch=16)) == "sparse_attn_mma_cluster_kernel"     # 128 rows x 2
    assert tls.tls_attn_kernel(c2_shape(tls, batch=1)) == "sparse_attn_mma_cluster_kernel"      # 8 rows x 16
    assert tls.tls_attn_kernel(c2_shape(tls, batch=64)) == "sparse_attn_mma_kernel"             # 512 rows
    # G > 16: head groups of 16 as virtual rows (1 row x 4 groups -> clusters of 8)
    assert tls.tls_attn_kernel(c2_shape(tls, batch=1, n_q_heads=64, n_kv_heads=1)) == "sparse_attn_mma_cluster_kernel"
    assert tls.tls_attn_kernel(c2_shape(tls, batch=40, n_q_heads=64, n_kv_heads=1)) == "sparse_attn_mma_kernel"
    mla = c2_shape(tls, batch=4, n_q_heads=128, n_kv_heads=1, qk_dim=576, v_dim=512, v_offset=0, n_label=32)
    assert tls.tls_attn_kernel(mla) == "sparse_attn_mla_kernel"
    assert tls.tls_attn_kernel(c2_shape(tls, batch=4, n_q_heads=32, n_kv_heads=1, qk_dim=576, v_dim=512, v_offset=0,
                                        n_label=32)) == "sparse_attn_mla_kernel"  # G = 32
    assert tls.tls_attn_kernel(c2_shape(tls, batch=4, n_q_heads=8, n_kv_heads=1, qk_dim=576, v_dim=512, v_offset=0,
                                        n_label=32)) == "sparse_attn_kernel"  # G = 8: not a multiple of 16
    assert tls.tls_attn_kernel(c2_shape(tls, qk_dim=64, v_dim=64)) == "sparse_attn_kernel"
    with pytest.raises(tls.TlsError):
        tls.tls_attn_kernel(c2_shape(tls, n_q_heads=30))


def test_level2_dispatch_names_the_kernel_per_workload(tls):
    # narrow groups (G <= 16, 16/32 label channels, <= 8192 candidates): the row kernel, up to 4
    # CTAs per row within two CTAs per SM, or one 1024-thread CTA per row when the resident
    # stagger keeps level 2 to half the SMs; wide groups: 16-CTA clusters for few long rows
    import synth
    want = {"c1": (("token_select_row_kernel", 2, 512), ("token_select_row_kernel", 2, 512)),
            "c2": (("token_select_row_kernel", 4, 512), ("token_select_row_kernel", 1, 1024)),
            "c3": (("token_select_cluster_kernel", 16, 256), ("token_select_cluster_kernel", 16, 256)),
            "c4": (("token_select_cluster_kernel", 16, 256), ("token_select_cluster_kernel", 16, 256)),
            "c5": (("token_select_row_kernel", 2, 512), ("token_select_row_kernel", 1, 1024))}
    for name, (sync, stag) in want.items():
        c = synth.get_config(name)
        shape = tls.make_shape(c.batch, c.n_q_heads, c.n_kv_heads, c.qk_dim, c.v_dim, c.v_offset, c.block_size,
                               c.n_label, c.ctx_len, c.softmax_scale)
        assert tls.tls_token_kernel(shape, c.K_b, c.k) == sync, name
        assert tls.tls_token_kernel(shape, c.K_b, c.k, staggered=True) == stag, name
    # label channels the tensor-core scorer does not take, or too many candidates for a row
    assert tls.tls_token_kernel(c2_shape(tls, n_label=8), 64, 2048)[0] == "token_select_cluster_kernel"
    assert tls.tls_token_kernel(c2_shape(tls), 256, 2048)[0] == "token_select_cluster_kernel"  # G*R*cand = 2^20
    assert tls.tls_token_kernel(c2_shape(tls, n_label=32), 256, 2048)[0] == "token_select_kernel"  # 2^21
    with pytest.raises(tls.TlsError):
        tls.tls_token_kernel(c2_shape(tls), 64, 4097)  # k > K_b * bs


def test_workspace_validation(tls):
    s = c2_shape(tls)
    a = tls.tls_workspace_bytes(s, 64, 2048)
    assert a > 0 and a % 256 == 0
    assert tls.tls_workspace_bytes(s, 64, 4096) > 0
    assert tls.tls_workspace_bytes(s, 64, 4097) == 0   # k > K_b * bs
    assert tls.tls_workspace_bytes(s, 513, 64) == 0    # K_b > NB
    assert tls.tls_workspace_bytes(s, 0, 1) == 0
    for bad in (dict(qk_dim=100), dict(n_q_heads=30), dict(block_size=12), dict(n_label=15),
                dict(ctx_len=32760), dict(v_offset=4), dict(softmax_scale=0.0), dict(v_dim=520)):
        assert tls.tls_workspace_bytes(c2_shape(tls, **bad), 64, 2048) == 0, bad
    mla = c2_shape(tls, batch=4, n_q_heads=128, n_kv_heads=1, qk_dim=576, v_dim=512, v_offset=0,
                   ctx_len=65536, n_label=32)
    assert tls.tls_workspace_bytes(mla, 128, 4096) > 0


def test_entry_points_reject_null_arguments_without_a_gpu(tls):
    s = c2_shape(tls)
    with pytest.raises(tls.TlsError) as e:
        tls.tls_select_blocks(s, None, None, 64, None, None, None, 0, stream=0)
    assert e.value.status == tls.TLS_ERR_INVALID_ARG
    with pytest.raises(tls.TlsError) as e:
        tls.tls_build_block_meta(s, None, 128, 0, 64, None, stream=0)
    assert e.value.status == tls.TLS_ERR_INVALID_ARG
    # the engines: a NULL cache (offloaded form) or a NULL / non-dense view (resident form)
    with pytest.raises(tls.TlsError) as e:
        tls.tls_engine_create(s, 64, 2048, None, None, None, None, None, None, None, None, 0)
    assert e.value.status == tls.TLS_ERR_INVALID_ARG
    lib = tls.lib()
    h = ctypes.c_void_p()
    assert lib.tls_engine_create_resident(ctypes.byref(s), 64, 2048, None, None, None, None, None, None, None, None, 0,
                                          ctypes.byref(h)) == tls.TLS_ERR_INVALID_ARG
    assert b"NULL" in lib.tls_last_error()
    assert tls.tls_engine_steps(None) == -1


def _trajectory(nb, K_b, steps, seed):
    """Block sets with temporal locality: each step swaps a few blocks."""
    rng = np.random.default_rng(seed)
    cur = np.sort(rng.choice(nb, K_b, replace=False))
    out = [cur]
    for _ in range(steps - 1):
        n_swap = int(rng.integers(0, max(2, K_b // 4)))
        keep = rng.choice(cur, K_b - n_swap, replace=False)
        rest = np.setdiff1d(np.arange(nb), keep)
        cur = np.sort(np.concatenate([keep, rng.choice(rest, n_swap, replace=False)]))
        out.append(cur)
    return out


@pytest.mark.parametrize("rows,n_slots_factor", [(1, 2), (3, 2), (2, 3)])
def test_block_cache_plan_follows_incremental_transfer(tls, rows, n_slots_factor):
    nb, K_b, bs = 64, 8, 16
    s = c2_shape(tls, batch=rows, n_q_heads=4, n_kv_heads=1, ctx_len=nb * bs, block_size=bs)
    n_slots = n_slots_factor * K_b * rows
    h = tls.tls_block_cache_create(s, None, None, 128, 128, n_slots, None, None, None)
    try:
        trajs = [_trajectory(nb, K_b, 40, seed=r) for r in range(rows)]
        resident = [set() for _ in range(rows)]
        prev = None
        for t in range(40):
            new = np.stack([trajs[r][t] for r in range(rows)]).astype(np.int32)
            cap = rows * K_b
            cr, cb, cs = (np.zeros(cap, np.int32) for _ in range(3))
            before = tls_table(tls, h, rows, nb)
            n = tls.tls_block_cache_plan(h, new, prev, K_b, cr, cb, cs)
            after = tls_table(tls, h, rows, nb)
            copied = {(int(cr[i]), int(cb[i])) for i in range(n)}
            for r in range(rows):
                want = oracle.plan_transfer(new[r], sorted(resident[r]))
                assert sorted(b for rr, b in copied if rr == r) == want.tolist()
                resident[r] = {b for b in range(nb) if after[r, b] >= 0}
                assert set(new[r].tolist()) <= resident[r]
            # a victim slot never held a block the running step still reads (M_{t-1}) or keeps (M_t)
            for i in range(n):
                slot = int(cs[i])
                for r in range(rows):
                    for blk in np.where(before[r] == slot)[0]:
                        assert blk not in new[r]
                        if prev is not None:
                            assert blk not in prev[r]
            # the slot table is a partial injection
            used = after[after >= 0]
            assert used.size == np.unique(used).size and used.max() < n_slots
            prev = new
    finally:
        tls.tls_block_cache_destroy(h)


def tls_table(tls, h, rows, nb):
    t = np.zeros((rows, nb), dtype=np.int32)
    tls.tls_block_cache_table(h, t)
    return t


def test_block_cache_plan_capacity_error_commits_nothing(tls):
    nb, K_b, bs = 32, 8, 16
    s = c2_shape(tls, batch=1, n_q_heads=4, n_kv_heads=1, ctx_len=nb * bs, block_size=bs)
    h = tls.tls_block_cache_create(s, None, None, 128, 128, 12, None, None, None)
    try:
        a = np.arange(8, dtype=np.int32)[None]
        assert tls.tls_block_cache_plan(h, a, None, K_b) == 8
        b = np.arange(8, 16, dtype=np.int32)[None]
        before = tls_table(tls, h, 1, nb)
        with pytest.raises(tls.TlsError) as e:
            tls.tls_block_cache_plan(h, b, a, K_b)  # needs 8 free slots, only 4 are not in use
        assert e.value.status == tls.TLS_ERR_CAPACITY
        assert np.array_equal(before, tls_table(tls, h, 1, nb))
        with pytest.raises(tls.TlsError) as e:
            tls.tls_block_cache_plan(h, np.array([[0, 0, 1, 2, 3, 4, 5, 6]], np.int32), None, K_b)
        assert e.value.status == tls.TLS_ERR_INVALID_ARG
    finally:
        tls.tls_block_cache_destroy(h)
