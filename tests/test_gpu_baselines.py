"""The operator baselines (English summary 4, Efficiency: the method against
full attention and against each level alone) on the GPU, against the oracle.

  tls_dense_decode_attn   full attention over every held token
  tls_quest_decode_step   level 1, then every token of the K_b blocks
  tls_ds_decode_step      level 2 over every token, then its k tokens

Small shapes take every attention kernel and every level-2 kernel, with and
without ragged lengths; the full-size workloads are checked on sampled rows.
"""

from __future__ import annotations

import functools

import numpy as np
import pytest
import torch

import oracle
import synth
from tests.parity import check_output, check_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from two_level_sparse_block_b200 import build
    build.build()


def _rt():
    from two_level_sparse_block_b200 import runtime, tls
    return runtime, tls


def cfg_of(name, **kw):
    base = dict(name=name, description="baseline parity shape", batch=3, n_q_heads=8, n_kv_heads=2, qk_dim=128,
                v_dim=128, v_offset=-1, ctx_len=2048, block_size=16, K_b=12, k=100, n_label=16, seed=91,
                n_outlier=3, planted_per_row=16, planted_blocks=4, label_from_outliers=True)
    base.update(kw)
    return synth.WorkloadConfig(**base)


SMALL = [
    (cfg_of("b_gqa4"), None),
    (cfg_of("b_gqa4_ragged"), [2048, 700, 9]),
    (cfg_of("b_mla_g16", batch=2, n_q_heads=16, n_kv_heads=1, qk_dim=576, v_dim=512, v_offset=0, ctx_len=1024,
            block_size=64, K_b=6, k=200, n_label=32, n_outlier=0, label_from_outliers=False, kv_std=0.7071, seed=92),
     [1024, 333]),
    (cfg_of("b_d64_simt", n_q_heads=12, qk_dim=64, v_dim=64, ctx_len=1024, K_b=9, k=144, n_label=8, seed=93), None),
    (cfg_of("b_g32_tc", batch=2, n_q_heads=32, n_kv_heads=1, ctx_len=4096, block_size=64, K_b=10, k=300, seed=94),
     [4096, 1500]),
]


@functools.lru_cache(maxsize=2)
def _data(cfg):
    q = synth.gen_queries(cfg)
    K, V, _ = synth.gen_kv(cfg, q)
    lab = synth.gen_label_channels(cfg)
    return q, K, V, lab


def _state(cfg, lens):
    runtime, tls = _rt()
    q, K, V, lab = _data(cfg)
    st = runtime.state_for_config(cfg, q, K, V, lab,
                                  seq_lens=None if lens is None else np.asarray(lens, dtype=np.int32))
    torch.cuda.synchronize()
    return st


def _rows(cfg, n=None):
    rows = [(b, h) for b in range(cfg.batch) for h in range(cfg.n_kv_heads)]
    if n is None or len(rows) <= n:
        return rows
    rng = np.random.default_rng(cfg.seed)
    return [rows[0], rows[-1]] + [rows[i] for i in rng.choice(np.arange(1, len(rows) - 1), n - 2, replace=False)]


def _row_args(cfg, b, h, n):
    q, K, V, lab = _data(cfg)
    g = cfg.group
    return q[b, h * g:(h + 1) * g], K[b, h, :n], (None if V is None else V[b, h, :n]), lab[h]


def _len(cfg, lens, b):
    return cfg.ctx_len if lens is None else lens[b]


def check_dense(cfg, lens, st, rows):
    out = st.out.float().cpu().numpy()
    lse = st.lse.cpu().numpy()
    g = cfg.group
    for b, h in rows:
        qg, kb, vb, _ = _row_args(cfg, b, h, _len(cfg, lens, b))
        ref, ref_lse = oracle.dense_row(qg, kb, vb, cfg.softmax_scale, v_offset=cfg.v_offset, v_dim=cfg.v_dim)
        where = f"{cfg.name} dense ({b},{h})"
        check_output(out[b, h * g:(h + 1) * g], ref, where)
        assert np.max(np.abs(lse[b, h * g:(h + 1) * g] - ref_lse)) <= 1e-4 * max(1.0, np.max(np.abs(ref_lse))), where


def check_quest(cfg, lens, st, block_idx, rows, K_b):
    out = st.out.float().cpu().numpy()
    bl = block_idx.cpu().numpy()
    g, bs = cfg.group, cfg.block_size
    for b, h in rows:
        n = _len(cfg, lens, b)
        qg, kb, vb, lab = _row_args(cfg, b, h, n)
        where = f"{cfg.name} quest ({b},{h})"
        nbr = -(-n // bs)
        kk = min(K_b, nbr)
        assert np.all(bl[b, h, kk:] == -1), where + ": padding"
        r1 = oracle.quest_row(qg, kb, vb, lab, bs, K_b, cfg.softmax_scale, v_offset=cfg.v_offset, v_dim=cfg.v_dim)
        check_selection(bl[b, h, :kk], r1["agg"], kk, where + " blocks")
        r = oracle.quest_row(qg, kb, vb, lab, bs, K_b, cfg.softmax_scale, block_idx=bl[b, h, :kk],
                             v_offset=cfg.v_offset, v_dim=cfg.v_dim)
        check_output(out[b, h * g:(h + 1) * g], r["out"], where + " out")


def check_ds(cfg, lens, st, token_idx, rows, k):
    out = st.out.float().cpu().numpy()
    tl = token_idx.cpu().numpy()
    g, bs = cfg.group, cfg.block_size
    for b, h in rows:
        n = _len(cfg, lens, b)
        qg, kb, vb, lab = _row_args(cfg, b, h, n)
        where = f"{cfg.name} ds ({b},{h})"
        kk = min(k, n)
        assert np.all(tl[b, h, kk:] == -1), where + ": padding"
        r1 = oracle.ds_row(qg, kb, vb, lab, bs, k, cfg.softmax_scale, v_offset=cfg.v_offset, v_dim=cfg.v_dim)
        check_selection(tl[b, h, :kk], r1["token_score"], kk, where + " tokens")  # candidates are 0 .. n-1
        r = oracle.ds_row(qg, kb, vb, lab, bs, k, cfg.softmax_scale, token_idx=tl[b, h, :kk], v_offset=cfg.v_offset,
                          v_dim=cfg.v_dim)
        check_output(out[b, h * g:(h + 1) * g], r["out"], where + " out")


@pytest.mark.parametrize("case", SMALL, ids=lambda c: c[0].name)
def test_baselines_small_all_rows(case):
    cfg, lens = case
    st = _state(cfg, lens)
    rows = _rows(cfg)
    st.dense()
    torch.cuda.synchronize()
    check_dense(cfg, lens, st, rows)
    bl = st.quest()
    torch.cuda.synchronize()
    check_quest(cfg, lens, st, bl, rows, cfg.K_b)
    tl = st.ds()
    torch.cuda.synchronize()
    check_ds(cfg, lens, st, tl, rows, cfg.k)
    assert st.check_device_error() == 0


@pytest.mark.parametrize("name", ["c2", "c3"])
def test_baselines_full_size_sampled_rows(name):
    # full attention over 32768 / 65536 tokens, level 1 with every token of its
    # blocks, level 2 over every token (32768 / 65536 candidates a row: the
    # cluster kernel with its keys spread over the cluster)
    cfg = synth.get_config(name)
    st = _state(cfg, None)
    rows = _rows(cfg, 3)
    st.dense()
    torch.cuda.synchronize()
    check_dense(cfg, None, st, rows)
    bl = st.quest()
    torch.cuda.synchronize()
    check_quest(cfg, None, st, bl, rows, cfg.K_b)
    tl = st.ds()
    torch.cuda.synchronize()
    check_ds(cfg, None, st, tl, rows, cfg.k)
    assert st.check_device_error() == 0


def test_ds_over_equal_scores_takes_the_lowest_positions():
    # every key the same: all 32768 label scores tie, so the cluster selection
    # cannot bin them and the row's keys are gathered in the workspace for one
    # CTA to select; ties go to the lowest positions
    runtime, tls = _rt()
    cfg = cfg_of("b_ties_big", batch=1, n_q_heads=4, n_kv_heads=1, ctx_len=32768, block_size=64, K_b=64, k=1000)
    q = synth.gen_queries(cfg)
    K = np.full((1, 1, cfg.ctx_len, cfg.qk_dim), 0x3F80, dtype=np.uint16)
    V = synth.gen_kv(cfg, q)[1]
    lab = synth.gen_label_channels(cfg)
    st = runtime.state_for_config(cfg, q, K, V, lab)
    assert tls.tls_token_kernel(st.shape, cfg.n_blocks, cfg.k)[0] == "token_select_cluster_kernel"
    tl = st.ds()
    torch.cuda.synchronize()
    assert tl[0, 0].cpu().numpy().tolist() == list(range(cfg.k))
    assert st.check_device_error() == 0
