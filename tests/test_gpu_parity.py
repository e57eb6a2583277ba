"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Index build: bit-exact.  Selections: bit-exact up to float32 ties at the k-th
boundary (tests/parity.py).  Outputs: <= 2e-3 max row-relative error.
Workloads are the five configured shapes (full size; the oracle checks a
sample of rows) and small ragged shapes that span several tiles.
"""

from __future__ import annotations

import functools

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import f32_from_bf16_bits, get_config
from tests.parity import check_output, check_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="session", autouse=True)
def _built():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from two_level_sparse_block_b200 import build
    build.build()


def _rt():
    from two_level_sparse_block_b200 import runtime, tls
    return runtime, tls


@functools.lru_cache(maxsize=2)
def gen_case(cfg):
    q = synth.gen_queries(cfg)
    K, V, planted = synth.gen_kv(cfg, q)
    lab = synth.gen_label_channels(cfg)
    return q, K, V, lab


def small(name, **kw):
    base = dict(name=name, description="small parity shape", batch=2, n_q_heads=8, n_kv_heads=2, qk_dim=128,
                v_dim=128, v_offset=-1, ctx_len=2048, block_size=16, K_b=12, k=100, n_label=16, seed=11,
                n_outlier=3, planted_per_row=16, planted_blocks=4, label_from_outliers=True)
    base.update(kw)
    return synth.WorkloadConfig(**base)


SMALL = [
    small("s_gqa4"),
    small("s_g3_ragged", n_q_heads=6, n_kv_heads=2, ctx_len=200 * 16, K_b=37, k=333, seed=12),
    small("s_g1", n_q_heads=3, n_kv_heads=3, K_b=5, k=80, seed=13),
    small("s_g6_d64", n_q_heads=12, n_kv_heads=2, qk_dim=64, v_dim=64, K_b=9, k=144, n_label=8, seed=14),
    small("s_g16_bs32", n_q_heads=16, n_kv_heads=1, block_size=32, ctx_len=4096, K_b=20, k=640, seed=15),
    small("s_mla", batch=2, n_q_heads=16, n_kv_heads=1, qk_dim=576, v_dim=512, v_offset=0, ctx_len=1024,
          block_size=64, K_b=6, k=200, n_label=32, n_outlier=0, label_from_outliers=False, kv_std=0.7071, seed=16),
    small("s_mla_g32", batch=2, n_q_heads=32, n_kv_heads=1, qk_dim=576, v_dim=512, v_offset=0, ctx_len=2048,
          block_size=64, K_b=7, k=333, n_label=32, n_outlier=0, label_from_outliers=False, kv_std=0.7071, seed=19),
    small("s_mla_g8_simt", batch=1, n_q_heads=8, n_kv_heads=1, qk_dim=576, v_dim=512, v_offset=0, ctx_len=1024,
          block_size=64, K_b=5, k=150, n_label=32, n_outlier=0, label_from_outliers=False, kv_std=0.7071, seed=20),
    small("s_k_eq_1", K_b=1, k=1, seed=17),
    small("s_all", ctx_len=512, K_b=32, k=512, seed=18),
]
FULL = [get_config(c) for c in ("c1", "c2", "c3", "c4", "c5")]
# rows the oracle checks per full-size workload (the first and last among them)
FULL_ROWS = {"c1": 1, "c2": 8, "c3": 4, "c4": 1, "c5": 6}
# row counts that send the 128-wide attention to its cluster form (16, 8, 4
# and 2 CTAs per row); ragged lists, idle CTAs, and a 64-head group split into
# four virtual rows of 16 heads
CLUSTER = [
    small("s_cl16", batch=2, n_q_heads=16, n_kv_heads=2, ctx_len=1024, K_b=9, k=120, seed=25),
    small("s_hg4_g64", batch=1, n_q_heads=64, n_kv_heads=1, ctx_len=2048, K_b=14, k=200, seed=26),
    small("s_cl8", batch=20, n_q_heads=4, n_kv_heads=1, ctx_len=1024, K_b=7, k=97, seed=21),
    small("s_cl4", batch=16, n_q_heads=16, n_kv_heads=4, ctx_len=2048, K_b=13, k=200, seed=22),
    small("s_cl4_g1", batch=8, n_q_heads=8, n_kv_heads=8, ctx_len=1024, K_b=8, k=128, seed=23),
    small("s_cl2_g16", batch=100, n_q_heads=16, n_kv_heads=1, ctx_len=1024, block_size=32, K_b=9, k=270, seed=24),
]


def make_state(cfg, **kw):
    runtime, tls = _rt()
    q, K, V, lab = gen_case(cfg)
    st = runtime.state_for_config(cfg, q, K, V, lab, **kw)
    torch.cuda.synchronize()
    return st, (q, K, V, lab)


def sample_rows(cfg, n=3):
    rows = [(b, h) for b in range(cfg.batch) for h in range(cfg.n_kv_heads)]
    if len(rows) <= n:
        return rows
    rng = np.random.default_rng(cfg.seed + 99)
    pick = [rows[0], rows[-1]] + [rows[i] for i in rng.choice(np.arange(1, len(rows) - 1), n - 2, replace=False)]
    return pick


def oracle_row(cfg, data, b, h, **kw):
    q, K, V, lab = data
    g = cfg.group
    vb = None if V is None else V[b, h]
    return oracle.decode_row(q[b, h * g:(h + 1) * g], K[b, h], vb, lab[h], cfg.block_size, cfg.K_b, cfg.k,
                             cfg.softmax_scale, v_offset=cfg.v_offset, v_dim=cfg.v_dim, **kw)


def run_stages(st):
    st.select_blocks(keep_scores=True)
    st.select_tokens(keep_scores=True)
    st.attend()
    torch.cuda.synchronize()
    assert st.check_device_error() == 0
    return dict(block_idx=st.block_idx.cpu().numpy(), token_idx=st.token_idx.cpu().numpy(),
                block_score=st.block_score.cpu().numpy(), token_score=st.token_score.cpu().numpy(),
                out=st.out.float().cpu().numpy(), lse=st.lse.cpu().numpy())


def check_row(cfg, data, got, st, b, h):
    q, K, V, lab = data
    g = cfg.group
    kb = K[b, h]
    meta = oracle.block_meta(kb, cfg.block_size)
    label = oracle.quant_label(kb, lab[h])
    where = f"{cfg.name} row ({b},{h})"

    # index: bit-exact
    gm = st.meta[b, h].float().cpu().numpy().astype(np.float64)
    assert np.array_equal(gm[:, :cfg.qk_dim], meta[0]), f"{where}: kmax differs"
    assert np.array_equal(gm[:, cfg.qk_dim:], meta[1]), f"{where}: kmin differs"
    assert np.array_equal(st.codes[b, h].cpu().numpy(), oracle.pack_codes(label[0])), f"{where}: INT4 codes differ"
    assert np.array_equal(st.scales[b, h].cpu().numpy().view(np.uint32), label[1].view(np.uint32)), \
        f"{where}: scales differ"

    # level 1
    r1 = oracle_row(cfg, data, b, h, meta=meta, label=label)
    agg = r1["agg"]
    scale = np.max(np.abs(agg))
    assert np.max(np.abs(got["block_score"][b, h] - agg)) <= 1e-5 * scale, f"{where}: block scores"
    swaps_b = check_selection(got["block_idx"][b, h], agg, cfg.K_b, where + " blocks")

    # Quest bound on the GPU scores (float32, 1e-5 relative slack), on sampled tokens
    qf = f32_from_bf16_bits(q[b, h * g:(h + 1) * g]).astype(np.float64)
    rng = np.random.default_rng(b * 131 + h)
    toks = rng.choice(cfg.ctx_len, size=min(2048, cfg.ctx_len), replace=False)
    dots = (qf @ f32_from_bf16_bits(kb[toks]).astype(np.float64).T).max(axis=0)
    bound = got["block_score"][b, h][toks // cfg.block_size]
    assert np.all(bound >= dots - 1e-5 * scale), f"{where}: Quest bound violated on the GPU"

    # level 2 on the GPU's block set
    gb = got["block_idx"][b, h]
    r2 = oracle_row(cfg, data, b, h, meta=meta, label=label, block_idx=gb)
    ts = r2["token_score"]
    tscale = np.max(np.abs(ts))
    assert np.max(np.abs(got["token_score"][b, h] - ts)) <= 1e-5 * tscale, f"{where}: token scores"
    cand = r2["cand"]
    pos = np.searchsorted(cand, got["token_idx"][b, h])
    assert np.array_equal(cand[pos], got["token_idx"][b, h]), f"{where}: token outside the chosen blocks"
    swaps_t = check_selection(pos, ts, cfg.k, where + " tokens")

    # attention on the GPU's token set
    r3 = oracle_row(cfg, data, b, h, meta=meta, label=label, block_idx=gb, token_idx=got["token_idx"][b, h])
    err = check_output(got["out"][b, h * g:(h + 1) * g], r3["out"], where + " out")
    assert np.max(np.abs(got["lse"][b, h * g:(h + 1) * g] - r3["lse"])) <= 1e-4 * max(1.0, np.max(np.abs(r3["lse"]))), \
        f"{where}: lse"
    return swaps_b, swaps_t, err


@pytest.mark.parametrize("cfg", SMALL, ids=lambda c: c.name)
def test_small_shapes_all_rows(cfg):
    st, data = make_state(cfg)
    got = run_stages(st)
    for b in range(cfg.batch):
        for h in range(cfg.n_kv_heads):
            check_row(cfg, data, got, st, b, h)


@pytest.mark.parametrize("cfg", CLUSTER, ids=lambda c: c.name)
def test_cluster_attention_sampled_rows(cfg):
    runtime, tls = _rt()
    st, data = make_state(cfg)
    assert tls.tls_attn_kernel(st.shape) == "sparse_attn_mma_cluster_kernel"
    got = run_stages(st)
    for b, h in sample_rows(cfg, 6):  # the first and last rows among them
        check_row(cfg, data, got, st, b, h)


@pytest.mark.parametrize("cfg", FULL, ids=lambda c: c.name)
def test_full_size_sampled_rows(cfg):
    st, data = make_state(cfg)
    got = run_stages(st)
    for b, h in sample_rows(cfg, FULL_ROWS[cfg.name[:2]]):
        check_row(cfg, data, got, st, b, h)
    # the fused step gives the same lists and outputs as the three calls
    st.step()
    torch.cuda.synchronize()
    assert np.array_equal(st.block_idx.cpu().numpy(), got["block_idx"])
    assert np.array_equal(st.token_idx.cpu().numpy(), got["token_idx"])
    assert np.array_equal(st.out.float().cpu().numpy(), got["out"])


def test_select_everything_equals_dense_attention():
    cfg = small("s_dense", ctx_len=1024, block_size=32, K_b=32, k=1024, seed=21)
    st, data = make_state(cfg)
    got = run_stages(st)
    q, K, V, lab = data
    g = cfg.group
    for b in range(cfg.batch):
        for h in range(cfg.n_kv_heads):
            assert got["block_idx"][b, h].tolist() == list(range(cfg.n_blocks))
            assert got["token_idx"][b, h].tolist() == list(range(cfg.ctx_len))
            qq = torch.from_numpy(f32_from_bf16_bits(q[b, h * g:(h + 1) * g]).astype(np.float64))
            kk = torch.from_numpy(f32_from_bf16_bits(K[b, h]).astype(np.float64))
            vv = torch.from_numpy(f32_from_bf16_bits(V[b, h]).astype(np.float64))
            ref = torch.nn.functional.scaled_dot_product_attention(
                qq[:, None, :], kk[None].expand(g, -1, -1), vv[None].expand(g, -1, -1),
                scale=cfg.softmax_scale)[:, 0, :].numpy()
            check_output(got["out"][b, h * g:(h + 1) * g], ref, "dense")


def test_equal_scores_pick_lowest_indices():
    runtime, tls = _rt()
    cfg = small("s_ties", batch=1, n_kv_heads=1, n_q_heads=4, ctx_len=1024, block_size=16, K_b=7, k=50)
    q = synth.gen_queries(cfg)
    K = np.full((1, 1, cfg.ctx_len, cfg.qk_dim), 0x3F80, dtype=np.uint16)  # every key = 1.0
    V = synth.gen_kv(cfg, q)[1]
    lab = synth.gen_label_channels(cfg)
    st = runtime.state_for_config(cfg, q, K, V, lab)
    got = run_stages(st)
    assert got["block_idx"][0, 0].tolist() == list(range(7))
    assert got["token_idx"][0, 0].tolist() == list(range(50))


def test_bf16_output_and_repeat_calls():
    runtime, tls = _rt()
    cfg = SMALL[1]
    st32, data = make_state(cfg)
    st16, _ = make_state(cfg, out_dtype=tls.TLS_OUT_BF16)
    a = run_stages(st32)
    for _ in range(3):  # counters in the workspace must reset after every call
        b = run_stages(st16)
    assert np.array_equal(a["token_idx"], b["token_idx"])
    ref = torch.from_numpy(a["out"]).to(torch.bfloat16).float().numpy()
    assert np.array_equal(b["out"], ref)


def test_slot_table_view_matches_dense():
    runtime, tls = _rt()
    cfg = SMALL[0]
    st, data = make_state(cfg)
    run_stages(st)
    dense = st.out.clone()
    # scatter every block into a shuffled slot pool and read through the table
    rows, nb, bs = cfg.rows, cfg.n_blocks, cfg.block_size
    perm = torch.randperm(rows * nb, generator=torch.Generator().manual_seed(5)).to(torch.int32)
    pool_k = torch.empty((rows * nb, bs, cfg.qk_dim), dtype=torch.bfloat16, device="cuda")
    pool_v = torch.empty((rows * nb, bs, cfg.v_dim), dtype=torch.bfloat16, device="cuda")
    pool_k[perm.long().cuda()] = st.kc.reshape(rows * nb, bs, cfg.qk_dim)
    pool_v[perm.long().cuda()] = st.vc.reshape(rows * nb, bs, cfg.v_dim)
    table = perm.reshape(cfg.batch, cfg.n_kv_heads, nb).cuda()
    kv = tls.make_kv_view(pool_k, pool_v, cfg.qk_dim, cfg.v_dim, table, rows * nb)
    st.attend(kv=kv)
    torch.cuda.synchronize()
    assert torch.equal(st.out, dense)


def test_invalid_arguments_launch_nothing():
    runtime, tls = _rt()
    cfg = SMALL[0]
    st, data = make_state(cfg)
    bad = tls.make_shape(cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.qk_dim, cfg.v_dim, -1, cfg.block_size,
                         cfg.n_label, cfg.ctx_len, cfg.softmax_scale)
    with pytest.raises(tls.TlsError) as e:
        tls.tls_select_blocks(bad, st.q, st.meta, cfg.n_blocks + 1, st.block_idx, None, st.ws, st.ws_bytes)
    assert e.value.status == tls.TLS_ERR_INVALID_ARG
    with pytest.raises(tls.TlsError):
        tls.tls_select_tokens(bad, st.q, st.label_ch, st.codes, st.scales, st.block_idx, cfg.K_b,
                              cfg.K_b * cfg.block_size + 1, st.token_idx, None, st.ws, st.ws_bytes)
    with pytest.raises(tls.TlsError):
        tls.tls_sparse_decode_attn(bad, st.q, st.kv, st.token_idx, cfg.k, 7, st.out, None, st.ws, st.ws_bytes)
    with pytest.raises(tls.TlsError):
        tls.tls_select_blocks(bad, st.q, st.meta, cfg.K_b, st.block_idx, None, st.ws, 16)
    torch.cuda.synchronize()
    assert st.check_device_error() == 0


def test_exact_ties_follow_the_lower_index_rule():
    # keys and queries from {-1, -0.5, 0, 0.5, 1}: every score is a short dyadic
    # sum, exact in float32, so the GPU and oracle scores are identical and the
    # many ties must be broken exactly as the rule says (no tie band applies)
    runtime, tls = _rt()
    cfg = small("s_exact_ties", batch=2, n_q_heads=8, n_kv_heads=2, ctx_len=1024, block_size=16, K_b=13, k=97,
                n_label=8, seed=31)
    rng = np.random.default_rng(31)
    vals = np.array([-1.0, -0.5, 0.0, 0.5, 1.0], dtype=np.float32)
    from synth import bf16_bits_from_f32
    K = bf16_bits_from_f32(rng.choice(vals, size=(2, 2, cfg.ctx_len, cfg.qk_dim)))
    q = bf16_bits_from_f32(rng.choice(vals, size=(2, 8, cfg.qk_dim)))
    V = synth.gen_kv(cfg, synth.gen_queries(cfg))[1]
    lab = synth.gen_label_channels(cfg)
    st = runtime.state_for_config(cfg, q, K, V, lab)
    got = run_stages(st)
    g = cfg.group
    for b in range(2):
        for h in range(2):
            r1 = oracle.decode_row(q[b, h * g:(h + 1) * g], K[b, h], V[b, h], lab[h], cfg.block_size, cfg.K_b,
                                   cfg.k, cfg.softmax_scale)
            assert np.array_equal(got["block_score"][b, h], r1["agg"].astype(np.float32))
            assert got["block_idx"][b, h].tolist() == r1["block_idx"].tolist()
            r2 = oracle.decode_row(q[b, h * g:(h + 1) * g], K[b, h], V[b, h], lab[h], cfg.block_size, cfg.K_b,
                                   cfg.k, cfg.softmax_scale, block_idx=got["block_idx"][b, h])
            assert got["token_idx"][b, h].tolist() == r2["token_idx"].tolist()


def test_crowded_threshold_takes_the_lowest_positions():
    # every K row is one of two patterns, so the token scores take exactly two
    # values; the k-th largest sits among ~half of the 1024 candidates, far more
    # than the pairwise ranking takes, and ties must fall to the lowest positions
    runtime, tls = _rt()
    cfg = small("s_two_valued", batch=1, n_q_heads=4, n_kv_heads=2, ctx_len=2048, block_size=64, K_b=16, k=300,
                n_label=16, seed=41)
    rng = np.random.default_rng(41)
    from synth import bf16_bits_from_f32
    pat = rng.standard_normal((2, cfg.qk_dim)).astype(np.float32)
    pick = rng.integers(0, 2, size=(1, 2, cfg.ctx_len))
    K = bf16_bits_from_f32(pat[pick])
    q = synth.gen_queries(cfg)
    V = synth.gen_kv(cfg, q)[1]
    lab = synth.gen_label_channels(cfg)
    st = runtime.state_for_config(cfg, q, K, V, lab)
    got = run_stages(st)
    g = cfg.group
    for h in range(2):
        r2 = oracle.decode_row(q[0, h * g:(h + 1) * g], K[0, h], V[0, h], lab[h], cfg.block_size, cfg.K_b,
                               cfg.k, cfg.softmax_scale, block_idx=got["block_idx"][0, h])
        ts = np.asarray(r2["token_score"], dtype=np.float64)
        vals = np.unique(ts)
        tau = np.sort(ts)[::-1][cfg.k - 1]
        assert vals.size == 2 and np.count_nonzero(ts == tau) > 128, "workload lost its construction"
        assert got["token_idx"][0, h].tolist() == r2["token_idx"].tolist()


def _crowd_depth(scores, k, levels=3):
    """Levels of 256 sub-bins (float32 arithmetic, as the cluster selection
    bins) needed before the bin of the k-th largest score holds <= 128."""
    s = np.asarray(scores, dtype=np.float32)
    lo, inv = np.float32(s.min()), np.float32(256.0) / np.float32(s.max() - s.min())
    cell = np.ones(s.size, dtype=bool)
    need = k
    for lv in range(levels):
        b = np.clip(((s - lo) * inv).astype(np.int64), 0, 255)
        cnt = np.bincount(b[cell], minlength=256)
        above = 0
        for tb in range(255, -1, -1):
            if above + cnt[tb] >= need:
                break
            above += cnt[tb]
        need -= above
        if cnt[tb] <= 128:
            return lv
        cell &= b == tb
        lo, inv = np.float32(lo + np.float32(tb) / inv), np.float32(inv * np.float32(256.0))
    return levels


# a few tokens with K rows 1e4 times the rest stretch the score range so far
# that all other candidates share one value bin: the selections (level 2 in
# one CTA a row, or in clusters of 16 and 8 CTAs; level 1 over several CTAs)
# must split that bin with sub-bins instead of falling back
DENSE = [
    small("s_dense_row_g16", batch=1, n_q_heads=16, n_kv_heads=1, ctx_len=16384, block_size=64, K_b=128, k=4096,
          seed=43),
    small("s_dense_cl16_g32", batch=1, n_q_heads=32, n_kv_heads=1, ctx_len=16384, block_size=64, K_b=128,
          k=4096, seed=45),
    small("s_dense_cl8_r32", batch=2, n_q_heads=64, n_kv_heads=2, ctx_len=8192, block_size=64, K_b=64, k=2000,
          n_label=32, seed=44),
]


@pytest.mark.parametrize("cfg", DENSE, ids=lambda c: c.name)
def test_dense_threshold_splits_with_sub_bins(cfg):
    runtime, tls = _rt()
    from synth import bf16_bits_from_f32
    q, K, V, lab = gen_case(cfg)
    Kf = f32_from_bf16_bits(K)
    rng = np.random.default_rng(cfg.seed)
    for b in range(cfg.batch):
        for h in range(cfg.n_kv_heads):
            Kf[b, h, rng.choice(cfg.ctx_len, 4, replace=False)] *= 1.0e4
    K = bf16_bits_from_f32(Kf)
    data = (q, K, V, lab)
    st = runtime.state_for_config(cfg, q, K, V, lab)
    got = run_stages(st)
    bs = cfg.block_size
    deepest = 0
    for b in range(cfg.batch):
        for h in range(cfg.n_kv_heads):
            where = f"{cfg.name} row ({b},{h})"
            # both selections are the exact top-k of the GPU's own float32
            # scores (ties to the lower position): the decision in one precision
            bsc = got["block_score"][b, h]
            assert got["block_idx"][b, h].tolist() == oracle.topk_ascending(bsc, cfg.K_b).tolist(), where + " blocks"
            gb = got["block_idx"][b, h]
            cand = (gb[:, None] * bs + np.arange(bs)[None, :]).reshape(-1)
            ts = got["token_score"][b, h]
            pos = np.searchsorted(cand, got["token_idx"][b, h])
            assert np.array_equal(cand[pos], got["token_idx"][b, h]), where + ": token outside the chosen blocks"
            assert pos.tolist() == oracle.topk_ascending(ts, cfg.k).tolist(), where + " tokens"
            deepest = max(deepest, _crowd_depth(ts, cfg.k))
            # and the scores, tokens and output are the oracle's
            check_row(cfg, data, got, st, b, h)
    assert deepest >= 1, "workload lost its construction: no sub-bins needed"
    assert st.check_device_error() == 0


@pytest.mark.parametrize("cfg", SMALL + [get_config("c1")], ids=lambda c: c.name)
def test_fused_select_equals_the_two_level_calls(cfg):
    st, data = make_state(cfg)
    got = run_stages(st)
    st.block_idx.fill_(-1)
    st.token_idx.fill_(-1)
    st.select()
    torch.cuda.synchronize()
    assert st.check_device_error() == 0
    assert np.array_equal(st.block_idx.cpu().numpy(), got["block_idx"])
    assert np.array_equal(st.token_idx.cpu().numpy(), got["token_idx"])


@pytest.mark.parametrize("cfg", SMALL + [get_config("c1"), get_config("c2")], ids=lambda c: c.name)
def test_decode_step_equals_select_then_attend(cfg):
    # one call for the whole step: the results of the separate calls, bit for bit
    st, data = make_state(cfg)
    got = run_stages(st)
    for t in (st.block_idx, st.token_idx):
        t.fill_(-1)
    st.out.fill_(float("nan"))
    st.lse.fill_(float("nan"))
    st.step()
    torch.cuda.synchronize()
    assert st.check_device_error() == 0
    assert np.array_equal(st.block_idx.cpu().numpy(), got["block_idx"])
    assert np.array_equal(st.token_idx.cpu().numpy(), got["token_idx"])
    assert np.array_equal(st.out.float().cpu().numpy(), got["out"])
    assert np.array_equal(st.lse.cpu().numpy(), got["lse"])


# more virtual rows than two CTAs per SM hold in clusters: the persistent
# attention (contiguous ranges of 16-token chunks, ticket merge through the
# workspace), with rows split across CTAs and CTAs spanning rows
PERSISTENT = [
    small("s_persist_g4", batch=80, n_q_heads=8, n_kv_heads=2, ctx_len=1024, K_b=9, k=133, seed=51),
    small("s_persist_g64", batch=40, n_q_heads=64, n_kv_heads=1, ctx_len=1024, K_b=10, k=150, seed=52),
]


@pytest.mark.parametrize("cfg", PERSISTENT, ids=lambda c: c.name)
def test_persistent_attention_sampled_rows(cfg):
    runtime, tls = _rt()
    st, data = make_state(cfg)
    assert tls.tls_attn_kernel(st.shape) == "sparse_attn_mma_kernel"
    got = run_stages(st)
    for b, h in sample_rows(cfg, 8):
        check_row(cfg, data, got, st, b, h)
    # and once more through the fused step: the tickets reset after every call
    st.out.fill_(float("nan"))
    st.step()
    torch.cuda.synchronize()
    assert st.check_device_error() == 0
    assert np.array_equal(st.out.float().cpu().numpy(), got["out"])


# level-2 work too heavy for one cluster on the CUDA cores (G * R * candidates
# above 2^20, label channels the tensor-core scorer does not take): scores go
# to the workspace and the last CTA of each row selects
CHUNKED = [
    small("s_chunked_r64", batch=2, n_q_heads=16, n_kv_heads=2, ctx_len=8192, block_size=64, K_b=64, k=1500,
          n_label=64, seed=53),
    small("s_chunked_r8_g32", batch=1, n_q_heads=64, n_kv_heads=2, ctx_len=16384, block_size=64, K_b=128, k=3000,
          n_label=8, seed=54),
]


@pytest.mark.parametrize("cfg", CHUNKED, ids=lambda c: c.name)
def test_chunked_level2_all_rows(cfg):
    runtime, tls = _rt()
    st, data = make_state(cfg)
    assert tls.tls_token_kernel(st.shape, cfg.K_b, cfg.k)[0] == "token_select_kernel"
    got = run_stages(st)
    for b in range(cfg.batch):
        for h in range(cfg.n_kv_heads):
            check_row(cfg, data, got, st, b, h)
