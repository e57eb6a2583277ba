"""Ragged batches, partial last blocks, paged K/V and the per-token append,
on the GPU against the oracle.

Sequence b holds its first len_b tokens (tls_shape.seq_lens).  Per row: the
index over the held tokens is bit-exact; level 1 chooses among the sequence's
blocks only and pads its list with -1 when it has fewer than K_b; level 2
chooses among the held positions of those blocks and pads with -1 when there
are fewer than k; the attention skips the padding (a sequence with no token
gets a zero output and lse -inf).  Selections follow the tie band of
tests/parity.py; outputs the 2e-3 row-relative bound.  The append must leave
exactly the index a rebuild over the grown sequence gives.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import f32_from_bf16_bits
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


def shape_cfg(name, **kw):
    base = dict(name=name, description="ragged parity shape", batch=6, n_q_heads=8, n_kv_heads=2, qk_dim=128,
                v_dim=128, v_offset=-1, ctx_len=2048, block_size=16, K_b=12, k=100, n_label=16, seed=71,
                n_outlier=3, planted_per_row=16, planted_blocks=4, label_from_outliers=True)
    base.update(kw)
    return synth.WorkloadConfig(**base)


# (config, tokens per sequence): full, partial last blocks, fewer blocks than
# K_b, fewer candidates than k, one token, none
RAGGED = [
    (shape_cfg("r_gqa4_row"), [2048, 1000, 181, 37, 1, 0]),
    (shape_cfg("r_mla_g16", batch=3, n_q_heads=16, n_kv_heads=1, qk_dim=576, v_dim=512, v_offset=0, ctx_len=1024,
               block_size=64, K_b=6, k=200, n_label=32, n_outlier=0, label_from_outliers=False, kv_std=0.7071,
               seed=72), [1024, 300, 50]),
    (shape_cfg("r_g32_cluster", batch=3, n_q_heads=32, n_kv_heads=1, ctx_len=2048, K_b=10, k=120, seed=73),
     [2048, 555, 20]),
    (shape_cfg("r_d64_simt", batch=3, n_q_heads=12, n_kv_heads=2, qk_dim=64, v_dim=64, ctx_len=1024, K_b=9, k=144,
               n_label=8, seed=74), [1024, 333, 7]),
    (shape_cfg("r_chunked_r64", batch=2, n_q_heads=16, n_kv_heads=2, ctx_len=8192, block_size=64, K_b=64, k=1500,
               n_label=64, seed=75), [8192, 3001]),
    (shape_cfg("r_persistent", batch=80, n_q_heads=8, n_kv_heads=2, ctx_len=1024, K_b=9, k=133, seed=76),
     [int(x) for x in np.random.default_rng(76).integers(0, 1025, 80)]),
]


def _case(cfg, lens):
    runtime, tls = _rt()
    q = synth.gen_queries(cfg)
    K, V, _ = synth.gen_kv(cfg, q)
    lab = synth.gen_label_channels(cfg)
    st = runtime.state_for_config(cfg, q, K, V, lab, seq_lens=np.asarray(lens, dtype=np.int32))
    torch.cuda.synchronize()
    return st, (q, K, V, lab)


def _run(st):
    st.select_blocks(keep_scores=True)
    st.select_tokens(keep_scores=True)
    st.attend()
    torch.cuda.synchronize()
    assert st.check_device_error() == 0
    return dict(block_idx=st.block_idx.cpu().numpy(), token_idx=st.token_idx.cpu().numpy(),
                block_score=st.block_score.cpu().numpy(), token_score=st.token_score.cpu().numpy(),
                out=st.out.float().cpu().numpy(), lse=st.lse.cpu().numpy())


def check_ragged_row(cfg, data, got, st, b, h, n, check_index=True):
    q, K, V, lab = data
    g, bs = cfg.group, cfg.block_size
    kb = K[b, h, :n]
    vb = None if V is None else V[b, h, :n]
    nbr = -(-n // bs)
    where = f"{cfg.name} row ({b},{h}) len {n}"
    qg = q[b, h * g:(h + 1) * g]
    kw = dict(v_offset=cfg.v_offset, v_dim=cfg.v_dim)
    meta = oracle.block_meta(kb, bs)
    label = oracle.quant_label(kb, lab[h])
    if check_index and n > 0:
        gm = st.meta[b, h, :nbr].float().cpu().numpy().astype(np.float64)
        assert np.array_equal(gm[:, :cfg.qk_dim], meta[0]), f"{where}: kmax differs"
        assert np.array_equal(gm[:, cfg.qk_dim:], meta[1]), f"{where}: kmin differs"
        assert np.array_equal(st.codes[b, h, :n].cpu().numpy(), oracle.pack_codes(label[0])), f"{where}: codes"
        assert np.array_equal(st.scales[b, h, :n].cpu().numpy().view(np.uint32), label[1].view(np.uint32)), \
            f"{where}: scales"

    # level 1: only the sequence's blocks compete; the list is padded with -1
    kk_b = min(cfg.K_b, nbr)
    gb_all = got["block_idx"][b, h]
    assert np.all(gb_all[kk_b:] == -1), f"{where}: block list not padded with -1"
    assert np.all(np.isneginf(got["block_score"][b, h, nbr:])), f"{where}: scores past the sequence"
    gb = gb_all[:kk_b]
    r1 = oracle.decode_row(qg, kb, vb, lab[h], bs, cfg.K_b, cfg.k, cfg.softmax_scale, meta=meta, label=label, **kw)
    if kk_b > 0:
        agg = r1["agg"]
        assert np.max(np.abs(got["block_score"][b, h, :nbr] - agg)) <= 1e-5 * np.max(np.abs(agg)), f"{where}: scores"
        check_selection(gb, agg, kk_b, where + " blocks")

    # level 2 among the held positions of the GPU's blocks; padded with -1
    r2 = oracle.decode_row(qg, kb, vb, lab[h], bs, cfg.K_b, cfg.k, cfg.softmax_scale, meta=meta, label=label,
                           block_idx=gb, **kw)
    cand, ts = r2["cand"], r2["token_score"]
    kk_t = min(cfg.k, cand.size)
    gt_all = got["token_idx"][b, h]
    assert np.all(gt_all[kk_t:] == -1), f"{where}: token list not padded with -1"
    assert np.all(np.isneginf(got["token_score"][b, h, cand.size:])), f"{where}: scores past the candidates"
    gt = gt_all[:kk_t]
    if kk_t > 0:
        assert np.max(np.abs(got["token_score"][b, h, :cand.size] - ts)) <= 1e-5 * np.max(np.abs(ts)), \
            f"{where}: token scores"
        pos = np.searchsorted(cand, gt)
        assert np.all(pos < cand.size) and np.array_equal(cand[np.minimum(pos, cand.size - 1)], gt), \
            f"{where}: token outside the candidates"
        check_selection(pos, ts, kk_t, where + " tokens")

    # attention over the GPU's tokens (none: zero output, lse -inf)
    r3 = oracle.decode_row(qg, kb, vb, lab[h], bs, cfg.K_b, cfg.k, cfg.softmax_scale, meta=meta, label=label,
                           block_idx=gb, token_idx=gt, **kw)
    out = got["out"][b, h * g:(h + 1) * g]
    lse = got["lse"][b, h * g:(h + 1) * g]
    if kk_t == 0:
        assert np.all(out == 0.0) and np.all(np.isneginf(lse)), f"{where}: empty sequence"
    else:
        check_output(out, r3["out"], where + " out")
        assert np.max(np.abs(lse - r3["lse"])) <= 1e-4 * max(1.0, np.max(np.abs(r3["lse"]))), f"{where}: lse"


def _rows(cfg, lens, n=None):
    rows = [(b, h) for b in range(cfg.batch) for h in range(cfg.n_kv_heads)]
    if n is None or len(rows) <= n:
        return rows
    rng = np.random.default_rng(cfg.seed)
    pick = set(rng.choice(len(rows), n, replace=False).tolist())
    # always the shortest and longest sequences
    pick |= {int(np.argmin(lens)) * cfg.n_kv_heads, int(np.argmax(lens)) * cfg.n_kv_heads}
    return [rows[i] for i in sorted(pick)]


@pytest.mark.parametrize("case", RAGGED, ids=lambda c: c[0].name)
def test_ragged_batch_follows_the_oracle(case):
    cfg, lens = case
    st, data = _case(cfg, lens)
    got = _run(st)
    for b, h in _rows(cfg, lens, 10):
        check_ragged_row(cfg, data, got, st, b, h, lens[b])
    # the fused step gives the same lists and outputs
    st.block_idx.fill_(7)
    st.token_idx.fill_(7)
    st.step()
    torch.cuda.synchronize()
    assert np.array_equal(st.block_idx.cpu().numpy(), got["block_idx"])
    assert np.array_equal(st.token_idx.cpu().numpy(), got["token_idx"])
    assert np.array_equal(st.out.float().cpu().numpy(), got["out"])


def test_paged_kv_of_a_ragged_batch():
    # K/V blocks scattered over a shuffled page pool and read through the slot
    # table (pages only for the blocks each sequence holds): the same output as
    # the dense cache, bit for bit
    runtime, tls = _rt()
    cfg, lens = RAGGED[0]
    st, data = _case(cfg, lens)
    got = _run(st)
    rows, nb, bs = cfg.rows, cfg.n_blocks, cfg.block_size
    held = [(b, h, j) for b in range(cfg.batch) for h in range(cfg.n_kv_heads) for j in range(-(-lens[b] // bs))]
    perm = np.random.default_rng(5).permutation(len(held) + 11)[:len(held)]
    n_slots = len(held) + 11
    table = np.full((cfg.batch, cfg.n_kv_heads, nb), -1, dtype=np.int32)
    pool_k = torch.zeros((n_slots, bs, cfg.qk_dim), dtype=torch.bfloat16, device="cuda")
    pool_v = torch.zeros((n_slots, bs, cfg.v_dim), dtype=torch.bfloat16, device="cuda")
    for (b, h, j), s in zip(held, perm):
        table[b, h, j] = s
        pool_k[s] = st.kc[b, h, j * bs:(j + 1) * bs]
        pool_v[s] = st.vc[b, h, j * bs:(j + 1) * bs]
    kv = tls.make_kv_view(pool_k, pool_v, cfg.qk_dim, cfg.v_dim, torch.from_numpy(table).cuda(), n_slots)
    dense = st.out.clone()
    st.out.fill_(float("nan"))
    st.attend(kv=kv)
    torch.cuda.synchronize()
    assert torch.equal(st.out, dense)


# token lists holding -1 entries with every sequence full (no seq_lens): the
# attention skips them wherever they stand.  Shapes reaching the cluster and
# persistent tensor-core kernels, the MLA kernel and the CUDA-core kernel.
HOLES = [
    (shape_cfg("h_gqa4_cluster", ctx_len=1024), "sparse_attn_mma_cluster_kernel"),
    (shape_cfg("h_gqa4_persistent", batch=80, ctx_len=1024, K_b=9, k=133, seed=77), "sparse_attn_mma_kernel"),
    (RAGGED[1][0], "sparse_attn_mla_kernel"),
    (RAGGED[3][0], "sparse_attn_kernel"),
]


@pytest.mark.parametrize("case", HOLES, ids=lambda c: c[0].name)
def test_minus_one_entries_are_skipped(case):
    runtime, tls = _rt()
    cfg, kernel = case
    q = synth.gen_queries(cfg)
    K, V, _ = synth.gen_kv(cfg, q)
    lab = synth.gen_label_channels(cfg)
    st = runtime.state_for_config(cfg, q, K, V, lab)
    assert tls.tls_attn_kernel(st.shape) == kernel
    st.select()
    torch.cuda.synchronize()
    lists = st.token_idx.cpu().numpy().reshape(cfg.rows, cfg.k).copy()
    rng = np.random.default_rng(cfg.seed + 1)
    for r in range(cfg.rows):
        kind = r % 4
        if kind == 0:      # a padded tail
            lists[r, cfg.k // 2:] = -1
        elif kind == 1:    # the first 16 entries (a whole chunk) and every 7th entry
            lists[r, :16] = -1
            lists[r, ::7] = -1
        elif kind == 2:    # scattered holes, some out of range
            hole = rng.random(cfg.k) < 0.3
            lists[r, hole] = rng.choice([-1, -5, cfg.ctx_len, cfg.ctx_len + 9], int(hole.sum()))
    lists[1 % cfg.rows] = -1  # a row with no token
    st.token_idx.copy_(torch.from_numpy(lists.reshape(st.token_idx.shape)).cuda())
    st.attend()
    torch.cuda.synchronize()
    assert st.check_device_error() == 0
    out = st.out.float().cpu().numpy()
    lse = st.lse.cpu().numpy()
    g = cfg.group
    for r in _rows_sample(cfg):
        b, h = divmod(r, cfg.n_kv_heads)
        where = f"{cfg.name} row ({b},{h})"
        keep = lists[r][(lists[r] >= 0) & (lists[r] < cfg.ctx_len)]
        o = out[b, h * g:(h + 1) * g]
        ls = lse[b, h * g:(h + 1) * g]
        if keep.size == 0:
            assert np.all(o == 0.0) and np.all(np.isneginf(ls)), f"{where}: empty list"
            continue
        kf = f32_from_bf16_bits(K[b, h, keep]).astype(np.float64)
        vf = kf[:, cfg.v_offset:cfg.v_offset + cfg.v_dim] if V is None else \
            f32_from_bf16_bits(V[b, h, keep]).astype(np.float64)
        ref_out, ref_lse = oracle.attention(f32_from_bf16_bits(q[b, h * g:(h + 1) * g]).astype(np.float64), kf, vf,
                                            cfg.softmax_scale)
        check_output(o, ref_out, where + " out")
        assert np.max(np.abs(ls - ref_lse)) <= 1e-4 * max(1.0, np.max(np.abs(ref_lse))), f"{where}: lse"


def _rows_sample(cfg, n=12):
    rows = list(range(cfg.rows))
    if len(rows) <= n:
        return rows
    pick = set(np.random.default_rng(cfg.seed).choice(len(rows), n, replace=False).tolist()) | {0, 1, 2, 3}
    return sorted(pick)


APPEND = [
    (shape_cfg("a_gqa4", batch=4, ctx_len=256, block_size=16, K_b=6, k=40, seed=81), [100, 63, 64, 0], 22),
    (shape_cfg("a_mla", batch=2, n_q_heads=16, n_kv_heads=1, qk_dim=576, v_dim=512, v_offset=0, ctx_len=512,
               block_size=64, K_b=4, k=100, n_label=32, n_outlier=0, label_from_outliers=False, kv_std=0.7071,
               seed=82), [127, 500], 14),
]


@pytest.mark.parametrize("case", APPEND, ids=lambda c: c[0].name)
@pytest.mark.parametrize("paged", [False, True], ids=["dense", "paged"])
def test_append_equals_rebuilding_the_index(case, paged):
    runtime, tls = _rt()
    cfg, lens0, steps = case
    q = synth.gen_queries(cfg)
    K, V, _ = synth.gen_kv(cfg, q)
    lab = synth.gen_label_channels(cfg)
    # the cache holds only each sequence's first tokens; the rest is zero and must be written by the appends
    Kc, Vc = K.copy(), (V.copy() if V is not None else None)
    for b, n in enumerate(lens0):
        Kc[b, :, n:] = 0
        if Vc is not None:
            Vc[b, :, n:] = 0
    st = runtime.state_for_config(cfg, q, Kc, Vc, lab, seq_lens=np.asarray(lens0, dtype=np.int32))
    bs, nb = cfg.block_size, cfg.n_blocks
    kv = None
    if paged:
        # every block of every row gets a page of a shuffled pool, filled from the dense cache
        n_slots = cfg.rows * nb
        perm = np.random.default_rng(3).permutation(n_slots).astype(np.int32).reshape(cfg.batch, cfg.n_kv_heads, nb)
        pool_k = torch.empty((n_slots, bs, cfg.qk_dim), dtype=torch.bfloat16, device="cuda")
        pool_k[torch.from_numpy(perm).long().cuda().reshape(-1)] = st.kc.reshape(-1, bs, cfg.qk_dim)
        pool_v = None
        if st.vc is not None:
            pool_v = torch.empty((n_slots, bs, cfg.v_dim), dtype=torch.bfloat16, device="cuda")
            pool_v[torch.from_numpy(perm).long().cuda().reshape(-1)] = st.vc.reshape(-1, bs, cfg.v_dim)
        kv = tls.make_kv_view(pool_k, pool_v if pool_v is not None else pool_k, cfg.qk_dim,
                              cfg.v_dim if pool_v is not None else cfg.qk_dim, torch.from_numpy(perm).cuda(), n_slots)
    lens = list(lens0)
    for _ in range(steps):
        k_new = np.stack([K[b, :, min(lens[b], cfg.ctx_len - 1)] for b in range(cfg.batch)])
        kd = torch.from_numpy(k_new.view(np.int16)).cuda().view(torch.bfloat16)
        vd = None
        if V is not None:
            v_new = np.stack([V[b, :, min(lens[b], cfg.ctx_len - 1)] for b in range(cfg.batch)])
            vd = torch.from_numpy(v_new.view(np.int16)).cuda().view(torch.bfloat16)
        if paged:
            tls.tls_append_kv(st.shape, st.seq_lens, kd, vd, kv, st.meta, st.label_ch, st.codes, st.scales)
        else:
            st.append(kd, vd)
        lens = [min(n + 1, cfg.ctx_len) for n in lens]
    torch.cuda.synchronize()
    assert st.seq_lens.cpu().numpy().tolist() == lens
    # the cache rows and the index equal a rebuild over the grown sequences
    got_k = (pool_k[torch.from_numpy(perm).long().cuda()].reshape(cfg.batch, cfg.n_kv_heads, -1, cfg.qk_dim)
             if paged else st.kc)
    got_k = got_k.view(torch.int16).cpu().numpy().view(np.uint16)
    for b in range(cfg.batch):
        for h in range(cfg.n_kv_heads):
            n = lens[b]
            assert np.array_equal(got_k[b, h, :n], K[b, h, :n]), f"row ({b},{h}): K rows"
    if paged:
        st.kv = kv
        if st.vc is not None:
            got_v = pool_v[torch.from_numpy(perm).long().cuda()].reshape(cfg.batch, cfg.n_kv_heads, -1, cfg.v_dim)
            got_v = got_v.view(torch.int16).cpu().numpy().view(np.uint16)
            for b in range(cfg.batch):
                assert np.array_equal(got_v[b, :, :lens[b]], V[b, :, :lens[b]])
    got = _run(st)
    for b in range(cfg.batch):
        for h in range(cfg.n_kv_heads):
            check_ragged_row(cfg, (q, K, V, lab), got, st, b, h, lens[b])


def test_resident_engine_on_a_ragged_batch():
    # the staggered engine over the same ragged batch: step t within the GPU's
    # M_{t-1}, with the padding rules of each level
    runtime, tls = _rt()
    cfg, lens = RAGGED[0]
    qs = synth.gen_query_trajectory(cfg.scaled(q_drift=0.3), 3)
    K, V, _ = synth.gen_kv(cfg, qs[0])
    lab = synth.gen_label_channels(cfg)
    st = runtime.state_for_config(cfg, qs[0], K, V, lab, seq_lens=np.asarray(lens, dtype=np.int32))
    eng = runtime.ResidentEngine(st)
    g = cfg.group
    try:
        for t, qb in enumerate(qs):
            qd = torch.from_numpy(np.ascontiguousarray(qb).view(np.int16)).cuda().view(torch.bfloat16)
            eng.step(qd)
            torch.cuda.synchronize()
            assert eng.check_device_error() == 0
            m_prev = eng.block_idx[(t + 1) & 1].cpu().numpy()
            tok = eng.token_idx.cpu().numpy()
            out = eng.out.float().cpu().numpy()
            for b in range(cfg.batch):
                n = lens[b]
                for h in range(cfg.n_kv_heads):
                    kb, vb = K[b, h, :n], V[b, h, :n]
                    nbr = -(-n // cfg.block_size)
                    gb = m_prev[b, h][:min(cfg.K_b, nbr)]
                    assert np.all(m_prev[b, h][gb.size:] == -1)
                    r = oracle.decode_row(qb[b, h * g:(h + 1) * g], kb, vb, lab[h], cfg.block_size, cfg.K_b, cfg.k,
                                          cfg.softmax_scale, block_idx=gb)
                    kk = min(cfg.k, r["cand"].size)
                    assert np.all(tok[b, h][kk:] == -1)
                    gt = tok[b, h][:kk]
                    if kk:
                        check_selection(np.searchsorted(r["cand"], gt), r["token_score"], kk, f"step {t} ({b},{h})")
                        r3 = oracle.decode_row(qb[b, h * g:(h + 1) * g], kb, vb, lab[h], cfg.block_size, cfg.K_b,
                                               cfg.k, cfg.softmax_scale, block_idx=gb, token_idx=gt)
                        check_output(out[b, h * g:(h + 1) * g], r3["out"], f"step {t} ({b},{h}) out")
                    else:
                        assert np.all(out[b, h * g:(h + 1) * g] == 0.0)
    finally:
        eng.close()
