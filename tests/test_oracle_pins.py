"""Pins that tie the oracle to facts other than itself (CPU only).

Each test checks a function of oracle/two_level.py against a closed form, a
theorem, a brute-force enumeration, a library routine or a hand-worked
example, so that a dropped term, a flipped sign, a wrong index or a transposed
operand in the oracle fails at least one of them.
"""

import json
import math
import os
import random

import numpy as np
import pytest
import torch

import oracle
from synth import bf16_bits_from_f32, f32_from_bf16_bits, get_config, gen_queries, gen_row, gen_label_channels

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")))


def bits(x):
    return bf16_bits_from_f32(np.asarray(x, dtype=np.float32))


def rand_bits(rng, shape, scale=1.0):
    return bits(rng.standard_normal(shape).astype(np.float32) * scale)


# ---------------------------------------------------------------- generator

def test_bf16_rounding_is_nearest_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties to even -> 1.0
    x = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5, 0.0], dtype=np.float32)
    b = bf16_bits_from_f32(x)
    back = f32_from_bf16_bits(b)
    assert back[0] == 1.0
    assert back[1] == np.float32(1.0 + 2 * 2.0 ** -7)
    assert back[2] == -2.5 and back[3] == 0.0
    # agrees with torch's own bf16 conversion on random data
    r = np.random.default_rng(0).standard_normal(10000).astype(np.float32) * 37
    ref = torch.from_numpy(r).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bf16_bits_from_f32(r), ref)


# ---------------------------------------------------------------- block meta

def test_block_meta_brute_force():
    rng = np.random.default_rng(1)
    kb = rand_bits(rng, (24, 5))
    kmax, kmin = oracle.block_meta(kb, 4)
    k = f32_from_bf16_bits(kb).astype(np.float64)
    for j in range(6):
        for c in range(5):
            vals = [float(k[t, c]) for t in range(4 * j, 4 * j + 4)]
            assert kmax[j, c] == max(vals)
            assert kmin[j, c] == min(vals)


# ---------------------------------------------------------------- block scores

def test_block_score_worked_example():
    g = GOLD["block"]
    kb = bits(g["keys"])
    kmax, kmin = oracle.block_meta(kb, 2)
    assert kmax[0].tolist() == g["kmax"] and kmin[0].tolist() == g["kmin"]
    s = oracle.block_scores(np.array([g["q"]]), kmax, kmin)
    assert s[0, 0] == g["score"]


@pytest.mark.parametrize("seed", range(4))
def test_quest_bound_holds_for_every_head_and_token(seed):
    # S[h, j] >= q_h . k_t for every token t of block j (the Quest upper bound)
    rng = np.random.default_rng(seed)
    n, d, bs, g = 64, 16, 8, 3
    kb = rand_bits(rng, (n, d), 3.0)
    q = f32_from_bf16_bits(rand_bits(rng, (g, d))).astype(np.float64)
    kmax, kmin = oracle.block_meta(kb, bs)
    s = oracle.block_scores(q, kmax, kmin)
    k = f32_from_bf16_bits(kb).astype(np.float64)
    for h in range(g):
        for t in range(n):
            dot = sum(q[h, c] * k[t, c] for c in range(d))
            assert s[h, t // bs] >= dot - 1e-9 * (1 + abs(dot))
    # the bound is attained when a block holds a single token
    kmax1, kmin1 = oracle.block_meta(kb, 1)
    s1 = oracle.block_scores(q, kmax1, kmin1)
    np.testing.assert_allclose(s1, q @ k.T, rtol=1e-12, atol=1e-12)


def test_quest_score_equals_gemm_form():
    # sum_c max(q_c kmax_c, q_c kmin_c) == [relu(q), min(q,0)] . [kmax; kmin]
    rng = np.random.default_rng(7)
    kb = rand_bits(rng, (256, 32), 2.0)
    q = f32_from_bf16_bits(rand_bits(rng, (5, 32))).astype(np.float64)
    kmax, kmin = oracle.block_meta(kb, 16)
    s = oracle.block_scores(q, kmax, kmin)
    qq = np.concatenate([np.maximum(q, 0), np.minimum(q, 0)], axis=1)
    mm = np.concatenate([kmax, kmin], axis=1)
    np.testing.assert_allclose(s, qq @ mm.T, rtol=1e-13, atol=1e-12)


def test_group_max():
    s = np.array([[1.0, -3.0, 2.0], [0.5, -1.0, 4.0]])
    assert oracle.group_max(s).tolist() == [1.0, -1.0, 4.0]


# ---------------------------------------------------------------- top-k

def test_topk_worked_example():
    g = GOLD["topk"]
    assert oracle.topk_ascending(np.array(g["scores"]), g["k"]).tolist() == g["selected"]


@pytest.mark.parametrize("seed", range(30))
def test_topk_matches_exhaustive_enumeration(seed):
    rnd = random.Random(seed)
    n = rnd.randint(1, 9)
    k = rnd.randint(1, n)
    scores = [float(rnd.choice([-1.0, 0.0, 0.5, 0.5, 2.0, 3.0])) for _ in range(n)]
    # exhaustive: among all k-subsets, the chosen one maximises the sorted score
    # vector, then prefers lower indices (lexicographically smallest index list)
    import itertools
    best = None
    for sub in itertools.combinations(range(n), k):
        key = (sorted((scores[i] for i in sub), reverse=True), [-i for i in sorted(sub)])
        if best is None or key > best[0]:
            best = (key, list(sub))
    got = oracle.topk_ascending(np.array(scores), k).tolist()
    assert got == sorted(best[1])


def test_topk_nan_ranks_last_and_extremes():
    s = np.array([np.nan, 1.0, -np.inf, 0.0])
    assert oracle.topk_ascending(s, 2).tolist() == [1, 3]
    assert oracle.topk_ascending(s, 4).tolist() == [0, 1, 2, 3]
    assert oracle.topk_ascending(np.zeros(5), 2).tolist() == [0, 1]


# ---------------------------------------------------------------- INT4 label cache

def test_int4_worked_example():
    g = GOLD["int4"]
    kb = bits([g["x"]])
    codes, scales = oracle.quant_label(kb, np.arange(4))
    assert scales[0] == np.float32(g["scale"])
    assert codes[0].tolist() == g["codes"]
    assert oracle.pack_codes(codes)[0].tolist() == g["packed"]
    assert oracle.unpack_codes(oracle.pack_codes(codes)).tolist() == codes.tolist()


def test_int4_exact_halves_round_to_even():
    # x / s lands exactly on n + 1/2 for seven of the eight channels: the codes
    # pin the tie rule (half to even), which no random input exercises
    g = GOLD["int4_ties"]
    kb = bits([g["x"]])
    codes, scales = oracle.quant_label(kb, np.arange(len(g["x"])))
    assert scales[0] == np.float32(g["scale"])
    assert codes[0].tolist() == g["codes"]


def test_int4_round_trip_within_half_step():
    rng = np.random.default_rng(3)
    kb = rand_bits(rng, (2000, 40), 5.0)
    label = np.sort(rng.choice(40, 16, replace=False))
    codes, scales = oracle.quant_label(kb, label)
    x = f32_from_bf16_bits(kb)[:, label].astype(np.float64)
    s = scales.astype(np.float64)[:, None]
    err = np.abs(x - s * codes)
    assert np.all(err <= s / 2 * (1 + 1e-6))
    assert codes.min() >= -7 and codes.max() <= 7
    # the largest |x| of each token maps to +-7
    amax = np.argmax(np.abs(x), axis=1)
    assert np.all(np.abs(codes[np.arange(len(x)), amax]) == 7)


def test_int4_zero_row_and_exact_multiples():
    kb = bits([[0.0, 0.0, 0.0, 0.0], [0.75, -0.375, 0.0, 2.625]])
    codes, scales = oracle.quant_label(kb, np.arange(4))
    assert scales[0] == 0 and codes[0].tolist() == [0, 0, 0, 0]
    # 2.625/7 = 0.375: every value is an exact multiple, so dequantisation is exact
    assert scales[1] == np.float32(0.375)
    assert (codes[1].astype(np.float64) * 0.375).tolist() == [0.75, -0.375, 0.0, 2.625]


def test_pack_nibble_layout_exhaustive():
    allc = np.array([[a, b] for a in range(-7, 8) for b in range(-7, 8)], dtype=np.int8)
    p = oracle.pack_codes(allc)
    for (a, b), byte in zip(allc.tolist(), p[:, 0].tolist()):
        assert byte == ((a % 16) | ((b % 16) << 4))
    assert np.array_equal(oracle.unpack_codes(p), allc)


# ---------------------------------------------------------------- token scores

def test_token_score_equals_exact_dot_when_quantisation_is_exact():
    # keys whose label values are integers in [-7, 7] with max |.| = 7 quantise
    # exactly, so the approximate score is the true partial dot product.
    rng = np.random.default_rng(5)
    n, d, g = 40, 12, 3
    label = np.array([1, 4, 5, 9])
    k = rng.standard_normal((n, d)).astype(np.float32)
    ints = rng.integers(-6, 7, size=(n, 4)).astype(np.float32)
    ints[:, 2] = np.where(rng.random(n) < 0.5, 7.0, -7.0)
    k[:, label] = ints * np.float32(0.5)
    kb = bits(k)
    codes, scales = oracle.quant_label(kb, label)
    q = f32_from_bf16_bits(rand_bits(rng, (g, d))).astype(np.float64)
    cand = np.arange(n)
    ts = oracle.token_scores(q, label, codes, scales, cand)
    kk = f32_from_bf16_bits(kb).astype(np.float64)
    for t in range(n):
        best = max(sum(q[h, c] * kk[t, c] for c in label) for h in range(g))
        assert abs(ts[t] - best) <= 1e-12 * (1 + abs(best))


def test_candidate_tokens():
    assert oracle.candidate_tokens(np.array([3, 0]), 2).tolist() == [0, 1, 6, 7]


# ---------------------------------------------------------------- attention

def test_attention_worked_example():
    g = GOLD["attention"]
    out, lse = oracle.attention(np.array(g["q"]), np.array(g["keys"]), np.array(g["values"]), g["softmax_scale"])
    np.testing.assert_allclose(out, g["out"], rtol=1e-14)
    np.testing.assert_allclose(lse, g["lse"], rtol=1e-14)


def test_attention_matches_torch_sdpa_float64():
    rng = np.random.default_rng(11)
    g, n, d, dv = 4, 50, 16, 12
    q = rng.standard_normal((g, d))
    k = rng.standard_normal((n, d)) * 3
    v = rng.standard_normal((n, dv))
    sc = 0.37
    out, lse = oracle.attention(q, k, v, sc)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, :, None, :], torch.from_numpy(k)[None, None].expand(1, g, n, d),
        torch.from_numpy(v)[None, None].expand(1, g, n, dv), scale=sc)[0, :, 0, :].numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
    ref_lse = torch.logsumexp(torch.from_numpy(sc * q @ k.T), dim=1).numpy()
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-13)


def _small_row(seed=0, n=256, d=32, dv=24, g=4, bs=16, r=8):
    rng = np.random.default_rng(seed)
    kb = rand_bits(rng, (n, d))
    vb = rand_bits(rng, (n, dv))
    qb = rand_bits(rng, (g, d))
    label = np.sort(rng.choice(d, r, replace=False)).astype(np.int32)
    return qb, kb, vb, label, bs


def test_select_everything_equals_dense_attention():
    # K_b = all blocks and k = all tokens removes every approximation
    qb, kb, vb, label, bs = _small_row()
    n = kb.shape[0]
    res = oracle.decode_row(qb, kb, vb, label, bs, n // bs, n, 0.2)
    assert res["block_idx"].tolist() == list(range(n // bs))
    assert res["token_idx"].tolist() == list(range(n))
    q = f32_from_bf16_bits(qb).astype(np.float64)
    k = f32_from_bf16_bits(kb).astype(np.float64)
    v = f32_from_bf16_bits(vb).astype(np.float64)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[:, None, :], torch.from_numpy(k)[None].expand(q.shape[0], -1, -1),
        torch.from_numpy(v)[None].expand(q.shape[0], -1, -1), scale=0.2)[:, 0, :].numpy()
    np.testing.assert_allclose(res["out"], ref, rtol=1e-12, atol=1e-13)


def test_sparse_attention_is_attention_over_the_gathered_rows():
    qb, kb, vb, label, bs = _small_row(seed=3)
    res = oracle.decode_row(qb, kb, vb, label, bs, 4, 32, 0.25)
    idx = res["token_idx"]
    assert len(idx) == 32 and np.all(np.diff(idx) > 0)
    assert set((idx // bs).tolist()) <= set(res["block_idx"].tolist())
    q = torch.from_numpy(f32_from_bf16_bits(qb).astype(np.float64))
    k = torch.from_numpy(f32_from_bf16_bits(kb[idx]).astype(np.float64))
    v = torch.from_numpy(f32_from_bf16_bits(vb[idx]).astype(np.float64))
    ref = torch.softmax(0.25 * q @ k.T, dim=1) @ v
    np.testing.assert_allclose(res["out"], ref.numpy(), rtol=1e-12, atol=1e-13)
    # the chosen tokens are the top-k of the token scores over the candidates
    cand = oracle.candidate_tokens(res["block_idx"], bs)
    ts = res["token_score"]
    chosen = np.isin(cand, idx)
    assert ts[chosen].min() >= ts[~chosen].max()


def test_mla_value_slice():
    rng = np.random.default_rng(4)
    n, d, dv, bs = 128, 40, 32, 8
    kb = rand_bits(rng, (n, d))
    qb = rand_bits(rng, (6, d))
    label = np.arange(0, 40, 5).astype(np.int32)
    res = oracle.decode_row(qb, kb, None, label, bs, 4, 16, 0.1, v_offset=0, v_dim=dv)
    res2 = oracle.decode_row(qb, kb, kb[:, :dv].copy(), label, bs, 4, 16, 0.1)
    np.testing.assert_array_equal(res["out"], res2["out"])


# ---------------------------------------------------------------- staggering / transfer

def test_staggered_step_reduces_to_the_synchronous_step():
    qb, kb, vb, label, bs = _small_row(seed=5)
    a = oracle.staggered_row(qb, qb, kb, vb, label, bs, 4, 32, 0.25)
    b = oracle.decode_row(qb, kb, vb, label, bs, 4, 32, 0.25)
    assert a["token_idx"].tolist() == b["token_idx"].tolist()
    np.testing.assert_array_equal(a["out"], b["out"])


def test_staggered_step_takes_blocks_from_the_previous_query():
    qb, kb, vb, label, bs = _small_row(seed=6)
    rng = np.random.default_rng(9)
    q_prev = rand_bits(rng, qb.shape)
    a = oracle.staggered_row(q_prev, qb, kb, vb, label, bs, 4, 32, 0.25)
    b_prev = oracle.decode_row(q_prev, kb, vb, label, bs, 4, 32, 0.25)
    assert a["block_idx"].tolist() == b_prev["block_idx"].tolist()
    c = oracle.decode_row(qb, kb, vb, label, bs, 4, 32, 0.25, block_idx=b_prev["block_idx"])
    np.testing.assert_array_equal(a["out"], c["out"])


def test_plan_transfer_set_difference():
    assert oracle.plan_transfer([5, 1, 9, 3], [1, 2, 3]).tolist() == [5, 9]
    assert oracle.plan_transfer([1, 2], [1, 2, 3]).tolist() == []


# ---------------------------------------------------------------- workload sanity

def test_c1_planted_tokens_carry_the_largest_exact_logits():
    # Sanity of the synthetic workload (not a statement of the pages): each
    # planted key leans 0.8*sqrt(d) along its head's query, so for its head it
    # outranks almost every unplanted token by the exact logit q.k.
    cfg = get_config("c1")
    q = gen_queries(cfg)
    row = gen_row(cfg, 0, 0, q)
    qf = f32_from_bf16_bits(q[0]).astype(np.float64)
    k = f32_from_bf16_bits(row.k).astype(np.float64)
    logits = qf @ k.T  # [G, N]
    mask = np.zeros(cfg.ctx_len, dtype=bool)
    mask[row.planted_pos] = True
    for h in range(cfg.group):
        mine = row.planted_pos[row.planted_head == h]
        assert mine.size == cfg.planted_per_row // cfg.group
        assert logits[h, mine].mean() > np.quantile(logits[h, ~mask], 0.999)


# ---------------------------------------------------------------- ragged sequences, partial blocks

def test_block_meta_partial_last_block_brute_force():
    # 37 tokens in blocks of 8: four full blocks and one holding tokens 32..36
    rng = np.random.default_rng(61)
    kb = rand_bits(rng, (37, 6))
    kmax, kmin = oracle.block_meta(kb, 8)
    assert kmax.shape == (5, 6)
    k = f32_from_bf16_bits(kb).astype(np.float64)
    for j in range(5):
        rows = range(8 * j, min(37, 8 * j + 8))
        for c in range(6):
            assert kmax[j, c] == max(float(k[t, c]) for t in rows)
            assert kmin[j, c] == min(float(k[t, c]) for t in rows)


def test_block_meta_grows_by_running_max_min():
    # adding one token at a time changes only its block, whose max/min is the
    # channel-wise max/min of the old one and the new key (a fresh block: the key)
    rng = np.random.default_rng(62)
    kb = rand_bits(rng, (29, 4))
    k = f32_from_bf16_bits(kb).astype(np.float64)
    for n in range(1, 29):
        a_max, a_min = oracle.block_meta(kb[:n], 5)
        b_max, b_min = oracle.block_meta(kb[:n + 1], 5)
        j = n // 5
        if n % 5 == 0:
            assert np.array_equal(b_max[j], k[n]) and np.array_equal(b_min[j], k[n])
        else:
            assert np.array_equal(b_max[j], np.maximum(a_max[j], k[n]))
            assert np.array_equal(b_min[j], np.minimum(a_min[j], k[n]))
        assert np.array_equal(b_max[:j], a_max[:j]) and np.array_equal(b_min[:j], a_min[:j])


def test_candidates_are_the_held_positions_of_the_chosen_blocks():
    c = oracle.candidate_tokens(np.array([4, 0, 2]), 4, n_tokens=18)
    assert c.tolist() == [0, 1, 2, 3, 8, 9, 10, 11, 16, 17]
    assert oracle.candidate_tokens(np.array([1]), 4).tolist() == [4, 5, 6, 7]


def test_short_sequence_takes_every_block_and_candidate():
    # fewer blocks than K_b and fewer candidates than k: both levels take all,
    # and the step is then full attention over the held tokens
    rng = np.random.default_rng(63)
    g, d, n, bs = 3, 16, 21, 8
    q = rand_bits(rng, (g, d))
    kb = rand_bits(rng, (n, d))
    vb = rand_bits(rng, (n, d))
    lab = np.array([1, 5, 7, 12])
    r = oracle.decode_row(q, kb, vb, lab, bs, K_b=9, k=500, softmax_scale=0.25)
    assert r["block_idx"].tolist() == [0, 1, 2]
    assert r["token_idx"].tolist() == list(range(n))
    qq = torch.from_numpy(f32_from_bf16_bits(q).astype(np.float64))
    kk = torch.from_numpy(f32_from_bf16_bits(kb).astype(np.float64))
    vv = torch.from_numpy(f32_from_bf16_bits(vb).astype(np.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(qq[:, None, :], kk[None].expand(g, -1, -1),
                                                           vv[None].expand(g, -1, -1), scale=0.25)[:, 0, :]
    assert np.allclose(r["out"], ref.numpy(), rtol=1e-12, atol=1e-12)


def test_empty_sequence_gives_zero_output_and_no_selection():
    q = bits([[1.0, 2.0]])
    r = oracle.decode_row(q, np.zeros((0, 2), np.uint16), np.zeros((0, 2), np.uint16), np.array([0, 1]), 4,
                          K_b=2, k=3, softmax_scale=1.0)
    assert r["block_idx"].size == 0 and r["token_idx"].size == 0
    assert r["out"].tolist() == [[0.0, 0.0]] and r["lse"][0] == -np.inf


# ---------------------------------------------------------------- operator baselines

def test_dense_row_is_softmax_attention():
    rng = np.random.default_rng(64)
    g, d, n = 4, 24, 57
    q, kb, vb = rand_bits(rng, (g, d)), rand_bits(rng, (n, d)), rand_bits(rng, (n, 16))
    out, lse = oracle.dense_row(q, kb, vb, 0.2)
    qq = torch.from_numpy(f32_from_bf16_bits(q).astype(np.float64))
    kk = torch.from_numpy(f32_from_bf16_bits(kb).astype(np.float64))
    vv = torch.from_numpy(f32_from_bf16_bits(vb).astype(np.float64))
    ref = torch.nn.functional.scaled_dot_product_attention(qq[:, None, :], kk[None].expand(g, -1, -1),
                                                           vv[None].expand(g, -1, -1), scale=0.2)[:, 0, :]
    assert np.allclose(out, ref.numpy(), rtol=1e-12, atol=1e-12)
    assert np.allclose(lse, torch.logsumexp(0.2 * qq @ kk.T, dim=1).numpy(), rtol=1e-12)
    # the MLA form: V is the K row slice
    out2, _ = oracle.dense_row(q, kb, None, 0.2, v_offset=4, v_dim=8)
    ref2 = torch.softmax(0.2 * qq @ kk.T, dim=1) @ kk[:, 4:12]
    assert np.allclose(out2, ref2.numpy(), rtol=1e-12, atol=1e-12)


def test_quest_row_attends_every_token_of_its_blocks():
    rng = np.random.default_rng(65)
    g, d, n, bs, K_b = 2, 16, 90, 8, 4
    q, kb, vb = rand_bits(rng, (g, d)), rand_bits(rng, (n, d)), rand_bits(rng, (n, d))
    lab = np.array([0, 3, 9, 15])
    r = oracle.quest_row(q, kb, vb, lab, bs, K_b, 0.25)
    meta = oracle.block_meta(kb, bs)
    agg = oracle.block_scores(f32_from_bf16_bits(q).astype(np.float64), *meta).max(axis=0)
    assert r["block_idx"].tolist() == sorted(np.argsort(-agg, kind="stable")[:K_b].tolist())
    want = [t for b in r["block_idx"] for t in range(b * bs, min(n, b * bs + bs))]
    assert r["token_idx"].tolist() == want
    ref, _ = oracle.dense_row(q, kb[want], vb[want], 0.25)
    assert np.allclose(r["out"], ref, rtol=1e-12, atol=1e-12)


def test_ds_row_with_every_token_is_full_attention():
    rng = np.random.default_rng(66)
    g, d, n, bs = 3, 16, 45, 8
    q, kb, vb = rand_bits(rng, (g, d)), rand_bits(rng, (n, d)), rand_bits(rng, (n, d))
    lab = np.array([2, 3, 11, 13])
    r = oracle.ds_row(q, kb, vb, lab, bs, n, 0.3)
    assert r["block_idx"].tolist() == list(range(6)) and r["token_idx"].tolist() == list(range(n))
    ref, _ = oracle.dense_row(q, kb, vb, 0.3)
    assert np.allclose(r["out"], ref, rtol=1e-12, atol=1e-12)
    # with a smaller budget: the top-k of the label scores over every held token
    r2 = oracle.ds_row(q, kb, vb, lab, bs, 10, 0.3)
    codes, scales = oracle.quant_label(kb, lab)
    ts = oracle.token_scores(f32_from_bf16_bits(q).astype(np.float64), lab, codes, scales, np.arange(n))
    assert r2["token_idx"].tolist() == sorted(sorted(range(n), key=lambda t: (-ts[t], t))[:10])
