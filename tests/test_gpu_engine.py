"""The staggered engine over an HBM block cache, on the GPU, against the oracle.

Step t: the blocks M_t chosen from q_t (checked against the oracle within the
tie band), the tokens and the attention of step t within the GPU's M_{t-1}
with q_t (the oracle's staggered row, re-run on the GPU's sets), and after the
last step the transfer invariants: every block of M_T is resident, its slot
holds exactly the host rows of K and V, and the slot table matches the
cache's host mirror.
"""

import os

import numpy as np
import pytest
import torch

import oracle
import synth
from parity import check_output, check_selection

pytestmark = pytest.mark.gpu


def _rt():
    from two_level_sparse_block_b200 import runtime, tls
    return runtime, tls


def offload(name, **kw):
    base = dict(name=name, description="small offload shape", batch=1, n_q_heads=16, n_kv_heads=1, qk_dim=128,
                v_dim=128, v_offset=-1, ctx_len=8192, block_size=64, K_b=16, k=512, n_label=16, seed=31,
                n_outlier=6, planted_per_row=64, planted_blocks=20, label_from_outliers=True, steps=6,
                offload=True, n_slots=32, q_drift=0.3)
    base.update(kw)
    return synth.WorkloadConfig(**base)


ENGINE = [
    offload("e_g16_persistent"),
    offload("e_mqa64_tc", n_q_heads=64, seed=32),
    offload("e_gqa4_cluster", batch=16, n_q_heads=16, n_kv_heads=4, ctx_len=4096, K_b=12, k=384, n_slots=24,
            seed=33, steps=4),
]


def _dev_q(q_bits):
    return torch.from_numpy(np.ascontiguousarray(q_bits).view(np.int16)).cuda().view(torch.bfloat16)


def _rows(cfg, n=3):
    rows = [(b, h) for b in range(cfg.batch) for h in range(cfg.n_kv_heads)]
    if len(rows) <= n:
        return rows
    rng = np.random.default_rng(cfg.seed)
    return [rows[0], rows[-1]] + [rows[i] for i in rng.choice(np.arange(1, len(rows) - 1), n - 2, replace=False)]


def _orow(cfg, q, K, V, lab, b, h, **kw):
    g = cfg.group
    return oracle.decode_row(q[b, h * g:(h + 1) * g], K[b, h], V[b, h], lab[h], cfg.block_size, cfg.K_b, cfg.k,
                             cfg.softmax_scale, **kw)


@pytest.mark.parametrize("planner", ["device", "host"])
@pytest.mark.parametrize("cfg", ENGINE, ids=lambda c: c.name)
def test_engine_follows_the_staggered_oracle(cfg, planner, monkeypatch):
    runtime, tls = _rt()
    monkeypatch.setenv("TLS_ENGINE_PLANNER", planner)
    qs = synth.gen_query_trajectory(cfg)
    K, V, _ = synth.gen_kv(cfg, qs[0])
    lab = synth.gen_label_channels(cfg)
    layer = runtime.offloaded_layer_for_config(cfg, K, V, lab)
    g = cfg.group
    try:
        copied = []
        for t, q in enumerate(qs):
            layer.step(_dev_q(q))
            torch.cuda.synchronize()
            assert layer.check_device_error() == 0
            m_prev = layer.block_idx[(t + 1) & 1].cpu().numpy()  # M_{t-1} (the prologue's M_{-1} at t = 0)
            m_cur = layer.block_idx[t & 1].cpu().numpy()         # M_t
            tok = layer.token_idx.cpu().numpy()
            out = layer.out.float().cpu().numpy()
            for b, h in _rows(cfg):
                where = f"{cfg.name} step {t} row ({b},{h})"
                # level 1 of step t chooses M_t from q_t
                r1 = _orow(cfg, q, K, V, lab, b, h)
                check_selection(m_cur[b, h], r1["agg"], cfg.K_b, where + " M_t")
                if t == 0:
                    check_selection(m_prev[b, h], r1["agg"], cfg.K_b, where + " M_-1")
                # level 2 and attention of step t within the GPU's M_{t-1}, with q_t
                r2 = _orow(cfg, q, K, V, lab, b, h, block_idx=m_prev[b, h])
                pos = np.searchsorted(r2["cand"], tok[b, h])
                assert np.array_equal(r2["cand"][pos], tok[b, h]), f"{where}: token outside M_t-1"
                check_selection(pos, r2["token_score"], cfg.k, where + " tokens")
                r3 = _orow(cfg, q, K, V, lab, b, h, block_idx=m_prev[b, h], token_idx=tok[b, h])
                check_output(out[b, h * g:(h + 1) * g], r3["out"], where + " out")
            copied.append(m_cur)
        torch.cuda.synchronize()

        # transfer invariants after the last step
        table = layer.slot_table.cpu().numpy()
        mirror = np.empty_like(table)
        tls.tls_block_cache_table(layer.cache, mirror)
        assert np.array_equal(table, mirror), "device slot table differs from the host mirror"
        slot_k = layer.slot_k.view(torch.int16).cpu().numpy().view(np.uint16)
        slot_v = layer.slot_v.view(torch.int16).cpu().numpy().view(np.uint16)
        bs = cfg.block_size
        last = copied[-1]
        for b in range(cfg.batch):
            for h in range(cfg.n_kv_heads):
                for blk in last[b, h]:
                    s = table[b, h, blk]
                    assert s >= 0, f"block {blk} of M_T not resident in row ({b},{h})"
                    assert np.array_equal(slot_k[s], K[b, h, blk * bs:(blk + 1) * bs]), "slot K differs"
                    assert np.array_equal(slot_v[s], V[b, h, blk * bs:(blk + 1) * bs]), "slot V differs"
        # occupancy: no slot holds two blocks
        used = table[table >= 0]
        assert used.size == np.unique(used).size

        # transfer figures: the prologue copies all of M_{-1}; later steps copy T_t = M_t \ C_t
        st = layer.stats(-1)
        assert st.n_copied == cfg.rows * cfg.K_b and st.copy_ms >= 0.0
        blk_bytes = cfg.block_size * (cfg.qk_dim + cfg.v_dim) * 2
        for t in range(len(qs) - 1):
            st = layer.stats(t)
            assert 0 <= st.n_copied <= cfg.rows * cfg.K_b
            assert st.bytes_copied == st.n_copied * blk_bytes
            assert st.copy_ms >= 0.0 and st.exposed_ms >= 0.0
        assert layer.stats(len(qs) - 1).exposed_ms == -1.0  # no later step has been issued
    finally:
        layer.close()


@pytest.mark.parametrize("pool", ["2K_b", "3K_b+5"])
@pytest.mark.parametrize("cfg", ENGINE, ids=lambda c: c.name)
def test_engine_planners_leave_the_same_tables(cfg, pool, monkeypatch):
    # the device planner keeps the slots its previous plan used (those of
    # M_{t-1}) without reading the list M_{t-1}; the host planner keeps the
    # slots of the list: step by step both engines copy as many blocks and
    # leave the same slot table (12 steps of the drifting trajectory; the
    # larger pool leaves older blocks resident, so the least-recently-used
    # order picks the victims)
    runtime, tls = _rt()
    n_slots = None if pool == "2K_b" else (3 * cfg.K_b + 5) * cfg.rows
    qs = synth.gen_query_trajectory(cfg, 12)
    K, V, _ = synth.gen_kv(cfg, qs[0])
    lab = synth.gen_label_channels(cfg)
    layers = []
    try:
        for planner in ("host", "device"):
            monkeypatch.setenv("TLS_ENGINE_PLANNER", planner)
            layers.append(runtime.offloaded_layer_for_config(cfg, K, V, lab, n_slots=n_slots))
        kernels = [tls.tls_engine_step_kernels(layer.engine) for layer in layers]
        assert kernels[1] == kernels[0] + 1  # plan + pull against the host planner's pull alone
        moved = 0
        for t, q in enumerate(qs):
            tabs = []
            for layer in layers:
                layer.step(_dev_q(q))
                torch.cuda.synchronize()
                assert layer.check_device_error() == 0
                tab = np.empty(tuple(layer.slot_table.shape), dtype=np.int32)
                tls.tls_block_cache_table(layer.cache, tab)
                tabs.append(tab)
            assert np.array_equal(tabs[0], tabs[1]), f"{cfg.name} step {t}: slot tables differ"
            if t > 0:
                n = [layer.stats(t - 1).n_copied for layer in layers]
                assert n[0] == n[1], f"{cfg.name} step {t - 1}: copied {n[1]} (device) vs {n[0]} (host)"
                moved += n[0]
        assert moved > 0  # the trajectory drifts: blocks were evicted and copied
    finally:
        for layer in layers:
            layer.close()


def test_engine_copy_failure_is_reported_and_sticks(monkeypatch):
    # host-side fault injection: the transfer of step 2 fails before anything
    # is issued; that step and every later one return TLS_ERR_COPY, and the
    # device stays healthy
    runtime, tls = _rt()
    cfg = ENGINE[0]
    qs = synth.gen_query_trajectory(cfg, 4)
    K, V, _ = synth.gen_kv(cfg, qs[0])
    lab = synth.gen_label_channels(cfg)
    layer = runtime.offloaded_layer_for_config(cfg, K, V, lab)
    try:
        layer.step(_dev_q(qs[0]))
        layer.step(_dev_q(qs[1]))
        monkeypatch.setenv("TLS_FAULT_INJECT", "copy")
        with pytest.raises(tls.TlsError) as e:
            layer.step(_dev_q(qs[2]))
        assert e.value.status == tls.TLS_ERR_COPY
        monkeypatch.delenv("TLS_FAULT_INJECT")
        with pytest.raises(tls.TlsError) as e2:
            layer.step(_dev_q(qs[3]))
        assert e2.value.status == tls.TLS_ERR_COPY
        assert layer.steps_taken() == 2
        torch.cuda.synchronize()
        assert layer.check_device_error() == 0
    finally:
        layer.close()
    # the device still runs work after the engine is gone
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0


def test_engine_host_wait_times_out_and_sticks(monkeypatch):
    # host-side deadline: with TLS_HOST_WAIT_MS = 50, a step whose level 1 is
    # held back ~1 s (a bounded spin kernel queued on the step's stream before
    # it) returns TLS_ERR_TIMEOUT instead of blocking; later steps return the
    # same status, and the device drains and stays healthy
    runtime, tls = _rt()
    monkeypatch.setenv("TLS_HOST_WAIT_MS", "50")
    monkeypatch.setenv("TLS_ENGINE_PLANNER", "host")  # the device planner has no host wait
    cfg = ENGINE[0]
    qs = synth.gen_query_trajectory(cfg, 3)
    K, V, _ = synth.gen_kv(cfg, qs[0])
    lab = synth.gen_label_channels(cfg)
    layer = runtime.offloaded_layer_for_config(cfg, K, V, lab)
    try:
        layer.step(_dev_q(qs[0]))
        torch.cuda.synchronize()
        q1 = _dev_q(qs[1])
        torch.cuda._sleep(2_000_000_000)  # about a second of GPU clock cycles, then it ends
        with pytest.raises(tls.TlsError) as e:
            layer.step(q1)
        assert e.value.status == tls.TLS_ERR_TIMEOUT
        with pytest.raises(tls.TlsError) as e2:
            layer.step(_dev_q(qs[2]))
        assert e2.value.status == tls.TLS_ERR_TIMEOUT
        torch.cuda.synchronize()
        assert layer.check_device_error() == 0
    finally:
        layer.close()
    x = torch.ones(1024, device="cuda")
    assert float(x.sum()) == 1024.0


def test_engine_on_the_offload_workload_sampled_steps():
    # c4 (MQA, 131072 tokens, 256 slots): three steps of the trajectory, the
    # row checked against the staggered oracle each step
    runtime, tls = _rt()
    cfg = synth.get_config("c4")
    qs = synth.gen_query_trajectory(cfg, 3)
    K, V, _ = synth.gen_kv(cfg, qs[0])
    lab = synth.gen_label_channels(cfg)
    layer = runtime.offloaded_layer_for_config(cfg, K, V, lab)
    g = cfg.group
    try:
        for t, q in enumerate(qs):
            layer.step(_dev_q(q))
            torch.cuda.synchronize()
            assert layer.check_device_error() == 0
            m_prev = layer.block_idx[(t + 1) & 1].cpu().numpy()
            m_cur = layer.block_idx[t & 1].cpu().numpy()
            tok = layer.token_idx.cpu().numpy()
            out = layer.out.float().cpu().numpy()
            where = f"c4 step {t}"
            r1 = _orow(cfg, q, K, V, lab, 0, 0)
            check_selection(m_cur[0, 0], r1["agg"], cfg.K_b, where + " M_t")
            r2 = _orow(cfg, q, K, V, lab, 0, 0, block_idx=m_prev[0, 0])
            pos = np.searchsorted(r2["cand"], tok[0, 0])
            assert np.array_equal(r2["cand"][pos], tok[0, 0]), where + ": token outside M_t-1"
            check_selection(pos, r2["token_score"], cfg.k, where + " tokens")
            r3 = _orow(cfg, q, K, V, lab, 0, 0, block_idx=m_prev[0, 0], token_idx=tok[0, 0])
            check_output(out[0, 0:g], r3["out"], where + " out")
        assert layer.stats(-1).n_copied == cfg.K_b
        assert all(0 <= layer.stats(t).n_copied <= cfg.K_b for t in range(len(qs) - 1))
    finally:
        layer.close()


def test_engine_on_the_36_layer_workload_sampled_steps():
    # c5's layer shape (batch 16, 32:8 heads, 122880 tokens, K_b 96, k 3072)
    # behind the offload engine with its 2 * K_b slots per row (24576 in all):
    # three steps of the trajectory, sampled rows against the staggered oracle
    runtime, tls = _rt()
    cfg = synth.get_config("c5")
    qs = synth.gen_query_trajectory(cfg, 3)
    K, V, _ = synth.gen_kv(cfg, qs[0])
    lab = synth.gen_label_channels(cfg)
    layer = runtime.offloaded_layer_for_config(cfg, K, V, lab)
    g = cfg.group
    try:
        for t, q in enumerate(qs):
            layer.step(_dev_q(q))
            torch.cuda.synchronize()
            assert layer.check_device_error() == 0
            m_prev = layer.block_idx[(t + 1) & 1].cpu().numpy()
            m_cur = layer.block_idx[t & 1].cpu().numpy()
            tok = layer.token_idx.cpu().numpy()
            out = layer.out.float().cpu().numpy()
            for b, h in _rows(cfg, 3):
                where = f"c5 step {t} row ({b},{h})"
                r1 = _orow(cfg, q, K, V, lab, b, h)
                check_selection(m_cur[b, h], r1["agg"], cfg.K_b, where + " M_t")
                r2 = _orow(cfg, q, K, V, lab, b, h, block_idx=m_prev[b, h])
                pos = np.searchsorted(r2["cand"], tok[b, h])
                assert np.array_equal(r2["cand"][pos], tok[b, h]), where + ": token outside M_t-1"
                check_selection(pos, r2["token_score"], cfg.k, where + " tokens")
                r3 = _orow(cfg, q, K, V, lab, b, h, block_idx=m_prev[b, h], token_idx=tok[b, h])
                check_output(out[b, h * g:(h + 1) * g], r3["out"], where + " out")
        assert layer.stats(-1).n_copied == cfg.rows * cfg.K_b
        assert all(0 <= layer.stats(t).n_copied <= cfg.rows * cfg.K_b for t in range(len(qs) - 1))
        # the slot table agrees with the host mirror, and sampled slots hold their blocks
        table = layer.slot_table.cpu().numpy()
        mirror = np.empty_like(table)
        tls.tls_block_cache_table(layer.cache, mirror)
        assert np.array_equal(table, mirror)
        last = layer.block_idx[(len(qs) - 1) & 1].cpu().numpy()
        bs = cfg.block_size
        for b, h in _rows(cfg, 3):
            for blk in last[b, h][:: 17]:
                s = int(table[b, h, blk])
                got = layer.slot_k[s].view(torch.int16).cpu().numpy().view(np.uint16)
                assert s >= 0 and np.array_equal(got, K[b, h, blk * bs:(blk + 1) * bs])
    finally:
        layer.close()


# ---------------------------------------------------------------------------
# resident engine: the same stagger over HBM-resident K/V, no transfers
# ---------------------------------------------------------------------------

def _resident(cfg, qs):
    runtime, tls = _rt()
    K, V, _ = synth.gen_kv(cfg, qs[0])
    lab = synth.gen_label_channels(cfg)
    st = runtime.state_for_config(cfg, qs[0], K, V, lab)
    return runtime, st, (K, V, lab)


# more resident shapes: 8 heads a group; 512 blocks with 32 label channels and
# an odd K_b; 4096 candidates and 2048 tokens a row
RESIDENT = [
    offload("f_g8", n_q_heads=8, ctx_len=4096, block_size=32, K_b=16, k=256, seed=34, steps=4),
    offload("f_r32_two_passes", batch=4, n_q_heads=16, n_kv_heads=4, ctx_len=16384, block_size=32, K_b=23, k=300,
            n_label=32, seed=35, steps=4),
    offload("f_c2_rows", batch=2, n_q_heads=8, n_kv_heads=2, ctx_len=32768, K_b=64, k=2048, seed=36, steps=3),
]


@pytest.mark.parametrize("cfg", ENGINE + RESIDENT, ids=lambda c: c.name)
def test_resident_engine_follows_the_staggered_oracle(cfg):
    qs = synth.gen_query_trajectory(cfg)
    runtime, st, (K, V, lab) = _resident(cfg, qs)
    eng = runtime.ResidentEngine(st)
    assert eng.step_kernels() == 3 + (1 if cfg.group > 32 else 0)
    g = cfg.group
    try:
        for t, q in enumerate(qs):
            eng.step(_dev_q(q))
            torch.cuda.synchronize()
            assert eng.check_device_error() == 0
            m_prev = eng.block_idx[(t + 1) & 1].cpu().numpy()
            m_cur = eng.block_idx[t & 1].cpu().numpy()
            tok = eng.token_idx.cpu().numpy()
            out = eng.out.float().cpu().numpy()
            for b, h in _rows(cfg):
                where = f"{cfg.name} resident step {t} row ({b},{h})"
                r1 = _orow(cfg, q, K, V, lab, b, h)
                check_selection(m_cur[b, h], r1["agg"], cfg.K_b, where + " M_t")
                if t == 0:
                    check_selection(m_prev[b, h], r1["agg"], cfg.K_b, where + " M_-1")
                r2 = _orow(cfg, q, K, V, lab, b, h, block_idx=m_prev[b, h])
                pos = np.searchsorted(r2["cand"], tok[b, h])
                assert np.array_equal(r2["cand"][pos], tok[b, h]), f"{where}: token outside M_t-1"
                check_selection(pos, r2["token_score"], cfg.k, where + " tokens")
                r3 = _orow(cfg, q, K, V, lab, b, h, block_idx=m_prev[b, h], token_idx=tok[b, h])
                check_output(out[b, h * g:(h + 1) * g], r3["out"], where + " out")
        assert eng.steps_taken() == len(qs)
        st0 = runtime.tls.tls_engine_stats(eng.engine, 0)
        assert st0.n_copied == 0 and st0.bytes_copied == 0
    finally:
        eng.close()


def test_resident_engine_steps_replay_from_graphs():
    # steps 1 and 2 captured into two graphs (the two parities of the block
    # lists), then replayed alternately: every step equals the eager engine's,
    # bit for bit
    cfg = ENGINE[2]
    qs = synth.gen_query_trajectory(cfg, 6)
    runtime, st, _ = _resident(cfg, qs)
    eager = runtime.ResidentEngine(st)
    want = []
    for q in qs:
        eager.step(_dev_q(q))
        torch.cuda.synchronize()
        want.append((eager.token_idx.clone(), eager.out.clone(), eager.lse.clone()))
    eager.close()

    eng = runtime.ResidentEngine(st)
    s = torch.cuda.Stream()
    qbuf = _dev_q(qs[0]).clone()
    graphs = []
    try:
        with torch.cuda.stream(s):
            eng.step(qbuf, stream=s)  # step 0 (with the prologue) eagerly
            s.synchronize()
            assert torch.equal(eng.token_idx, want[0][0]) and torch.equal(eng.out, want[0][1])
            for _ in range(2):
                gr = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gr, stream=s):
                    eng.step(qbuf, stream=s)
                graphs.append(gr)
            for t in range(1, len(qs)):
                qbuf.copy_(_dev_q(qs[t]))
                graphs[(t - 1) & 1].replay()
                s.synchronize()
                assert torch.equal(eng.token_idx, want[t][0]), f"step {t}: token lists differ"
                assert torch.equal(eng.out, want[t][1]) and torch.equal(eng.lse, want[t][2]), f"step {t}: output"
        assert eng.check_device_error() == 0
    finally:
        del graphs
        eng.close()


def test_resident_engine_on_the_headline_workload_sampled_rows():
    # c2 (Qwen3-8B shape, 32K context) through the resident engine, the path
    # the benchmark times: level 2 on half the SMs beside level 1; three steps
    # of a q trajectory, sampled rows checked against the staggered oracle
    cfg = synth.get_config("c2")
    qs = synth.gen_query_trajectory(cfg, 3)
    runtime, st, (K, V, lab) = _resident(cfg, qs)
    eng = runtime.ResidentEngine(st)
    g = cfg.group
    try:
        for t, q in enumerate(qs):
            eng.step(_dev_q(q))
            torch.cuda.synchronize()
            assert eng.check_device_error() == 0
            m_prev = eng.block_idx[(t + 1) & 1].cpu().numpy()
            m_cur = eng.block_idx[t & 1].cpu().numpy()
            tok = eng.token_idx.cpu().numpy()
            out = eng.out.float().cpu().numpy()
            for b, h in _rows(cfg, 2):
                where = f"c2 resident step {t} row ({b},{h})"
                r1 = _orow(cfg, q, K, V, lab, b, h)
                check_selection(m_cur[b, h], r1["agg"], cfg.K_b, where + " M_t")
                r2 = _orow(cfg, q, K, V, lab, b, h, block_idx=m_prev[b, h])
                pos = np.searchsorted(r2["cand"], tok[b, h])
                assert np.array_equal(r2["cand"][pos], tok[b, h]), f"{where}: token outside M_t-1"
                check_selection(pos, r2["token_score"], cfg.k, where + " tokens")
                r3 = _orow(cfg, q, K, V, lab, b, h, block_idx=m_prev[b, h], token_idx=tok[b, h])
                check_output(out[b, h * g:(h + 1) * g], r3["out"], where + " out")
    finally:
        eng.close()


def test_prefetch_diff_records_its_done_event():
    # the plain C call: plan T_t = M_t \ C_t, queue the copies on a copy stream
    # and record the caller's event after them; work ordered after the event
    # sees every block of M_t in its slot (three rounds, the last one evicting)
    runtime, tls = _rt()
    cfg = ENGINE[2]
    q = synth.gen_queries(cfg)
    K, V, _ = synth.gen_kv(cfg, q)
    rows, nb, bs, K_b = cfg.rows, cfg.n_blocks, cfg.block_size, cfg.K_b
    n_slots = 2 * rows * K_b
    host_k = torch.from_numpy(np.ascontiguousarray(K).view(np.int16)).pin_memory()
    host_v = torch.from_numpy(np.ascontiguousarray(V).view(np.int16)).pin_memory()
    slot_k = torch.zeros((n_slots, bs, cfg.qk_dim), dtype=torch.bfloat16, device="cuda")
    slot_v = torch.zeros((n_slots, bs, cfg.v_dim), dtype=torch.bfloat16, device="cuda")
    table = torch.full((cfg.batch, cfg.n_kv_heads, nb), -1, dtype=torch.int32, device="cuda")
    shape = tls.make_shape(cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.qk_dim, cfg.v_dim, -1, bs, cfg.n_label,
                           cfg.ctx_len, cfg.softmax_scale)
    cache = tls.tls_block_cache_create(shape, host_k, host_v, cfg.qk_dim, cfg.v_dim, n_slots, slot_k, slot_v, table)
    rng = np.random.default_rng(7)
    copy_stream = torch.cuda.Stream()
    try:
        prev = None
        resident = np.zeros((cfg.batch, cfg.n_kv_heads, nb), dtype=bool)
        evicted = 0
        for rnd in range(3):
            m = np.stack([np.sort(rng.choice(nb, K_b, replace=False)) for _ in range(rows)]).astype(np.int32)
            m = m.reshape(cfg.batch, cfg.n_kv_heads, K_b)
            done = torch.cuda.Event()
            done.record(copy_stream)  # the event exists before the library records it
            n = tls.tls_prefetch_diff(cache, m, prev, K_b, copy_stream, done)
            torch.cuda.current_stream().wait_event(done)
            tab = table.cpu().numpy()  # ordered after the event on the current stream
            sk = slot_k.view(torch.int16).cpu().numpy().view(np.uint16)
            sv = slot_v.view(torch.int16).cpu().numpy().view(np.uint16)
            # |T_t| = |M_t \ C_t| summed over rows, C_t = the blocks resident before the call
            want = sum(len(oracle.plan_transfer(m[b, h], np.flatnonzero(resident[b, h])))
                       for b in range(cfg.batch) for h in range(cfg.n_kv_heads))
            assert n == want
            now = tab >= 0
            evicted += int(np.count_nonzero(resident & ~now))
            resident = now
            for b in range(cfg.batch):
                for h in range(cfg.n_kv_heads):
                    if prev is not None:
                        assert np.all(tab[b, h, prev[b, h]] >= 0), "a block of M_t-1 was evicted"
                    for blk in m[b, h]:
                        sl = tab[b, h, blk]
                        assert sl >= 0
                        assert np.array_equal(sk[sl], K[b, h, blk * bs:(blk + 1) * bs])
                        assert np.array_equal(sv[sl], V[b, h, blk * bs:(blk + 1) * bs])
            prev = m
        assert evicted > 0, "the workload lost its construction: nothing was evicted"
    finally:
        torch.cuda.synchronize()
        tls.tls_block_cache_destroy(cache)


def _cache_pair(tls, cfg, n_slots):
    # two caches over the same pinned K/V: one planned on the host, one on the device
    q = synth.gen_queries(cfg)
    K, V, _ = synth.gen_kv(cfg, q)
    bs, nb = cfg.block_size, cfg.n_blocks
    host_k = torch.from_numpy(np.ascontiguousarray(K).view(np.int16)).pin_memory()
    host_v = torch.from_numpy(np.ascontiguousarray(V).view(np.int16)).pin_memory()
    shape = tls.make_shape(cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.qk_dim, cfg.v_dim, -1, bs, cfg.n_label,
                           cfg.ctx_len, cfg.softmax_scale)
    out = []
    for _ in range(2):
        slot_k = torch.zeros((n_slots, bs, cfg.qk_dim), dtype=torch.bfloat16, device="cuda")
        slot_v = torch.zeros((n_slots, bs, cfg.v_dim), dtype=torch.bfloat16, device="cuda")
        table = torch.full((cfg.batch, cfg.n_kv_heads, nb), -1, dtype=torch.int32, device="cuda")
        cache = tls.tls_block_cache_create(shape, host_k, host_v, cfg.qk_dim, cfg.v_dim, n_slots, slot_k, slot_v,
                                           table)
        out.append((cache, slot_k, slot_v, table))
    return K, V, host_k, host_v, out


def test_device_planner_evicts_what_the_host_planner_evicts():
    # the same churning sequence of block lists through tls_prefetch_diff (host
    # plan) and tls_prefetch_diff_device (device plan): after every round both
    # caches have the same slot table (the same victims -- free slots, then
    # least recently used, then lower slot -- taken in slot order) and copied
    # as many; every resident block's slot holds its K and V rows
    runtime, tls = _rt()
    cfg = ENGINE[2]
    rows, nb, bs, K_b = cfg.rows, cfg.n_blocks, cfg.block_size, cfg.K_b
    n_slots = 2 * rows * K_b + 5
    K, V, host_k, host_v, caches = _cache_pair(tls, cfg, n_slots)
    (hc, _, _, htab), (dc, dk, dv, dtab) = caches
    rng = np.random.default_rng(11)
    stream = torch.cuda.Stream()
    n_dev = torch.zeros(1, dtype=torch.int32, device="cuda")
    try:
        prev = None
        base = np.stack([np.sort(rng.choice(nb, K_b, replace=False)) for _ in range(rows)])
        for rnd in range(12):
            # a drifting selection: a few blocks of each row change per round
            m = base.copy()
            for r in range(rows):
                keep = rng.choice(K_b, K_b - 3, replace=False)
                fresh = rng.choice(np.setdiff1d(np.arange(nb), m[r]), 3, replace=False)
                m[r] = np.sort(np.concatenate([m[r][keep], fresh]))
            base = m
            mm = m.astype(np.int32).reshape(cfg.batch, cfg.n_kv_heads, K_b)
            n_host = tls.tls_prefetch_diff(hc, mm, prev, K_b, stream)
            md = torch.from_numpy(mm).cuda()
            pd = None if prev is None else torch.from_numpy(prev).cuda()
            torch.cuda.synchronize()
            tls.tls_prefetch_diff_device(dc, md, pd, K_b, stream, None, n_dev)
            torch.cuda.synchronize()
            assert int(n_dev.item()) == n_host, f"round {rnd}: copied {int(n_dev.item())} vs {n_host}"
            th = np.empty((cfg.batch, cfg.n_kv_heads, nb), dtype=np.int32)
            td = np.empty_like(th)
            tls.tls_block_cache_table(hc, th)
            tls.tls_block_cache_table(dc, td)
            assert np.array_equal(th, td), f"round {rnd}: slot tables differ"
            used = td[td >= 0]
            assert used.size == np.unique(used).size and used.max() < n_slots
            prev = mm
        sk = dk.view(torch.int16).cpu().numpy().view(np.uint16)
        sv = dv.view(torch.int16).cpu().numpy().view(np.uint16)
        td = dtab.cpu().numpy()
        for b in range(cfg.batch):
            for h in range(cfg.n_kv_heads):
                for blk in np.flatnonzero(td[b, h] >= 0):
                    s = td[b, h, blk]
                    assert np.array_equal(sk[s], K[b, h, blk * bs:(blk + 1) * bs])
                    assert np.array_equal(sv[s], V[b, h, blk * bs:(blk + 1) * bs])
        # the host path reads the device state back and continues from it
        m = np.stack([np.sort(rng.choice(nb, K_b, replace=False)) for _ in range(rows)]).astype(np.int32)
        mm = m.reshape(cfg.batch, cfg.n_kv_heads, K_b)
        n1 = tls.tls_prefetch_diff(dc, mm, prev, K_b, stream)
        n2 = tls.tls_prefetch_diff(hc, mm, prev, K_b, stream)
        assert n1 == n2
    finally:
        for c in caches:
            tls.tls_block_cache_destroy(c[0])


def test_device_planner_failures_stick():
    # too few evictable slots, and a list that is not ascending: the plan
    # changes nothing, writes -1, and the cache refuses every later transfer
    runtime, tls = _rt()
    cfg = ENGINE[2]
    rows, nb, K_b = cfg.rows, cfg.n_blocks, cfg.K_b
    stream = torch.cuda.Stream()
    n_dev = torch.zeros(1, dtype=torch.int32, device="cuda")
    rng = np.random.default_rng(12)
    for kind in ("capacity", "order"):
        n_slots = rows * K_b + (0 if kind == "capacity" else rows * K_b)
        _, _, _, _, caches = _cache_pair(tls, cfg, n_slots)
        try:
            cache = caches[1][0]
            m = np.stack([np.sort(rng.choice(nb, K_b, replace=False)) for _ in range(rows)]).astype(np.int32)
            tls.tls_prefetch_diff_device(cache, torch.from_numpy(m).cuda(), None, K_b, stream, None, n_dev)
            torch.cuda.synchronize()
            assert int(n_dev.item()) == rows * K_b
            table0 = np.empty((cfg.batch, cfg.n_kv_heads, nb), dtype=np.int32)
            tls.tls_block_cache_table(cache, table0)
            m2 = np.stack([np.sort(rng.choice(np.setdiff1d(np.arange(nb), m[r]), K_b, replace=False))
                           for r in range(rows)]).astype(np.int32)
            if kind == "order":
                m2 = m2[:, ::-1].copy()  # descending
            tls.tls_prefetch_diff_device(cache, torch.from_numpy(m2).cuda(), torch.from_numpy(m).cuda(), K_b,
                                         stream, None, n_dev)
            torch.cuda.synchronize()
            assert int(n_dev.item()) == -1
            table1 = np.empty_like(table0)
            tls.tls_block_cache_table(cache, table1)
            assert np.array_equal(table0, table1), "a failed plan changed the table"
            want = tls.TLS_ERR_CAPACITY if kind == "capacity" else tls.TLS_ERR_INVALID_ARG
            with pytest.raises(tls.TlsError) as e:
                tls.tls_prefetch_diff_device(cache, torch.from_numpy(m).cuda(), None, K_b, stream, None, n_dev)
            assert e.value.status == want
            with pytest.raises(tls.TlsError) as e2:
                tls.tls_prefetch_diff(cache, m, None, K_b, stream)
            assert e2.value.status == want
        finally:
            for c in caches:
                tls.tls_block_cache_destroy(c[0])


def test_copy_from_host_moves_pinned_bytes():
    # the per-step input path of a serving loop: pinned host bytes into device
    # memory by one kernel (sizes from one 16-byte word to several grid
    # strides, an interior source address); memory that is not pinned is
    # refused before anything runs
    runtime, tls = _rt()
    rng = np.random.default_rng(5)
    for n in (16, 4096 + 48, 65536, (4 << 20) + 16):
        src = torch.from_numpy(rng.integers(0, 256, n + 32, dtype=np.uint8)).pin_memory()
        dst = torch.zeros(n, dtype=torch.uint8, device="cuda")
        tls.tls_copy_from_host(dst, src[16:16 + n].data_ptr(), n)
        torch.cuda.synchronize()
        assert torch.equal(dst.cpu(), src[16:16 + n]), f"{n} bytes"
    # the same buffer again: the remembered check, the same result
    tls.tls_copy_from_host(dst, src[16:16 + n].data_ptr(), n)
    torch.cuda.synchronize()
    assert torch.equal(dst.cpu(), src[16:16 + n])
    plain = np.zeros(4096, dtype=np.uint8)
    off = (-plain.ctypes.data) % 16
    with pytest.raises(tls.TlsError) as e:
        tls.tls_copy_from_host(dst, plain.ctypes.data + off, 1024)
    assert e.value.status == tls.TLS_ERR_INVALID_ARG
    torch.cuda.synchronize()
