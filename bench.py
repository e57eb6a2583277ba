"""Benchmark of the two-level sparse decode step (AsyncTLS hot path) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config c2] [--impl tls|reference]

A step is one pass of the per-step path over one batch: level-1 block
selection and level-2 token selection (tls_select, two launches) and sparse
attention (tls_sparse_decode_attn, one launch).  Inputs are seeded synthetic caches of the workload's shape,
resident in HBM before timing.  Between timed steps (untimed) a 256 MB buffer
is written and another 256 MB buffer is read, so every step starts with a cold
L2 that holds no dirty line; each step is timed with CUDA events on the
launching stream.  Multi-GPU runs are weak scaling: every rank
owns an independent batch (no collective on the data path); the reported
time is the max over ranks.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle on
the host cores instead (the only reference arm this method has).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse decode-attn µs/step, achieved HBM GB/s vs peak; decode tokens/s"
FLUSH_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", default="c2")
    ap.add_argument("--impl", default="tls", choices=["tls", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="budget of the CPU-oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-offload", action="store_true", help="skip the offload-engine measurement (c4)")
    ap.add_argument("--no-other-configs", action="store_true", help="skip the c1 / c3 step measurements")
    ap.add_argument("--no-c5", action="store_true", help="skip the c5 per-layer measurements")
    ap.add_argument("--no-baselines", action="store_true",
                    help="skip the operator baselines (full attention, block or token selection alone)")
    ap.add_argument("--no-staggered", action="store_true",
                    help="time the synchronous step (tls_decode_step) as the headline instead of the staggered one")
    ap.add_argument("--e2e-steps", type=int, default=300)
    return ap.parse_args()


# ----------------------------------------------------------------------------- workload

def workload(cfg, rank):
    import synth
    c = cfg.scaled(seed=cfg.seed + 1000 * rank) if rank else cfg
    q = synth.gen_queries(c)
    K, V, _ = synth.gen_kv(c, q)
    lab = synth.gen_label_channels(c)
    return c, q, K, V, lab


def max_over_ranks(values, world, device=None):
    """Each timing (ms) as the slowest rank saw it: the job's step time is set
    by its last rank.  One all-reduce (MAX) over the process group."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def job_tokens_per_s(world, batch, ms_per_step):
    """Whole-job decode tokens/s: every rank decodes its own batch of `batch` rows per step."""
    return world * batch / (ms_per_step / 1e3)


def algorithmic_bytes(cfg):
    """Bytes the step must move: metadata, candidate label codes+scales,
    gathered K/V rows, queries, index lists and the fp32 output."""
    rows = cfg.rows
    meta = rows * cfg.n_blocks * 2 * cfg.qk_dim * 2
    n_cand = cfg.K_b * cfg.block_size
    label = rows * n_cand * (cfg.n_label // 2 + 4)
    row_bytes = (cfg.qk_dim + (cfg.v_dim if cfg.separate_v else 0)) * 2
    gather = rows * cfg.k * row_bytes
    q = cfg.batch * cfg.n_q_heads * cfg.qk_dim * 2
    out = cfg.batch * cfg.n_q_heads * cfg.v_dim * 4
    idx = rows * (cfg.K_b + cfg.k) * 4 * 2
    attn = gather + q + out + rows * cfg.k * 4
    return dict(meta=meta, label=label, gather=gather, q=q, out=out, idx=idx,
                step=meta + label + gather + q + out + idx, attn=attn)


def launches_per_step(cfg):
    """Kernels one step launches: level 1 (block scores + top-K_b), level 2
    (token scores + top-k) and the attention kernel, plus the query-prep
    kernel of level 1 for groups padded to 64 heads or more."""
    g = cfg.n_q_heads // cfg.n_kv_heads
    return 3 + (1 if g > 32 else 0)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# Sources compiled into each attention kernel: a recorded ncu traffic figure
# holds only while all of them are unchanged.
ATTN_SOURCES = {
    "sparse_attn_mma_kernel": ("decode_attn_mma.cu", "mma_attn.cuh", "attn_common.cuh", "device_common.cuh"),
    "sparse_attn_mma_cluster_kernel": ("decode_attn_mma.cu", "mma_attn.cuh", "attn_common.cuh", "device_common.cuh"),
    "sparse_attn_mla_kernel": ("decode_attn_mla.cu", "attn_common.cuh", "device_common.cuh"),
    "sparse_attn_kernel": ("decode_attn.cu", "attn_common.cuh", "device_common.cuh"),
}


def kernel_source_hash(files):
    h = hashlib.sha256()
    for name in files:
        h.update(open(os.path.join(ROOT, "two_level_sparse_block_b200", "csrc", name), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload_name):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current source of the kernel; otherwise None."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kernel, {}).get(workload_name)
    if not e or e.get("source_sha256_16") != kernel_source_hash(ATTN_SOURCES[kernel]):
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 10:
                continue
            if self.uuid and self.uuid not in f[1]:
                continue
            try:
                rows.append((float(f[2]), float(f[3]), f[6:10]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, fl in rows for i, v in enumerate(fl) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- CPU oracle arm

def _oracle_rows(args):
    """Worker of the oracle timing: decode_row over its rows until `seconds`
    have passed; returns (rows done, seconds).  Rows are (q of the group, K,
    V, label channels, meta, label cache), or (b, kvh) pairs that the worker
    regenerates from the seeded generator first (untimed)."""
    rows, cfg_fields, seconds = args
    import oracle
    import synth
    cfg = synth.WorkloadConfig(**cfg_fields)
    g = cfg.group
    if rows and len(rows[0]) == 2:
        q = synth.gen_queries(cfg)
        lab_all = synth.gen_label_channels(cfg)
        made = []
        for b, h in rows:
            r = synth.gen_row(cfg, b, h, q)
            made.append((q[b, h * g:(h + 1) * g], r.k, r.v, lab_all[h], oracle.block_meta(r.k, cfg.block_size),
                         oracle.quant_label(r.k, lab_all[h])))
        rows = made
    done = 0
    t0 = time.perf_counter()
    while True:
        qg, kb, vb, lab, meta, label = rows[done % len(rows)]
        oracle.decode_row(qg, kb, vb, lab, cfg.block_size, cfg.K_b, cfg.k, cfg.softmax_scale,
                          v_offset=cfg.v_offset, v_dim=cfg.v_dim, meta=meta, label=label)
        done += 1
        el = time.perf_counter() - t0
        if el >= seconds and done >= len(rows):
            return done, el


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def time_oracle(cfg, q, K, V, lab, seconds, rows_sample=8, all_cores=True):
    """Times the float64 oracle's per-step path (levels 1, 2 and attention;
    the index build is prepared outside the timed region, as on the GPU):
    single-threaded, and (all_cores) with one single-threaded process per host
    core working on the sampled rows at once (a spawn pool, so no CUDA state is
    forked)."""
    import dataclasses
    import oracle
    try:
        import threadpoolctl
        limiter = threadpoolctl.threadpool_limits(1)
    except Exception:
        limiter = None
    rng = np.random.default_rng(0)
    all_rows = [(b, h) for b in range(cfg.batch) for h in range(cfg.n_kv_heads)]
    pick = [all_rows[i] for i in sorted(rng.choice(len(all_rows), min(rows_sample, len(all_rows)), replace=False))]
    g = cfg.group
    prepared = []
    for b, h in pick:
        kb = K[b, h]
        prepared.append((q[b, h * g:(h + 1) * g], kb, None if V is None else V[b, h], lab[h],
                         oracle.block_meta(kb, cfg.block_size), oracle.quant_label(kb, lab[h])))
    fields = dataclasses.asdict(cfg)
    done, el = _oracle_rows((prepared, fields, seconds))
    if limiter is not None:
        limiter.unregister()
    per_row = el / done
    step_s = per_row * cfg.rows
    res = {"value": cfg.batch / step_s, "unit": "decode tokens/s", "cores": 1, "kind": "oracle",
           "sample": f"{done} (batch row, KV head) decode_row calls over {len(pick)} seeded rows of "
                     f"{cfg.name} in {el:.1f} s; scaled to all {cfg.rows} rows of one step",
           "s_per_step": step_s, "nproc": os.cpu_count(), "cpu_model": cpu_model()}
    if all_cores and (os.cpu_count() or 1) > 1:
        import multiprocessing as mp
        n = min(os.cpu_count(), 64)
        saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        for k in saved:
            os.environ[k] = "1"
        try:
            ctx = mp.get_context("spawn")
            with ctx.Pool(n) as pool:
                # each worker regenerates two of the sampled rows (the arrays are too large to ship)
                work = [([pick[(2 * i + j) % len(pick)] for j in range(2)], fields, seconds) for i in range(n)]
                t0 = time.perf_counter()
                outs = pool.map(_oracle_rows, work)
                wall = time.perf_counter() - t0
        finally:
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        rows_done = sum(d for d, _ in outs)
        span = max(e for _, e in outs)
        step_all = span / rows_done * cfg.rows
        res["all_cores"] = {"value": cfg.batch / step_all, "unit": "decode tokens/s", "cores": n,
                            "sample": f"{n} single-threaded processes (of {os.cpu_count()} host threads), each "
                                      f"decoding two of the sampled rows for {seconds:.0f} s ({rows_done} "
                                      f"decode_row calls, {wall:.1f} s wall with regeneration); scaled to all "
                                      f"{cfg.rows} rows of one step"}
    return res


def time_step_graph(st, dev, steps=200, warmup=10):
    """tls_decode_step of a DecodeState replayed from a CUDA graph, L2 flushed
    (write + read of 256 MB) before each step, CUDA events around each replay.
    Returns the per-step times in ms."""
    import torch
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    cap = torch.cuda.Stream(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        st.step(stream=cap)
        with torch.cuda.graph(g, stream=cap):
            st.step(stream=cap)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    times = []
    for i in range(warmup + steps):
        flush.fill_(float(i))
        torch.sum(flush_rd, dim=0, out=sink)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        if i >= warmup:
            times.append((a, b))
    torch.cuda.synchronize(dev)
    if st.check_device_error() != 0:
        raise RuntimeError("device error in a timed step")
    del g
    return [x.elapsed_time(y) for x, y in times]


def time_staggered_graphs(st, dev, steps=200, warmup=10):
    """The resident engine's staggered step over a DecodeState, captured into
    two graphs (the block-list parities) and replayed alternately, L2 flushed
    before each step, CUDA events around each replay.  Per-step times in ms."""
    import torch
    from two_level_sparse_block_b200 import runtime
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    eng = runtime.ResidentEngine(st)
    cap = torch.cuda.Stream(dev)
    graphs = [torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()]
    with torch.cuda.stream(cap):
        eng.step(stream=cap)
        for g in graphs:
            with torch.cuda.graph(g, stream=cap):
                eng.step(stream=cap)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    times = []
    for i in range(warmup + steps):
        flush.fill_(float(i))
        torch.sum(flush_rd, dim=0, out=sink)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        graphs[i & 1].replay()
        b.record(stream)
        if i >= warmup:
            times.append((a, b))
    torch.cuda.synchronize(dev)
    err = eng.check_device_error()
    del graphs
    eng.close()
    if err != 0:
        raise RuntimeError("device error in a staggered step")
    return [x.elapsed_time(y) for x, y in times]


def time_graph(fn, dev, steps=100, warmup=5):
    """Mean ms of fn() captured into a CUDA graph and replayed, L2 flushed
    (write + read of 256 MB) before each replay, CUDA events around it."""
    import torch
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)
    cap = torch.cuda.Stream(dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(cap):
        fn(cap)
        with torch.cuda.graph(g, stream=cap):
            fn(cap)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    times = []
    for i in range(warmup + steps):
        flush.fill_(float(i))
        torch.sum(flush_rd, dim=0, out=sink)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        if i >= warmup:
            times.append((a, b))
    torch.cuda.synchronize(dev)
    del g
    return statistics.mean(x.elapsed_time(y) for x, y in times)


def measure_baselines(st, cfg, dev, staggered_us=None, steps=100):
    """The operator comparison of the pages (English summary 4, Efficiency) on
    this GPU: the two-level step against full attention (every token), block
    selection alone (Quest: every token of the K_b blocks) and token selection
    alone (Double Sparsity: the top-k over every token), each one graph replay
    with a cold L2, same inputs."""
    two = 1e3 * time_graph(lambda s: st.step(stream=s), dev, steps)
    full = 1e3 * time_graph(lambda s: st.dense(stream=s), dev, steps)
    quest = 1e3 * time_graph(lambda s: st.quest(stream=s), dev, steps)
    ds = 1e3 * time_graph(lambda s: st.ds(stream=s), dev, steps)
    if st.check_device_error() != 0:
        raise RuntimeError("device error in the baselines")
    best = min(two, staggered_us) if staggered_us else two
    return {"workload": cfg.name, "two_level_us": two, "two_level_staggered_us": staggered_us,
            "full_attention_us": full, "quest_only_us": quest, "ds_only_us": ds,
            "speedup_vs_full": full / best, "speedup_vs_ds": ds / best, "speedup_vs_quest": quest / best,
            "budgets": {"two_level": f"K_b {cfg.K_b}, k {cfg.k}", "quest_only": f"K_b {cfg.K_b} (all {cfg.K_b * cfg.block_size} tokens of them)",
                        "ds_only": f"k {cfg.k} of all {cfg.ctx_len} tokens", "full": f"all {cfg.ctx_len} tokens"},
            "speedups_use": "the faster of the synchronous and the staggered two-level step",
            "pages": "operator speedups quoted for context (GPU unstated): GQA 1.2-4.0x vs Double Sparsity and "
                     "1.7-6.2x vs full attention; MLA 1.9-4.0x and 3.3-10.0x (English summary 4)",
            "timing": "each path one CUDA graph, L2 flushed before every replay, mean of CUDA-event times"}


def measure_config(name, dev, steps=200, warmup=10):
    """One more workload measured like the headline (time_step_graph)."""
    import synth
    from two_level_sparse_block_b200 import runtime, tls
    c = synth.get_config(name)
    q = synth.gen_queries(c)
    K, V, _ = synth.gen_kv(c, q)
    lab = synth.gen_label_channels(c)
    st = runtime.state_for_config(c, q, K, V, lab, device=dev)
    del K, V
    tss = time_staggered_graphs(st, dev, steps, warmup)
    ts = time_step_graph(st, dev, steps, warmup)
    ms = statistics.mean(tss)  # (event ticks are coarse: the mean, not the median, averages them out)
    ab = algorithmic_bytes(c)
    base = measure_baselines(st, c, dev, ms * 1e3) if name == "c3" else None
    return {"us_per_step": ms * 1e3, "us_per_step_median": statistics.median(tss) * 1e3,
            "baselines": base,
            "decode_tokens_per_s": c.batch / (ms / 1e3),
            "algorithmic_bytes": ab["step"], "achieved_gbs": ab["step"] / (ms / 1e3) / 1e9,
            "synchronous_us_per_step": statistics.mean(ts) * 1e3,
            "attention_kernel": tls.tls_attn_kernel(st.shape), "steps": steps,
            "schedule": "staggered step (resident engine), as the headline; synchronous_us_per_step: "
                        "tls_decode_step",
            "l2": "flushed before every step (write + read of 256 MB)"}


def pcie_h2d_peak(dev, nbytes=256 << 20, reps=5):
    """Host -> device bandwidth of one large copy from pinned memory (best of
    reps, CUDA events): the copy engines' ceiling the block transfers are
    compared against."""
    import torch
    src = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dst = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    best = None
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        dst.copy_(src, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms = a.elapsed_time(b)
        best = ms if best is None else min(best, ms)
    return nbytes / (best / 1e3) / 1e9


def measure_offload_engine(dev, steps=64, name="c4", data=None):
    """An offload workload (c4 by default): the staggered engine over an HBM
    block cache (2 K_b slots a row unless the workload names a count), K/V in
    pinned host memory, `steps` consecutive decode steps along the seeded query
    trajectory.  Steps run back to back (no L2 flush, nothing between them),
    which leaves the copies the least time to hide.  data: (q trajectory, K, V,
    label channels) already generated, or None."""
    import synth
    import torch
    from two_level_sparse_block_b200 import runtime
    cfg = synth.get_config(name)
    if data is None:
        qs = synth.gen_query_trajectory(cfg, steps)
        K, V, _ = synth.gen_kv(cfg, qs[0])
        lab = synth.gen_label_channels(cfg)
    else:
        qs, K, V, lab = data
    qd = [torch.from_numpy(np.ascontiguousarray(q).view(np.int16)).to(dev).view(torch.bfloat16) for q in qs]
    stream = torch.cuda.current_stream(dev)
    # the same layer and q trajectory with its K/V resident in HBM (the
    # resident engine: the same stagger, no transfer), issued the same way: the
    # step time the transfers would add to if they were not hidden
    st = runtime.state_for_config(cfg, qs[0], K, V, lab, device=dev)
    eng = runtime.ResidentEngine(st)
    try:
        r_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize(dev)
        for t in range(steps):
            r_evs[t][0].record(stream)
            eng.step(q=qd[t], stream=stream)
            r_evs[t][1].record(stream)
        torch.cuda.synchronize(dev)
        resident_ms = [a.elapsed_time(b) for a, b in r_evs][1:]
    finally:
        eng.close()
        del st
        torch.cuda.empty_cache()
    layer = runtime.offloaded_layer_for_config(cfg, K, V, lab)
    del K, V
    try:
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize(dev)
        host_s = []
        for t in range(steps):
            evs[t][0].record(stream)
            h0 = time.perf_counter()
            layer.step(qd[t], stream=stream)
            host_s.append(time.perf_counter() - h0)
            evs[t][1].record(stream)
        torch.cuda.synchronize(dev)
        if layer.check_device_error() != 0:
            raise RuntimeError("device error in the offload engine")
        step_ms = [a.elapsed_time(b) for a, b in evs]
        st = [layer.stats(t) for t in range(steps - 1)]  # the transfer of step t, awaited by step t + 1
        copy_ms = sum(x.copy_ms for x in st)
        exposed_ms = sum(x.exposed_ms for x in st)
        moved = sum(x.bytes_copied for x in st)
        blocks = [x.n_copied for x in st]
        prologue = layer.stats(-1)
    finally:
        layer.close()
    steady = step_ms[1:]
    peak = pcie_h2d_peak(dev)
    copy_us = 1e3 * copy_ms / len(st)
    added_us = max(0.0, 1e3 * (statistics.mean(steady) - statistics.mean(resident_ms)))
    h2d = moved / (copy_ms / 1e3) / 1e9 if copy_ms > 0 else None
    return {
        "workload": cfg.name, "steps": steps, "n_slots": (cfg.n_slots or 2 * cfg.K_b) * cfg.rows, "K_b": cfg.K_b,
        "resident_us_per_step_mean": 1e3 * statistics.mean(resident_ms),
        "added_us_per_step_vs_resident": added_us,
        "hidden_frac_vs_resident": (1.0 - min(1.0, added_us / copy_us)) if copy_us > 0 else None,
        "pcie_peak_gbs": peak, "h2d_frac_of_pcie_peak": (h2d / peak) if h2d else None,
        "us_per_step_median": 1e3 * statistics.median(steady), "us_per_step_mean": 1e3 * statistics.mean(steady),
        "us_first_step": 1e3 * step_ms[0], "prologue_blocks": prologue.n_copied,
        "host_us_per_step_median": 1e6 * statistics.median(host_s[1:]),
        "transfer_blocks_per_step_mean": statistics.mean(blocks),
        "transfer_frac_of_K_b_mean": statistics.mean(blocks) / (cfg.K_b * cfg.rows),
        "h2d_gbs": h2d,
        "copy_us_per_step_mean": copy_us, "exposed_us_per_step_mean": 1e3 * exposed_ms / len(st),
        "copy_hidden_frac": 1.0 - exposed_ms / copy_ms if copy_ms > 0 else None, "target_hidden_frac": 0.9,
        "planner": "device (tls_prefetch_diff_device on the copy stream: the step call never waits on the host)",
        "timing": "per step: CUDA events on the caller's stream around tls_engine_step (level 2 + wait for the "
                  "previous transfer + attention; level 1 runs on the engine's second stream), so the step time "
                  "is the device's, and host_us_per_step the call's own time; transfer figures "
                  "from the engine's copy-stream events.  copy_hidden_frac counts the time the attention waited "
                  "on a transfer past its own readiness; hidden_frac_vs_resident compares the step with the same "
                  "layer and q trajectory over HBM-resident K/V (resident engine, no transfer): 1 - (step time "
                  "added by offloading) / (copy-stream time)",
    }


def measure_c5(dev, steps_resident=50, steps_offload=24, n_resident=20):
    """The 36-layer workload (c5), one layer of it measured two ways: resident in
    HBM (time_step_graph) and offloaded to pinned host memory behind the
    staggered engine (measure_offload_engine, 2 K_b slots a row).  Each layer's
    KV is 8 GB, so the 36 layers (290 GB) cannot all be resident: the step is
    reported as n_resident resident layers plus the rest offloaded, each layer
    at its measured time (layers run one after another and share nothing)."""
    import synth
    from two_level_sparse_block_b200 import runtime
    c = synth.get_config("c5")
    qs = synth.gen_query_trajectory(c, steps_offload)
    K, V, _ = synth.gen_kv(c, qs[0])
    lab = synth.gen_label_channels(c)
    st = runtime.state_for_config(c, qs[0], K, V, lab, device=dev)
    ts = time_step_graph(st, dev, steps_resident, 5)
    del st
    import torch
    torch.cuda.empty_cache()
    off = measure_offload_engine(dev, steps_offload, "c5", (qs, K, V, lab))
    res_us = statistics.mean(ts) * 1e3
    off_us = off["us_per_step_mean"]
    n_layers = 36
    step_us = n_resident * res_us + (n_layers - n_resident) * off_us
    ab = algorithmic_bytes(c)
    return {"layers": n_layers, "layer_kv_bytes": 2 * c.rows * c.ctx_len * c.qk_dim * 2,
            "resident_layer_us": res_us, "resident_layer_achieved_gbs": ab["step"] / (res_us / 1e6) / 1e9,
            "offloaded_layer": off, "n_resident_layers": n_resident,
            "step_us_composed": step_us, "decode_tokens_per_s_composed": c.batch / (step_us / 1e6),
            "composition": f"{n_resident} layers resident in HBM (each layer's 8 GB KV plus index; about 20 fit "
                           f"in 180 GB) + {n_layers - n_resident} offloaded, each at its measured per-layer time"}


def measure_c5_loop(dev, steps=6, n_resident=20, n_layers=36):
    """The 36-layer workload (c5) as one decode loop: per step, n_resident
    layers with their KV in HBM (resident staggered engines) and the rest
    offloaded to pinned host memory behind their own block caches (offload
    engines), layer after layer on one stream, each layer with its own q
    trajectory.  Every layer decodes the same seeded 8 GB KV (one HBM copy for
    the resident layers, one pinned host copy for the offloaded ones, one
    index), since 36 distinct copies (290 GB) fit neither memory; each layer
    keeps its own block lists, token lists, slot pool and transfers.  Every
    layer reads more than L2 holds, so consecutive layers share no cached
    lines.  CUDA events around each whole decode step."""
    import synth
    import torch
    from two_level_sparse_block_b200 import runtime
    c = synth.get_config("c5")
    qs = [synth.gen_query_trajectory(c, steps, layer=l) for l in range(n_layers)]
    K, V, _ = synth.gen_kv(c, qs[0][0])
    lab = synth.gen_label_channels(c)
    st = runtime.state_for_config(c, qs[0][0], K, V, lab, device=dev)
    resident = [runtime.ResidentEngine(st) for _ in range(n_resident)]
    first = runtime.offloaded_layer_for_config(c, K, V, lab)
    del K, V
    offloaded = [first] + [runtime.offloaded_layer_for_config(c, None, None, lab, share_from=first)
                           for _ in range(n_layers - n_resident - 1)]
    try:
        qd = [[torch.from_numpy(np.ascontiguousarray(q).view(np.int16)).to(dev).view(torch.bfloat16) for q in ql]
              for ql in qs]
        stream = torch.cuda.current_stream(dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize(dev)
        for t in range(steps):
            evs[t][0].record(stream)
            for l in range(n_layers):
                if l < n_resident:
                    resident[l].step(q=qd[l][t], stream=stream)
                else:
                    offloaded[l - n_resident].step(qd[l][t], stream=stream)
            evs[t][1].record(stream)
        torch.cuda.synchronize(dev)
        if any(e.check_device_error() != 0 for e in resident) or any(o.check_device_error() != 0 for o in offloaded):
            raise RuntimeError("device error in the 36-layer loop")
        step_ms = [a.elapsed_time(b) for a, b in evs]
        moved = [sum(o.stats(t).bytes_copied for o in offloaded) for t in range(steps - 1)]
        blocks = [sum(o.stats(t).n_copied for o in offloaded) for t in range(steps - 1)]
    finally:
        for e in resident:
            e.close()
        for o in offloaded:
            o.close()
    steady = step_ms[1:]  # the first step also makes every offloaded layer's M_{-1} resident
    ms = statistics.mean(steady)
    return {"layers": n_layers, "n_resident_layers": n_resident, "steps": steps,
            "ms_per_step_mean": ms, "decode_tokens_per_s": c.batch / (ms / 1e3),
            "ms_first_step": step_ms[0], "h2d_bytes_per_step_mean": statistics.mean(moved),
            "transfer_blocks_per_step_mean": statistics.mean(blocks),
            "h2d_gbs_needed": statistics.mean(moved) / (ms / 1e3) / 1e9,
            "timing": "CUDA events around each decode step (36 layer steps issued back to back on one stream; "
                      "each offloaded layer's transfer is planned on the device, so no call waits on the host)"}


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    cfg, q, K, V, lab = workload(cfg, 0)
    per_step = max(0.5, args.cpu_seconds / max(1, args.steps))
    for _ in range(args.warmup):
        time_oracle(cfg, q, K, V, lab, 0.0, rows_sample=1, all_cores=False)
    t = []
    res = None
    for _ in range(args.steps):
        res = time_oracle(cfg, q, K, V, lab, per_step, rows_sample=2, all_cores=False)
        t.append(res["s_per_step"])
    step_s = statistics.mean(t)
    value = cfg.batch / step_s
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "decode tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": cfg.name, "batch": cfg.batch, "ctx_len": cfg.ctx_len, "K_b": cfg.K_b, "k": cfg.k},
            "cpu_baseline": {"value": value, "unit": "decode tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"each step: {res['sample']}"},
            "e2e": {"value": value, "unit": "decode tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm

def main():
    args = parse()
    import synth
    cfg = synth.get_config(args.config)
    if args.impl == "reference":
        run_reference(args, cfg)
        return

    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    from two_level_sparse_block_b200 import build, runtime, tls
    build.build()

    c, q, K, V, lab = workload(cfg, rank)
    st = runtime.state_for_config(c, q, K, V, lab, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2(i):
        # write 256 MB (evicts every line of the step), then read another 256 MB
        # so the dirty lines of the write are written back before the step starts
        flush.fill_(float(i))
        torch.sum(flush_rd, dim=0, out=sink)
    torch.cuda.synchronize(dev)

    # The timed step is the hot path as the method schedules it: the resident
    # staggered engine (tls_engine_create_resident / tls_engine_step), where
    # step t runs level 2 and the attention within the blocks chosen at step
    # t-1 while level 1 chooses M_t for q_t beside them.  Its steps are
    # captured into two CUDA graphs (the two parities of its block lists) and
    # replayed alternately, so the timed loop spends no host time per kernel
    # and the events measure the GPU alone.  The synchronous step
    # (tls_decode_step: levels 1, 2 and the attention in order) is captured
    # too and timed beside it, and two more graphs hold tls_select and
    # tls_sparse_decode_attn for the per-stage times (the attention alone, K
    # and V read from HBM).
    eng = runtime.ResidentEngine(st)
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    g_step, g_sel, g_att = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    g_stag = [torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()]
    with torch.cuda.stream(cap):
        st.step(stream=cap)
        st.select(stream=cap)
        st.attend(stream=cap)
        eng.step(stream=cap)  # step 0 with its prologue (M_{-1} from q_0)
        with torch.cuda.graph(g_step, stream=cap):
            st.step(stream=cap)
        with torch.cuda.graph(g_sel, stream=cap):
            st.select(stream=cap)
        with torch.cuda.graph(g_att, stream=cap):
            st.attend(stream=cap)
        for g in g_stag:
            with torch.cuda.graph(g, stream=cap):
                eng.step(stream=cap)
    stream.wait_stream(cap)
    torch.cuda.synchronize(dev)

    def step_events(n):
        return [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]

    def timed_steps(n, evs, synchronous=False):
        for i in range(n):
            flush_l2(i)
            e = evs[i]
            e[0].record(stream)
            if synchronous:
                g_step.replay()
            else:
                g_stag[i & 1].replay()
            e[1].record(stream)

    def stage_times(n):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n)]
        for i in range(n):
            flush_l2(i)
            evs[i][0].record(stream)
            g_sel.replay()
            evs[i][1].record(stream)
            g_att.replay()
            evs[i][2].record(stream)
        torch.cuda.synchronize(dev)
        return ([e[0].elapsed_time(e[1]) for e in evs], [e[1].elapsed_time(e[2]) for e in evs])

    sync_headline = args.no_staggered
    warm = step_events(args.warmup)
    timed_steps(args.warmup, warm)
    timed_steps(args.warmup, warm, synchronous=True)
    torch.cuda.synchronize(dev)
    if st.check_device_error() != 0 or eng.check_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    evs = step_events(args.steps)
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    sampler.start()
    time.sleep(0.3)
    wall0 = time.perf_counter()
    timed_steps(args.steps, evs, synchronous=sync_headline)
    torch.cuda.synchronize(dev)
    wall = time.perf_counter() - wall0
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    err = st.check_device_error() if sync_headline else eng.check_device_error()
    if err != 0:
        raise RuntimeError(f"device error {err} during the timed steps")

    step_ms = [e[0].elapsed_time(e[1]) for e in evs]
    # the synchronous step, timed the same way (untimed by the headline)
    n_sync = min(args.steps, 500)
    sync_evs = step_events(n_sync)
    timed_steps(n_sync, sync_evs, synchronous=True)
    torch.cuda.synchronize(dev)
    if st.check_device_error() != 0:
        raise RuntimeError("device error in the synchronous steps")
    sync_ms = [e[0].elapsed_time(e[1]) for e in sync_evs]
    # stage breakdown (separate graphs, so each stage also pays its own launch)
    sel_ms, att_ms = stage_times(n_sync)
    total_ms, att_mean_ms, sync_mean_ms = max_over_ranks(
        [sum(step_ms), statistics.mean(att_ms), statistics.mean(sync_ms)], world, dev)
    ms_per_step = total_ms / args.steps
    value = job_tokens_per_s(world, c.batch, ms_per_step)

    # end to end through the public API: pinned host q in, host out back, every
    # step.  As a serving loop runs it: q brought in from pinned host memory by
    # tls_copy_from_host (one kernel whose loads cross PCIe), the engine step,
    # and a device -> host copy of the output, captured together into graphs
    # (one per block-list parity) and replayed; for reference, the same calls
    # issued eagerly every step, and the graphs with q brought in by a
    # host -> device copy instead.
    q_host = torch.empty(st.q.shape, dtype=torch.bfloat16).pin_memory()
    q_host.copy_(st.q.cpu())
    out_host = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()
    q_dev = torch.empty_like(st.q)

    def e2e_step(s, copy_back):
        if copy_back:
            q_dev.copy_(q_host, non_blocking=True)
        else:
            tls.tls_copy_from_host(q_dev, q_host, None, s)
        eng.step(q=q_dev, stream=s)
        out_host.copy_(eng.out, non_blocking=True)

    e2e_step(stream, False)  # checks the pinned source once, outside the captures
    torch.cuda.synchronize(dev)
    graphs = {}
    cap.wait_stream(stream)
    with torch.cuda.stream(cap):
        for copy_back in (False, True):
            graphs[copy_back] = [torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()]
            for g in graphs[copy_back]:
                with torch.cuda.graph(g, stream=cap):
                    e2e_step(cap, copy_back)
    stream.wait_stream(cap)
    torch.cuda.synchronize(dev)

    def e2e_times(n, eager, copy_back=False):
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
        for i in range(n):
            flush_l2(i)
            evs[i][0].record(stream)
            if eager:
                e2e_step(stream, copy_back)
            else:
                graphs[copy_back][i & 1].replay()
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        return sum(e[0].elapsed_time(e[1]) for e in evs) / n

    e2e_ms = e2e_times(args.e2e_steps, eager=False)
    e2e_eager_ms = e2e_times(args.e2e_steps, eager=True)
    e2e_copy_ms = e2e_times(args.e2e_steps, eager=False, copy_back=True)
    if eng.check_device_error() != 0:
        raise RuntimeError("device error in the end-to-end steps")
    # the two ways of bringing q in give the same output (the same q every
    # step, so every steady step has the same output); reported, not fatal
    e2e_times(1, eager=True, copy_back=False)
    kernel_q_out = out_host.clone()
    e2e_times(1, eager=True, copy_back=True)
    e2e_same = bool(torch.equal(kernel_q_out, out_host))
    e2e_ms, e2e_eager_ms, e2e_copy_ms = max_over_ranks([e2e_ms, e2e_eager_ms, e2e_copy_ms], world, dev)
    del graphs

    ab = algorithmic_bytes(c)
    attn_kernel = tls.tls_attn_kernel(st.shape)
    peak, peak_kind = load_peaks()
    att_avg_s = att_mean_ms / 1e3
    achieved = ab["attn"] / att_avg_s / 1e9
    step_gbs = ab["step"] / (ms_per_step / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "decode tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "us_per_step": ms_per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, fp32 accumulate",
        "data": "synthetic (seeded; shapes of the workload, random K/V with outlier channels and planted tokens)",
        "config": {"workload": c.name, "batch_per_gpu": c.batch, "q_heads": c.n_q_heads, "kv_heads": c.n_kv_heads,
                   "head_dim": c.qk_dim, "ctx_len": c.ctx_len, "block_size": c.block_size, "K_b": c.K_b,
                   "k": c.k, "label_channels": c.n_label, "parallelism": f"weak x{world} (independent batches)",
                   "l2": "between timed steps (untimed): write a 256 MB buffer, then read another 256 MB buffer; "
                         "every step starts with none of its lines in L2 and no dirty line to write back"},
        "schedule": ("synchronous step (tls_decode_step), one graph" if sync_headline else
                     "the method's staggered step (tls_engine_step on a resident engine): level 2 and the "
                     "attention within the blocks chosen at step t-1, level 1 for q_t beside them on a second "
                     "stream; two graphs (block-list parities) replayed alternately"),
        "synchronous_step": {"us_per_step": sync_mean_ms * 1e3,
                             "decode_tokens_per_s": job_tokens_per_s(world, c.batch, sync_mean_ms), "steps": n_sync,
                             "path": "tls_decode_step (levels 1, 2 and the attention in order), one graph"},
        "stage_us": {"select (levels 1+2)": 1e3 * statistics.mean(sel_ms),
                     "sparse_decode_attn": 1e3 * statistics.mean(att_ms),
                     "note": "tls_select and tls_sparse_decode_attn replayed as separate graphs (each pays its own "
                             "launch, the attention reads K and V from HBM)"},
        "step_hbm": {"algorithmic_bytes": ab["step"], "achieved_gbs": step_gbs, "frac_of_peak": step_gbs / peak},
        "roofline": {"kernel": attn_kernel, "bound": "hbm", "achieved": achieved,
                     "peak": peak, "peak_source": f"hbm_gbs {peak_kind}", "unit": "GB/s", "frac": achieved / peak,
                     "algorithmic_bytes_per_launch": ab["attn"],
                     "traffic": recorded_traffic(attn_kernel, c.name)},
        "gpu_launches": launches_per_step(c) * args.steps,
        "e2e": {"value": job_tokens_per_s(world, c.batch, e2e_ms), "unit": "decode tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": int(st.q.numel() * 2), "d2h_bytes_per_step": int(st.out.numel() * st.out.element_size()),
                "path": "tls_copy_from_host (q from pinned host memory, one kernel whose loads cross PCIe), "
                        "tls_engine_step (resident engine) and a device -> host copy of the output via the Python "
                        "binding every step, the three captured together in graphs (one per block-list parity) "
                        "and replayed",
                "eager_ms_per_step": e2e_eager_ms,
                "eager_path": "the same calls issued from Python every step, no graph",
                "copy_back_ms_per_step": e2e_copy_ms,
                "copy_back_path": "the same graphs with q brought in by a host -> device copy",
                "outputs_equal": e2e_same},
        "clocks": clocks,
        "wall_s_timed": wall,
    }
    if rank == 0 and world == 1 and not args.no_baselines:
        line["baselines"] = measure_baselines(st, c, dev, ms_per_step * 1e3)
    if rank == 0 and world == 1 and not args.no_offload:
        line["offload_engine"] = measure_offload_engine(dev)
    if rank == 0 and world == 1 and not args.no_c5:
        line["c5_layers"] = measure_c5(dev)
        line["c5_layers"]["loop_36_layers"] = measure_c5_loop(dev)
    if rank == 0 and world == 1 and not args.no_other_configs:
        line["other_configs"] = {n: measure_config(n, dev) for n in ("c1", "c3") if n != c.name}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = time_oracle(c, q, K, V, lab, args.cpu_seconds)
        line["cpu_baseline"].pop("s_per_step", None)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
