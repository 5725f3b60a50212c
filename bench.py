"""Benchmark of the MISA indexer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload ID]

One step is one decode step of MISA-dagger over a batch of sequences (default: 32 sequences x
131072 keys, H_I = 64, d = 128, B = 128, h = 8, k' = 8192, k = 2048):
    pool the block that holds the newest key -> route (block-pooled router, top-h heads) ->
    routed token scores -> top-k' candidates -> dense re-rank of the candidates -> top-k.
Inputs are seeded synthetic tensors resident in HBM (the key cache of 1 GiB per GPU is larger
than L2, so every step streams it from HBM).  Metric: scored query-tokens per second
(T x L / step time), summed over GPUs.  With torchrun every rank runs its own batch of sequences
(independent problems, weak scaling); the time is the max over ranks.

The reference arm (--impl reference) times the CPU oracle, as it stands, on the host cores, on a
bounded sample of the same workload.

--block-filter M (decode workloads) adds, outside the timed step, MISA with the token-axis block
filter keeping M blocks per query on the same inputs (route + misa_block_filter_topk) as the
line's "block_filter_same_inputs" object; --paged PAGE_SIZE adds the same MISA-dagger step on the
inputs stored in shuffled pages ("paged_same_inputs").
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_sparse_mean_b200 import workloads as W  # noqa: E402

METRIC = "scored query-tokens/s (Tq x L per s) at L=128K; % of HBM / bf16 TC roofline"
UNIT = "query-tokens/s"

# DRAM traffic of the routed scoring kernel from one ncu capture (dram__bytes_read.sum +
# dram__bytes_write.sum), per scored key, with the hash of the source it was taken on; the
# bench reports null once the kernel source has changed since.
TRAFFIC = {"file": "long_context_sparse_mean_b200/csrc/score.cu",
           "sha256": "63ad9e52310709f8745fdb1ae7c3406bfae625c2343add5a1deb685d3bae57c2",
           "bytes_per_key": (1.073953e9 + 19.169792e6) / 4194304,
           "capture": "profiles/score_persist_decode_L131072_b32.md"}
# The same for the tensor-core prefill scorer, per scored (query, key) pair, from a capture of one
# chunk's launch; the step's traffic is that rate times the pairs the step scores.
TRAFFIC_PREFILL = {"file": "long_context_sparse_mean_b200/csrc/score_tc.cu",
                   "sha256": "3aa6df1f296fc7e0cb8afde7e9ae237d607084f9533b601ca428cd9b148f33ba",
                   "bytes_per_pair": (52.319232e6 + 984.943616e6) / 260048896,
                   "capture": "profiles/score_tc_prefill_L65536_chunk15.md"}


def _sha(path):
    with open(os.path.join(ROOT, path), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def _tc_peaks():
    """Dense bf16 tensor-core peaks in TFLOP/s: burst (a kernel timed alone) and sustained (a
    seconds-long loop under the power cap)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"burst": float(d["bf16_tflops"]), "sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "kind": "measured"}
    return {"burst": 1590.0, "sustained": 1400.0, "kind": "fallback"}


class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML while the timed region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, index):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def _graphed(torch, step, use_graph):
    """The step as a CUDA graph captured from the same C-ABI calls (all launches and memsets of one
    step replayed with one call), or the plain step.  Call after warm-up: the workspaces are sized."""
    if not use_graph:
        return step
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    torch.cuda.synchronize()
    return g.replay


def rank_sequences(rank, world, per_rank):
    """The decode sequences of one rank: a contiguous share of world x per_rank, disjoint from the
    other ranks' (independent problems; no data-path collective)."""
    return list(range(rank * per_rank, (rank + 1) * per_rank))


def rank_workload(wl, rank):
    """The workload a rank runs: rank 0 the named one, every other rank the same shapes with its own
    seed (its own prefill sequence)."""
    return wl if rank == 0 else W.small(wl.cid, seed=wl.seed + 7919 * rank)


def max_over_ranks(ms, dist, device):
    """The largest elapsed time over all ranks: the job's time (one all-reduce of one number)."""
    if dist is None or not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return ms
    import torch
    tt = torch.tensor([float(ms)], device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _workload(args):
    return W.WORKLOADS[args.workload]


def _config(wl, extra=None):
    c = {"workload": wl.name, "T_per_gpu": wl.T, "L": wl.L, "H_I": wl.H_I, "d": wl.d, "B": wl.B, "h": wl.h,
         "kp": wl.kp, "topk": wl.topk, "accumulate": "f32",
         "l2": f"inputs larger than L2 ({wl.T * wl.L * wl.d * 2 / 2**30:.2f} GiB key cache per GPU)",
         "step": "pool newest block + route + routed scores + top-k' + dense re-rank + top-k"}
    if extra:
        c.update(extra)
    return c


def cpu_baseline_sample(wl, seqs, threads=None):
    """Time the oracle, as it stands, on the given sequences (one decode query each)."""
    import oracle
    o = oracle.get()
    k, q, w, n, _ = W.decode_batch(wl, seqs)
    L, d = k.shape[1], k.shape[2]
    t0 = time.perf_counter()
    o.indexer(oracle.MODE_DAGGER if wl.kp else oracle.MODE_MISA, q, w, k, L * d, n, wl.B, wl.h, wl.topk,
              kp=wl.kp or 0)
    dt = time.perf_counter() - t0
    return dt, o.num_threads()


def cpu_block_filter_sample(wl, seqs, m):
    """Time the oracle's route + block filter + refinement on the given decode sequences."""
    import oracle
    o = oracle.get()
    k, q, w, n, _ = W.decode_batch(wl, seqs)
    L, d = k.shape[1], k.shape[2]
    t0 = time.perf_counter()
    o.block_filter(q, w, k, L * d, n, wl.B, wl.h, m, wl.topk)
    return time.perf_counter() - t0, o.num_threads()


def block_filter_leg(args, torch, M, qd, wd, kd, kbar, nd, wl, stream, dev, h_d):
    """MISA with the token-axis block filter on the decode inputs of the main step, outside its
    timed region: route + misa_block_filter_topk keeping m blocks, replayed as a CUDA graph, and
    the block filter call alone.  Algorithmic bytes of the call per query: the M_t pooled keys
    (fp32) and the routed q rows for the block scores, then m*B key rows (bf16), their ids and
    scores for the refinement, and the kept-block and token outputs."""
    m, B, h, kk = args.block_filter, wl.B, wl.h, wl.topk
    T, L = kd.shape[0], kd.shape[1]
    Mb = -(-L // B)
    P = min(m, Mb) * B
    heads = torch.empty((T, h), dtype=torch.int32, device=dev)
    idx = torch.empty((T, kk), dtype=torch.int32, device=dev)
    vals = torch.empty((T, kk), dtype=torch.float32, device=dev)
    blocks = torch.empty((T, m), dtype=torch.int32, device=dev)
    wsp = M.Workspace(dev)

    def route():
        M.misa_route(qd, wd, kd, kbar, nd, B, h, heads=heads, ws=wsp)

    def filt():
        M.misa_block_filter_topk(qd, wd, kd, kbar, nd, heads, B, m, kk, idx=idx, vals=vals, blocks=blocks, ws=wsp)

    def both():
        route()
        filt()

    for _ in range(3):
        both()
    torch.cuda.synchronize()
    nrep = max(1, min(args.steps, 50))
    e = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    run = _graphed(torch, both, not args.no_graph)
    for _ in range(3):
        run()
    e[0].record(stream)
    for _ in range(nrep):
        run()
    e[1].record(stream)
    torch.cuda.synchronize()
    call_ms = 0.0
    for _ in range(nrep):
        route()
        e[2].record(stream)
        filt()
        e[3].record(stream)
        torch.cuda.synchronize()
        call_ms += e[2].elapsed_time(e[3])
    step_ms = e[0].elapsed_time(e[1]) / nrep
    alg = T * (Mb * h_d * 4 + h * h_d * 2 + h * 4 + P * (h_d * 2 + 4 + 4 + 4) + m * 4 + kk * 8)
    return {"m": m, "kept_tokens_per_query": P, "route_plus_filter_ms": step_ms,
            "query_tokens_per_s": T * L / (step_ms / 1000.0), "call_ms": call_ms / nrep,
            "algorithmic_bytes_per_call": alg, "launches_per_call": 5}


def paged_leg(args, torch, M, qd, wd, kd, nd, wl, stream, dev):
    """MISA-dagger on the same decode inputs stored in pages of one shared pool, outside the timed
    step: the caches are copied page by page into a shuffled pool (page_size keys a page), then
    route + routed scores + top-k' + re-rank + top-k through the *_paged calls are replayed as a
    CUDA graph (pooling, like the main step's newest block, refreshes one block per sequence)."""
    ps = args.paged
    T, L, d = kd.shape
    B, h, kp, kk = wl.B, wl.h, wl.kp, wl.topk
    lp = -(-L // ps)
    g = torch.Generator(device="cpu").manual_seed(20261200 + ps)
    perm = torch.randperm(T * lp, generator=g).to(dev)
    pool = torch.zeros((T * lp, ps, d), dtype=kd.dtype, device=dev)
    padded = torch.zeros((T, lp * ps, d), dtype=kd.dtype, device=dev)
    padded[:, :L] = kd
    pool[perm] = padded.reshape(T * lp, ps, d)
    del padded
    table = perm.reshape(T, lp).to(torch.int32).contiguous()
    kbar = M.misa_pool_keys_paged(pool, table, B, L=L)
    M_ = -(-L // B)
    heads = torch.empty((T, h), dtype=torch.int32, device=dev)
    cand = torch.empty((T, kp), dtype=torch.int32, device=dev)
    idx = torch.empty((T, kk), dtype=torch.int32, device=dev)
    vals = torch.empty((T, kk), dtype=torch.float32, device=dev)
    wsp = M.Workspace(dev)

    def step():
        M.misa_pool_keys_paged(pool, table, B, L=L, kbar=kbar, block_begin=M_ - 1, block_end=M_)
        M.misa_route_paged(qd, wd, pool, table, kbar, nd, B, h, L=L, heads=heads, ws=wsp)
        M.misa_score_topk_paged(qd, wd, pool, table, nd, heads, kp, L=L, idx=cand, want_vals=False, ws=wsp)
        M.misa_hier_rerank_paged(qd, wd, pool, table, nd, cand, kk, L=L, idx=idx, vals=vals, ws=wsp)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    run = _graphed(torch, step, not args.no_graph)
    for _ in range(3):
        run()
    nrep = max(1, min(args.steps, 50))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(nrep):
        run()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / nrep
    return {"page_size": ps, "pages_per_sequence": lp, "ms_per_step": ms,
            "query_tokens_per_s": T * L / (ms / 1000.0), "launches_per_step": 9}


def prefill_sample_inputs(wl, count):
    """The last `count` queries of a shared-cache workload (the longest prefixes) and the cache."""
    ch = wl.chunk or wl.T
    c0 = (wl.T - 1) // ch * ch
    q, w = W.shared_queries(wl, c0, wl.T)
    n = W.prefix_lengths(wl, c0, wl.T)
    return W.shared_keys(wl), q[-count:], w[-count:], n[-count:]


def cpu_prefill_sample(wl, inputs):
    """Time the oracle, as it stands, on a few prefill queries: route + routed scores + top-k."""
    import oracle
    o = oracle.get()
    k, q, w, n = inputs
    t0 = time.perf_counter()
    o.indexer(oracle.MODE_MISA, q, w, k, 0, n, wl.B, wl.h, wl.topk)
    dt = time.perf_counter() - t0
    return dt, o.num_threads(), int(n.astype(np.int64).sum())


def run_reference(args):
    """The reference arm: the CPU oracle on a bounded sample of the workload."""
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    wl = _workload(args)
    import oracle
    nthr = oracle.get().num_threads()
    if wl.n_seq == 1:
        return run_reference_prefill(args, wl, nthr)
    per_step = max(1, min(wl.T, nthr))
    seqs = list(range(per_step))
    for _ in range(args.warmup):
        cpu_baseline_sample(wl, seqs)
    times = []
    for _ in range(args.steps):
        dt, thr = cpu_baseline_sample(wl, seqs)
        times.append(dt)
    units = per_step * wl.L
    total = sum(times)
    value = units * args.steps / total
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": _config(wl, {"sample_sequences_per_step": per_step}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                         "sample": f"{per_step} of {wl.T} sequences per step, whole MISA-dagger path, "
                                   f"double precision, OpenMP over sequences"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference_prefill(args, wl, nthr):
    count = max(1, min(64, 2 * nthr))
    inputs = prefill_sample_inputs(wl, count)
    for _ in range(args.warmup):
        cpu_prefill_sample(wl, inputs)
    total, units = 0.0, 0
    for _ in range(args.steps):
        dt, thr, u = cpu_prefill_sample(wl, inputs)
        total += dt
        units += u
    value = units / total
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": _config(wl, {"sample_queries_per_step": count}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                         "sample": f"the last {count} of {wl.T} prefill queries per step (prefixes of "
                                   f"{int(inputs[3].min())}-{int(inputs[3].max())} keys): route + routed scores "
                                   f"+ top-k, double precision, OpenMP over queries; units = scored "
                                   f"(query, key) pairs"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _gen_chunk(cid, seed, c):
    wl = W.small(cid, seed=seed)
    ch = wl.chunk
    q, w = W.shared_queries(wl, c * ch, min((c + 1) * ch, wl.T))
    return q, w


def run_prefill(args, wl):
    """One step = the whole chunked causal prefill of one sequence: pool every block of the shared
    cache once, then for each chunk of queries route, score with the routed heads on the tensor
    cores, and select the top-k of every query."""
    import multiprocessing as mp

    ws, rank, local = _dist()
    wl = rank_workload(wl, rank)
    ch = wl.chunk
    nch = -(-wl.T // ch)
    with mp.get_context("spawn").Pool(min(nch, max(1, os.cpu_count() or 1))) as pool:
        parts = pool.starmap(_gen_chunk, [(wl.cid, wl.seed, c) for c in range(nch)])
    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))
    from long_context_sparse_mean_b200 import binding as M

    k_h = W.shared_keys(wl)
    n_h = W.prefix_lengths(wl)
    L, d, T, B, h, kk = wl.L, wl.d, wl.T, wl.B, wl.h, wl.topk
    kd = torch.from_numpy(k_h).to(torch.bfloat16).to(dev)
    qd = torch.cat([torch.from_numpy(p[0]).to(torch.bfloat16) for p in parts]).to(dev)
    wd = torch.cat([torch.from_numpy(p[1]) for p in parts]).to(dev)
    nd = torch.from_numpy(n_h).to(dev)
    del parts
    stream = torch.cuda.current_stream()
    wsp = M.Workspace(dev)
    sel_ws = M.Workspace(dev)
    kbar = M.misa_pool_keys(kd, B)
    heads = torch.empty((ch, h), dtype=torch.int32, device=dev)
    scores = torch.empty((ch, L), dtype=torch.float32, device=dev)
    idx = torch.empty((T, kk), dtype=torch.int32, device=dev)
    pairs = int(n_h.astype(np.int64).sum())
    flops = 2 * h * d * pairs
    chunks = [(c * ch, min((c + 1) * ch, T)) for c in range(nch)]
    score_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in chunks]
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in chunks]
    pool_ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    def step(time_scores=False, stages=False):
        if stages:
            pool_ev[0].record(stream)
        M.misa_pool_keys(kd, B, kbar=kbar)
        if stages:
            pool_ev[1].record(stream)
        for c, (a, b) in enumerate(chunks):
            qc, wc, nc = qd[a:b], wd[a:b], nd[a:b]
            hc, sc = heads[: b - a], scores[: b - a]
            if stages:
                stage_ev[c][0].record(stream)
            M.misa_route(qc, wc, kd, kbar, nc, B, h, heads=hc, ws=wsp)
            if stages:
                stage_ev[c][1].record(stream)
            if time_scores:
                score_ev[c][0].record(stream)
            M.misa_token_scores(qc, wc, kd, nc, hc, out=sc)
            if time_scores:
                score_ev[c][1].record(stream)
            if stages:
                stage_ev[c][2].record(stream)
            M.misa_topk_select(sc, nc, kk, idx=idx[a:b], want_vals=False, ws=sel_ws)
            if stages:
                stage_ev[c][3].record(stream)

    # launches per step: pool + per chunk (route 1, tensor-core scores 1, selection 3)
    launches_per_step = 1 + nch * 5
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    score_ms = 0.0
    nsc = min(args.steps, 5)
    for _ in range(nsc):
        step(time_scores=True)
        torch.cuda.synchronize()
        score_ms += sum(e0.elapsed_time(e1) for e0, e1 in score_ev)
    score_ms /= nsc
    acc = {"pool_all_blocks": 0.0, "route": 0.0, "routed_scores": 0.0, "topk": 0.0}
    nst = min(args.steps, 5)
    for _ in range(nst):
        step(stages=True)
        torch.cuda.synchronize()
        acc["pool_all_blocks"] += pool_ev[0].elapsed_time(pool_ev[1])
        for c in range(nch):
            e = stage_ev[c]
            acc["route"] += e[0].elapsed_time(e[1])
            acc["routed_scores"] += e[1].elapsed_time(e[2])
            acc["topk"] += e[2].elapsed_time(e[3])
    stages_us = {k_: round(1000 * v / nst, 1) for k_, v in acc.items()}

    run_step = _graphed(torch, step, not args.no_graph)
    for _ in range(2):
        run_step()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            run_step()
        t1.record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    if ws > 1:
        ms = max_over_ranks(ms, dist, dev)
    value = pairs * ws * args.steps / (ms / 1000.0)

    # end to end: every step copies the cache, the queries, their weights and n from pinned host
    # memory and reads every query's top-k indices back
    k_pin = torch.from_numpy(k_h).to(torch.bfloat16).pin_memory()
    q_pin = qd.cpu().pin_memory()
    w_pin = wd.cpu().pin_memory()
    n_pin = torch.from_numpy(n_h).pin_memory()
    idx_pin = torch.empty((T, kk), dtype=torch.int32).pin_memory()
    h2d = k_pin.numel() * 2 + q_pin.numel() * 2 + w_pin.numel() * 4 + n_pin.numel() * 4
    d2h = idx_pin.numel() * 4

    def e2e_step():
        kd.copy_(k_pin, non_blocking=True)
        qd.copy_(q_pin, non_blocking=True)
        wd.copy_(w_pin, non_blocking=True)
        nd.copy_(n_pin, non_blocking=True)
        step()
        idx_pin.copy_(idx, non_blocking=True)

    ne = max(1, min(args.steps, 5))
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(ne):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = e0.elapsed_time(e1)
    if ws > 1:
        e_ms = max_over_ranks(e_ms, dist, dev)
    e2e_value = pairs * ws * ne / (e_ms / 1000.0)

    if rank == 0:
        peaks = _tc_peaks()
        achieved = flops / (score_ms / 1000.0) / 1e12
        traffic = None
        if TRAFFIC_PREFILL["sha256"] == _sha(TRAFFIC_PREFILL["file"]):
            traffic = TRAFFIC_PREFILL["bytes_per_pair"] * pairs
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "L": L, "T": T, "chunk": ch, "H_I": wl.H_I, "d": d, "B": B, "h": h,
                       "topk": kk, "accumulate": "f32", "causal": "n_t = t + 1",
                       "units": f"scored (query, key) pairs, sum of n_t = {pairs} per step "
                                f"(T x L = {T * L})",
                       "l2": f"score rows of one chunk ({ch * L * 4 / 2**30:.1f} GiB) exceed L2; the "
                             f"16 MiB key cache stays in L2",
                       "parallelism": f"{ws} GPU(s), one independent sequence per GPU",
                       "cuda_graph": not args.no_graph,
                       "step": "pool all blocks + per chunk: route + routed scores + top-k"},
            "roofline": {"bound": "tensor", "kernel": "routed token scoring (score_tc_kernel, tcgen05)",
                         "achieved": achieved, "peak": peaks["sustained"], "peak_kind": peaks["kind"] + " sustained",
                         "unit": "TFLOP/s", "frac": achieved / peaks["sustained"],
                         "frac_of_burst_peak": achieved / peaks["burst"], "traffic": traffic,
                         "traffic_per_launch_note": "per step (16 chunk launches): bytes per scored pair from "
                                                    "the capture x pairs per step",
                         "algorithmic_flops_per_step": flops, "score_ms_per_step": score_ms},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "stages_us": stages_us,
            "clocks": clk.summary(),
        }
        if not args.no_cpu_baseline:
            count = max(1, min(64, 2 * (os.cpu_count() or 1)))
            dt, thr, u = cpu_prefill_sample(wl, prefill_sample_inputs(wl, count))
            line["cpu_baseline"] = {"value": u / dt, "unit": UNIT, "cores": thr, "kind": "oracle",
                                    "sample": f"the last {count} of {T} prefill queries: route + routed scores + "
                                              f"top-k, double precision, OpenMP over queries"}
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    ws, rank, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))
    from long_context_sparse_mean_b200 import binding as M

    wl = _workload(args)
    if wl.n_seq == 1:
        raise SystemExit("shared-cache workloads run through run_prefill")
    big = W.small(wl.cid, n_seq=wl.n_seq * ws, T=wl.T * ws)
    seqs = rank_sequences(rank, ws, wl.T)
    k_h, q_h, w_h, n_h, _ = W.decode_batch(big, seqs)
    T, L, d = k_h.shape
    kd = torch.from_numpy(k_h).to(torch.bfloat16).to(dev)
    qd = torch.from_numpy(q_h).to(torch.bfloat16).to(dev)
    wd = torch.from_numpy(w_h).to(dev)
    nd = torch.from_numpy(n_h).to(dev)
    B, h, kp, kk, H_I = wl.B, wl.h, wl.kp, wl.topk, wl.H_I
    M_ = -(-L // B)
    stream = torch.cuda.current_stream()
    wsp = M.Workspace(dev)
    sel_ws = M.Workspace(dev)  # selection state shared by the scoring and top-k' calls
    kbar = M.misa_pool_keys(kd, B)
    heads = torch.empty((T, h), dtype=torch.int32, device=dev)
    scores = torch.empty((T, L), dtype=torch.float32, device=dev)
    cand = torch.empty((T, kp), dtype=torch.int32, device=dev)
    idx = torch.empty((T, kk), dtype=torch.int32, device=dev)
    vals = torch.empty((T, kk), dtype=torch.float32, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    score_ms = []
    # pool, router, scores, top-k' (one CTA per row), re-rank scores, top-k of the candidates; with
    # the fused histogram the top-k' is partition + resolve
    launches_per_step = 7 if args.fused_histogram else 6

    stage_ev = [torch.cuda.Event(enable_timing=True) for _ in range(6)]

    def step(time_scores=False, stages=False):
        mark = (lambda i: stage_ev[i].record(stream)) if stages else (lambda i: None)
        mark(0)
        M.misa_pool_keys(kd, B, kbar=kbar, block_begin=M_ - 1, block_end=M_)
        mark(1)
        M.misa_route(qd, wd, kd, kbar, nd, B, h, heads=heads, ws=wsp)
        mark(2)
        if time_scores:
            ev[0].record(stream)
        if args.fused_histogram:
            M.misa_token_scores(qd, wd, kd, nd, heads, out=scores, select_topk=kp, select_ws=sel_ws)
        else:
            M.misa_token_scores(qd, wd, kd, nd, heads, out=scores)
        if time_scores:
            ev[1].record(stream)
        mark(3)
        M.misa_topk_select(scores, nd, kp, idx=cand, want_vals=False, ws=sel_ws, ws_prepared=args.fused_histogram)
        mark(4)
        M.misa_hier_rerank(qd, wd, kd, nd, cand, kk, idx=idx, vals=vals, ws=wsp)
        mark(5)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    # one timed pass over the step for the scoring-kernel duration (events bracket that launch)
    for _ in range(min(args.steps, 50)):
        step(time_scores=True)
        torch.cuda.synchronize()
        score_ms.append(ev[0].elapsed_time(ev[1]))

    # per-stage breakdown (events between the calls; separate untimed steps)
    stage_names = ["pool_newest_block", "route", "routed_scores", "topk_kprime", "rerank"]
    stage_acc = [0.0] * len(stage_names)
    nst = min(args.steps, 20)
    for _ in range(nst):
        step(stages=True)
        torch.cuda.synchronize()
        for i in range(len(stage_names)):
            stage_acc[i] += stage_ev[i].elapsed_time(stage_ev[i + 1])
    stages_us = {nm: round(1000 * a / nst, 2) for nm, a in zip(stage_names, stage_acc)}

    # the timed region: K whole steps
    run_step = _graphed(torch, step, not args.no_graph)
    for _ in range(3):
        run_step()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if ws > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            run_step()
        t1.record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    if ws > 1:
        ms = max_over_ranks(ms, dist, dev)
    units_per_step = T * L * ws
    value = units_per_step * args.steps / (ms / 1000.0)

    # end to end through the public API with host buffers: per step the new query q, its head
    # weights w, the newest key of every sequence (written into the cache) and n go host->device,
    # and the selected indices come back device->host.
    q_pin = torch.from_numpy(q_h).to(torch.bfloat16).pin_memory()
    w_pin = torch.from_numpy(w_h).pin_memory()
    n_pin = torch.from_numpy(n_h).pin_memory()
    knew_pin = torch.from_numpy(k_h[:, L - 1, :].copy()).to(torch.bfloat16).pin_memory()
    knew_d = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    idx_pin = torch.empty((T, kk), dtype=torch.int32).pin_memory()
    h2d = q_pin.numel() * 2 + w_pin.numel() * 4 + n_pin.numel() * 4 + knew_pin.numel() * 2
    d2h = idx_pin.numel() * 4

    def e2e_step():
        qd.copy_(q_pin, non_blocking=True)
        wd.copy_(w_pin, non_blocking=True)
        nd.copy_(n_pin, non_blocking=True)
        knew_d.copy_(knew_pin, non_blocking=True)
        kd[:, L - 1, :].copy_(knew_d)
        step()
        idx_pin.copy_(idx, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = e0.elapsed_time(e1)
    if ws > 1:
        e_ms = max_over_ranks(e_ms, dist, dev)
    e2e_value = units_per_step * args.steps / (e_ms / 1000.0)

    # dense DSA on the same inputs (the baseline the pages compare against), not part of the step
    dsa_ms = None
    if not args.no_dense:
        for _ in range(3):
            M.dsa_dense_topk(qd, wd, kd, nd, kk, idx=idx, vals=vals, ws=wsp)
        torch.cuda.synchronize()
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        nrep = min(args.steps, 20)
        d0.record(stream)
        for _ in range(nrep):
            M.dsa_dense_topk(qd, wd, kd, nd, kk, idx=idx, vals=vals, ws=wsp)
        d1.record(stream)
        torch.cuda.synchronize()
        dsa_ms = d0.elapsed_time(d1) / nrep

    bf = block_filter_leg(args, torch, M, qd, wd, kd, kbar, nd, wl, stream, dev, h_d=d) if args.block_filter else None
    paged = paged_leg(args, torch, M, qd, wd, kd, nd, wl, stream, dev) if args.paged else None

    if rank == 0:
        hbm, kind = _peaks()
        score_avg = sum(score_ms) / len(score_ms)
        alg_bytes = T * (L * d * 2 + h * d * 2 + h * 4)
        achieved = alg_bytes / (score_avg / 1000.0) / 1e9
        traffic = None
        if TRAFFIC["sha256"] and TRAFFIC["sha256"] == _sha(TRAFFIC["file"]) and TRAFFIC["bytes_per_key"]:
            traffic = TRAFFIC["bytes_per_key"] * T * L
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": _config(wl, {"parallelism": f"{ws} GPU(s), independent sequences per GPU",
                                   "cuda_graph": not args.no_graph}),
            "roofline": {"bound": "hbm", "kernel": "routed token scoring (score_persist_kernel)",
                         "achieved": achieved, "peak": hbm, "peak_kind": kind, "unit": "GB/s",
                         "frac": achieved / hbm, "traffic": traffic,
                         "algorithmic_bytes_per_launch": alg_bytes, "avg_launch_ms": score_avg},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "stages_us": stages_us,
            "clocks": clk.summary(),
            "dense_dsa_same_inputs": None if dsa_ms is None else {
                "ms_per_call": dsa_ms, "query_tokens_per_s": T * L / (dsa_ms / 1000.0)},
        }
        if bf is not None:
            bf["achieved_GBps"] = bf["algorithmic_bytes_per_call"] / (bf["call_ms"] / 1000.0) / 1e9
            bf["frac_of_hbm"] = bf["achieved_GBps"] / hbm
            if not args.no_cpu_baseline:
                dt, thr = cpu_block_filter_sample(wl, [0], args.block_filter)
                bf["cpu_oracle"] = {"query_tokens_per_s": L / dt, "cores": thr,
                                    "sample": "1 sequence, route + block filter + refinement, double precision"}
            line["block_filter_same_inputs"] = bf
        if paged is not None:
            line["paged_same_inputs"] = paged
        if not args.no_cpu_baseline:
            per = max(1, min(T, os.cpu_count() or 1))
            dt, thr = cpu_baseline_sample(wl, list(range(per)))
            line["cpu_baseline"] = {"value": per * L / dt, "unit": UNIT, "cores": thr, "kind": "oracle",
                                    "sample": f"{per} of {T} sequences, one pass of the whole MISA-dagger path, "
                                              f"double precision, OpenMP over sequences"}
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=4, choices=[2, 3, 4, 5])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--fused-histogram", action="store_true",
                    help="decode: build the top-k' histogram inside the scoring kernel and select with the "
                         "partition/resolve kernels (instead of one CTA per row)")
    ap.add_argument("--no-graph", action="store_true", help="launch every call of a step instead of replaying "
                                                              "the step as a CUDA graph")
    ap.add_argument("--paged", type=int, default=0, metavar="PAGE_SIZE",
                    help="decode: also time the MISA-dagger step on the same inputs stored in shuffled pages of "
                         "PAGE_SIZE keys (the *_paged calls), outside the timed step")
    ap.add_argument("--block-filter", type=int, default=0, metavar="M",
                    help="decode: also time MISA with the token-axis block filter keeping M blocks per query "
                         "(route + misa_block_filter_topk) on the same inputs, outside the timed step")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    wl = _workload(args)
    if wl.n_seq == 1:
        return run_prefill(args, wl)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
