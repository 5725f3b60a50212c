"""Benchmark of the MISA indexer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload ID]

One step is one decode step of MISA-dagger over a batch of sequences (default: 32 sequences x
131072 keys, H_I = 64, d = 128, B = 128, h = 8, k' = 8192, k = 2048):
    route (block-pooled router, top-h heads; the block holding the newest key is averaged from the
    keys) -> routed token scores -> candidate lists of the score rows and top-k' -> dense re-rank
    of the candidates (tensor cores) -> top-k.
(A block is pooled once the prefix has moved past it, once every B = 128 steps of a sequence; the
step does not repeat it.)
Inputs are seeded synthetic tensors resident in HBM (the key cache of 1 GiB per GPU is larger
than L2, so every step streams it from HBM).  Metric: scored query-tokens per second
(T x L / step time), summed over GPUs.  With torchrun every rank runs its own batch of sequences
(independent problems, weak scaling); the time is the max over ranks.

On one GPU the same run also measures, outside the timed step and reported as keys of the same
JSON line:
  dense_dsa_same_inputs     the dense indexer on the decode inputs, and the MISA-dagger:dense ratio
  block_filter_same_inputs  MISA with the token-axis block filter (--block-filter M blocks, 128)
  paged_same_inputs         the MISA-dagger step on the inputs stored in shuffled pages
                            (--paged PAGE_SIZE, 64), checked against the contiguous step
  prefill                   the chunked causal prefill (65536 queries on one 65536-key cache,
                            chunks of 4096): the whole step, the tensor-core scorer's TFLOP/s,
                            and the dense indexer over the same chunks
  glm5_decode               64 sequences x 131072 keys, H_I = 32, B = 256: the MISA step against
                            the dense indexer on the same inputs (time ratio, token IoU)
(--no-legs skips the last two, 0 turns off the first ones).

The reference arm (--impl reference) times the CPU oracle, as it stands, on the host cores, on a
bounded sample of the same workload.
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
           "sha256": "2a95e40e8e18e3539ab5c2cf9f6f0e1967940c2ba9bb48f2df57609ca3e91cbc",
           "bytes_per_key": (1.073908352e9 + 16.844928e6) / 4194304}
# The same for the tensor-core prefill scorer, per scored (query, key) pair, from a capture of one
# chunk's launch; the step's traffic is that rate times the pairs the step scores.
TRAFFIC_PREFILL = {"file": "long_context_sparse_mean_b200/csrc/score_tc.cu",
                   "sha256": "c4db6753fea8fcc662f8a92e3f98af9f7ade68f519c2221d137c1b4b0fb06537",
                   "bytes_per_pair": (56.73728e6 + 984.10624e6) / 260048896}


def _sha(path):
    with open(os.path.join(ROOT, path), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def _traffic(entry, key, units):
    return entry[key] * units if entry["sha256"] == _sha(entry["file"]) else None


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
    """Polls SM clock and clock-event reasons through NVML while the measured region runs."""

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
            time.sleep(0.001)

    def __enter__(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self, window=None):
        s = {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
             "reasons": sorted(self.reasons), "samples": len(self.samples)}
        if window:
            s["window"] = window
        return s


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


def _event_ms(torch, stream, fn, reps):
    """Average device time of fn() over reps back-to-back calls (CUDA events on `stream`)."""
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / reps


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
         "step": ("route + routed scores + candidate lists and top-k' + dense re-rank + top-k" if wl.kp
                  else "route + routed scores + candidate lists and top-k")}
    if extra:
        c.update(extra)
    return c


# ---- seeded inputs, drawn in parallel by spawned worker processes -----------------------------------

def _pool_processes():
    return max(1, min(32, os.cpu_count() or 1))


def _gen_decode_into(task):
    """Worker: draw one decode sequence and store its keys as bf16 bits in the shared block."""
    from multiprocessing import shared_memory
    cid, over, s, slot, shm_name, shape = task
    wl = W.small(cid, **over)
    seq = W.decode_sequence(wl, s)
    shm = shared_memory.SharedMemory(name=shm_name)
    try:
        arr = np.ndarray(shape, dtype=np.uint16, buffer=shm.buf)
        arr[slot] = (seq.k.view(np.uint32) >> 16).astype(np.uint16)
    finally:
        shm.close()
    return slot, seq.q, seq.w, seq.n, seq.needle_pos


class DecodeInputs:
    """Keys of a decode batch as bf16 bits [S, L, d] in shared memory, queries, weights, prefix
    lengths and needle positions."""

    def __init__(self, wl, seqs, pool):
        from multiprocessing import shared_memory
        S, L, d = len(seqs), wl.L, wl.d
        self.shape = (S, L, d)
        self.shm = shared_memory.SharedMemory(create=True, size=max(1, S * L * d * 2))
        over = {f: getattr(wl, f) for f in wl.__dataclass_fields__ if f != "cid"}
        tasks = [(wl.cid, over, s, a, self.shm.name, self.shape) for a, s in enumerate(seqs)]
        res = sorted(pool.map(_gen_decode_into, tasks), key=lambda r: r[0])
        self.k_bits = np.ndarray(self.shape, dtype=np.uint16, buffer=self.shm.buf)
        self.q = np.stack([r[1] for r in res])
        self.w = np.stack([r[2] for r in res])
        self.n = np.array([r[3] for r in res], dtype=np.int32)
        self.needles = [r[4] for r in res]

    def k_f32(self, rows):
        """Keys of the given batch rows as float32 (exactly the bf16 values)."""
        return (self.k_bits[rows].astype(np.uint32) << 16).view(np.float32)

    def k_device(self, torch, dev):
        t = torch.from_numpy(self.k_bits.view(np.int16)).to(dev)
        return t.view(torch.bfloat16)

    def close(self):
        self.k_bits = None
        self.shm.close()
        self.shm.unlink()


def _gen_chunk(cid, seed, c, over=None):
    wl = W.small(cid, seed=seed, **(over or {}))
    ch = wl.chunk
    q, w = W.shared_queries(wl, c * ch, min((c + 1) * ch, wl.T))
    return q, w


def cpu_baseline_sample(wl, seqs, threads=None, inputs=None):
    """Time the oracle, as it stands, on the given sequences (one decode query each).  inputs:
    (k, q, w, n) of exactly those sequences, or None to draw them."""
    import oracle
    o = oracle.get()
    if inputs is None:
        k, q, w, n, _ = W.decode_batch(wl, seqs)
    else:
        k, q, w, n = inputs
    L, d = k.shape[1], k.shape[2]
    t0 = time.perf_counter()
    o.indexer(oracle.MODE_DAGGER if wl.kp else oracle.MODE_MISA, q, w, k, L * d, n, wl.B, wl.h, wl.topk,
              kp=wl.kp or 0)
    dt = time.perf_counter() - t0
    return dt, o.num_threads()


def cpu_block_filter_sample(wl, seqs, m, inputs=None):
    """Time the oracle's route + block filter + refinement on the given decode sequences."""
    import oracle
    o = oracle.get()
    if inputs is None:
        k, q, w, n, _ = W.decode_batch(wl, seqs)
    else:
        k, q, w, n = inputs
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
    run = _graphed(torch, both, not args.no_graph)
    for _ in range(3):
        run()
    step_ms = _event_ms(torch, stream, run, nrep)
    route()
    call_ms = _event_ms(torch, stream, filt, nrep)
    alg = T * (Mb * h_d * 4 + h * h_d * 2 + h * 4 + P * (h_d * 2 + 4 + 4 + 4) + m * 4 + kk * 8)
    return {"m": m, "kept_tokens_per_query": P, "route_plus_filter_ms": step_ms,
            "query_tokens_per_s": T * L / (step_ms / 1000.0), "call_ms": call_ms,
            "algorithmic_bytes_per_call": alg, "launches_per_call": 5}


def paged_leg(args, torch, M, qd, wd, kd, nd, wl, stream, dev, ref_idx=None):
    """MISA-dagger on the same decode inputs stored in pages of one shared pool, outside the timed
    step: the caches are copied page by page into a shuffled pool (page_size keys a page), then
    route + routed scores + top-k' + re-rank + top-k through the *_paged calls are replayed as a
    CUDA graph (as in the main step, the router averages each prefix's last block from the keys).
    The final selection is compared with the contiguous step's (ref_idx) on the same inputs; the
    paged routed-scoring call is timed alone against its algorithmic bytes (the key rows and the
    page-table entries it reads)."""
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
    heads = torch.empty((T, h), dtype=torch.int32, device=dev)
    cand = torch.empty((T, kp), dtype=torch.int32, device=dev) if kp is not None else None
    idx = torch.empty((T, kk), dtype=torch.int32, device=dev)
    vals = torch.empty((T, kk), dtype=torch.float32, device=dev)
    wsp = M.Workspace(dev)

    def score():
        M.misa_score_topk_paged(qd, wd, pool, table, nd, heads, kp, L=L, idx=cand, want_vals=False, ws=wsp)

    def step():
        M.misa_route_paged(qd, wd, pool, table, kbar, nd, B, h, L=L, heads=heads, ws=wsp)
        score()
        M.misa_hier_rerank_paged(qd, wd, pool, table, nd, cand, kk, L=L, idx=idx, vals=vals, ws=wsp)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    same = None
    if ref_idx is not None:
        same = bool(torch.equal(torch.sort(idx, dim=1).values, torch.sort(ref_idx, dim=1).values))
    run = _graphed(torch, step, not args.no_graph)
    for _ in range(3):
        run()
    nrep = max(1, min(args.steps, 50))
    ms = _event_ms(torch, stream, run, nrep)
    score_ms = _event_ms(torch, stream, score, nrep)
    hbm, kind = _peaks()
    alg = T * (L * d * 2 + lp * 4)
    return {"page_size": ps, "pages_per_sequence": lp, "ms_per_step": ms,
            "query_tokens_per_s": T * L / (ms / 1000.0), "launches_per_step": 10,
            "matches_contiguous": same,
            "routed_scoring_call": {"ms": score_ms, "algorithmic_bytes": alg,
                                    "achieved_GBps": alg / (score_ms / 1000.0) / 1e9,
                                    "frac_of_hbm": alg / (score_ms / 1000.0) / 1e9 / hbm, "peak_kind": kind,
                                    "launches": 5}}


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


# ---- the reference arm: the oracle on the host cores -------------------------------------------------

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
    k, q, w, n, _ = W.decode_batch(wl, seqs)
    for _ in range(args.warmup):
        cpu_baseline_sample(wl, seqs, inputs=(k, q, w, n))
    times = []
    for _ in range(args.steps):
        dt, thr = cpu_baseline_sample(wl, seqs, inputs=(k, q, w, n))
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
                         "sample": f"{per_step} of {wl.T} sequences per step, whole "
                                   f"{'MISA-dagger' if wl.kp else 'MISA'} path, double precision, OpenMP over "
                                   f"sequences"},
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


# ---- chunked causal prefill (shared cache) ------------------------------------------------------------

def prefill_measure(args, wl, dev, gen_pool, steps, warmup, dist=None, ws=1, want_e2e=True, want_dense=True,
                    want_cpu=True, fused=False, inputs=None):
    """One step = the whole chunked causal prefill of one sequence: pool every block of the shared
    cache once, then for each chunk of queries route, score with the routed heads on the tensor
    cores, and select the top-k of every query (fused: scoring and selection in one call that writes
    no score rows, misa_score_topk_fused).  Returns the measurements as a dict; inputs: the device
    tensors of an earlier call, to measure the other path on the same inputs."""
    import torch
    from long_context_sparse_mean_b200 import binding as M

    ch = wl.chunk
    nch = -(-wl.T // ch)
    k_h = W.shared_keys(wl)
    n_h = W.prefix_lengths(wl)
    L, d, T, B, h, kk = wl.L, wl.d, wl.T, wl.B, wl.h, wl.topk
    if inputs is None:
        over = {f: getattr(wl, f) for f in wl.__dataclass_fields__ if f not in ("cid", "seed")}
        parts = gen_pool.starmap(_gen_chunk, [(wl.cid, wl.seed, c, over) for c in range(nch)])
        kd = torch.from_numpy(k_h).to(torch.bfloat16).to(dev)
        qd = torch.cat([torch.from_numpy(p[0]).to(torch.bfloat16) for p in parts]).to(dev)
        wd = torch.cat([torch.from_numpy(p[1]) for p in parts]).to(dev)
        nd = torch.from_numpy(n_h).to(dev)
        del parts
    else:
        kd, qd, wd, nd = inputs
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
            if fused:
                M.misa_score_topk_fused(qc, wc, kd, nc, hc, kk, idx=idx[a:b], want_vals=False, ws=sel_ws)
            else:
                M.misa_token_scores(qc, wc, kd, nc, hc, out=sc)
            if time_scores:
                score_ev[c][1].record(stream)
            if stages:
                stage_ev[c][2].record(stream)
            if not fused:
                M.misa_topk_select(sc, nc, kk, idx=idx[a:b], want_vals=False, ws=sel_ws)
            if stages:
                stage_ev[c][3].record(stream)

    # launches per step: pool + per chunk: the router (pooled-key split, tensor-core router, finish)
    # and scores + selection, or fused: sample, cuts, compact scores, list selection and the two
    # launches of the exact redo (empty unless a list could not answer)
    launches_per_step = 1 + nch * (3 + (6 if fused else 2))
    for _ in range(max(3, warmup)):
        step()
    torch.cuda.synchronize()

    clk = ClockSampler(dev.index)
    with clk:
        score_ms = 0.0
        nsc = max(1, min(steps, 5))
        for _ in range(nsc):
            step(time_scores=True)
            torch.cuda.synchronize()
            score_ms += sum(e0.elapsed_time(e1) for e0, e1 in score_ev)
        score_ms /= nsc
        acc = {"pool_all_blocks": 0.0, "route": 0.0, "routed_scores": 0.0, "topk": 0.0}
        nst = max(1, min(steps, 5))
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
        t0.record(stream)
        for _ in range(steps):
            run_step()
        t1.record(stream)
        torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1)
    if ws > 1:
        ms = max_over_ranks(ms, dist, dev)
    out = {"ms": ms, "steps": steps, "pairs": pairs, "flops": flops, "score_ms": score_ms, "stages_us": stages_us,
           "launches_per_step": launches_per_step, "clocks": clk.summary("score, stage and timed passes"),
           "inputs": (kd, qd, wd, nd), "idx": idx}

    if want_e2e:
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
            run_step()
            idx_pin.copy_(idx, non_blocking=True)

        ne = max(1, min(steps, 5))
        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        if ws > 1:
            dist.barrier()
        e_ms = _event_ms(torch, stream, e2e_step, ne) * ne
        if ws > 1:
            e_ms = max_over_ranks(e_ms, dist, dev)
        out["e2e"] = {"ms": e_ms, "steps": ne, "h2d": h2d, "d2h": d2h}

    if want_dense:
        # the dense indexer over the same chunks (all H_I heads on the tensor cores, then top-k)
        didx = torch.empty((ch, kk), dtype=torch.int32, device=dev)

        def dense_step():
            for a, b in chunks:
                M.dsa_dense_topk(qd[a:b], wd[a:b], kd, nd[a:b], kk, idx=didx[: b - a], want_vals=False, ws=wsp)

        dense_step()
        torch.cuda.synchronize()
        run_dense = _graphed(torch, dense_step, not args.no_graph)
        run_dense()
        dense_ms = _event_ms(torch, stream, run_dense, max(1, min(steps, 3)))
        out["dense"] = {"ms_per_step": dense_ms, "pairs_per_s": pairs / (dense_ms / 1000.0),
                        "misa_over_dense_time": (ms / steps) / dense_ms,
                        "dense_speedup_of_misa": dense_ms / (ms / steps),
                        "launches_per_step": nch * 2}
    if want_cpu and not args.no_cpu_baseline:
        count = max(1, min(64, 2 * (os.cpu_count() or 1)))
        dt, thr, u = cpu_prefill_sample(wl, prefill_sample_inputs(wl, count))
        out["cpu_baseline"] = {"value": u / dt, "unit": UNIT, "cores": thr, "kind": "oracle",
                               "sample": f"the last {count} of {T} prefill queries: route + routed scores + "
                                         f"top-k, double precision, OpenMP over queries"}
    return out


def _prefill_roofline(wl, r):
    peaks = _tc_peaks()
    achieved = r["flops"] / (r["score_ms"] / 1000.0) / 1e12
    return {"bound": "tensor", "kernel": "routed token scoring (score_tc_kernel, tcgen05)",
            "achieved": achieved, "peak": peaks["burst"], "peak_kind": peaks["kind"] + " burst", "unit": "TFLOP/s",
            "frac": achieved / peaks["burst"], "frac_of_sustained_peak": achieved / peaks["sustained"],
            "sustained_peak": peaks["sustained"],
            "traffic": _traffic(TRAFFIC_PREFILL, "bytes_per_pair", r["pairs"]),
            "traffic_note": "per step (one scorer launch per 4096-query chunk): DRAM bytes per scored pair from "
                            "one chunk's ncu capture x pairs per step",
            "algorithmic_flops_per_step": r["flops"], "score_ms_per_step": r["score_ms"],
            "peak_choice": "burst: the scorer is event-timed per chunk launch (about 0.3 ms each)"}


def _prefill_config(wl, ws, args):
    L, T, ch, pairs = wl.L, wl.T, wl.chunk, int(W.prefix_lengths(wl).astype(np.int64).sum())
    return {"workload": wl.name, "L": L, "T": T, "chunk": ch, "H_I": wl.H_I, "d": wl.d, "B": wl.B, "h": wl.h,
            "topk": wl.topk, "accumulate": "f32", "causal": "n_t = t + 1",
            "units": f"scored (query, key) pairs, sum of n_t = {pairs} per step (T x L = {T * L})",
            "l2": f"score rows of one chunk ({ch * L * 4 / 2**30:.1f} GiB) exceed L2; the 16 MiB key cache stays "
                  f"in L2",
            "parallelism": f"{ws} GPU(s), one independent sequence per GPU", "cuda_graph": not args.no_graph,
            "step": "pool all blocks + per chunk: route + routed scores + top-k"}


def run_prefill(args, wl):
    """The prefill workload as the main line (--workload 3)."""
    import multiprocessing as mp

    ws, rank, local = _dist()
    wl = rank_workload(wl, rank)
    with mp.get_context("spawn").Pool(_pool_processes()) as gen_pool:
        import torch
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dev = torch.device("cuda", local)
        if ws > 1:
            dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))
        r = prefill_measure(args, wl, dev, gen_pool, args.steps, args.warmup, dist if ws > 1 else None, ws,
                            want_dense=not args.no_dense, want_cpu=rank == 0, fused=args.fused)
    if rank == 0:
        e = r["e2e"]
        line = {
            "metric": METRIC, "value": r["pairs"] * ws * args.steps / (r["ms"] / 1000.0), "unit": UNIT,
            "n_gpus": ws, "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms"] / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(_prefill_config(wl, ws, args), fused=bool(args.fused)),
            "roofline": _prefill_roofline(wl, r),
            "e2e": {"value": r["pairs"] * ws * e["steps"] / (e["ms"] / 1000.0), "unit": UNIT,
                    "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"]},
            "gpu_launches": r["launches_per_step"] * args.steps,
            "stages_us": r["stages_us"],
            "clocks": r["clocks"],
        }
        if "dense" in r:
            line["dense_dsa_same_inputs"] = r["dense"]
        if "cpu_baseline" in r:
            line["cpu_baseline"] = r["cpu_baseline"]
        print(json.dumps(line), flush=True)
    if ws > 1:
        dist.destroy_process_group()
    return 0


# ---- decode legs ------------------------------------------------------------------------------------

def misa_decode_leg(args, torch, M, wl, dev, gen_pool, steps):
    """MISA (routed top-k, no re-rank) against the dense indexer on one decode workload, outside the
    main timed step: the step (route + routed scores + top-k) replayed as a CUDA graph, the routed
    scoring call alone against its algorithmic bytes, the dense indexer on the same inputs, and the
    token IoU of the two selections."""
    inp = DecodeInputs(wl, list(range(wl.T)), gen_pool)
    try:
        kd = inp.k_device(torch, dev)
    finally:
        inp.close()
    qd = torch.from_numpy(inp.q).to(torch.bfloat16).to(dev)
    wd = torch.from_numpy(inp.w).to(dev)
    nd = torch.from_numpy(inp.n).to(dev)
    T, L, d = kd.shape
    B, h, kk = wl.B, wl.h, wl.topk
    stream = torch.cuda.current_stream()
    wsp, sel_ws = M.Workspace(dev), M.Workspace(dev)
    kbar = M.misa_pool_keys(kd, B)
    heads = torch.empty((T, h), dtype=torch.int32, device=dev)
    scores = torch.empty((T, L), dtype=torch.float32, device=dev)
    idx = torch.empty((T, kk), dtype=torch.int32, device=dev)
    didx = torch.empty((T, kk), dtype=torch.int32, device=dev)

    def route():
        M.misa_route(qd, wd, kd, kbar, nd, B, h, heads=heads, ws=wsp)

    def score():
        M.misa_token_scores(qd, wd, kd, nd, heads, out=scores)

    def step():
        route()
        score()
        M.misa_topk_select(scores, nd, kk, idx=idx, want_vals=False, ws=sel_ws)

    def dense():
        M.dsa_dense_topk(qd, wd, kd, nd, kk, idx=didx, want_vals=False, ws=wsp)

    for _ in range(3):
        step()
        dense()
    torch.cuda.synchronize()
    a, b = idx.cpu().numpy(), didx.cpu().numpy()
    ious = [len(np.intersect1d(a[t][a[t] >= 0], b[t][b[t] >= 0])) /
            max(1, len(np.union1d(a[t][a[t] >= 0], b[t][b[t] >= 0]))) for t in range(T)]
    run = _graphed(torch, step, not args.no_graph)
    run_dense = _graphed(torch, dense, not args.no_graph)
    for _ in range(3):
        run()
        run_dense()
    nrep = max(3, min(steps, 50))
    clk = ClockSampler(dev.index)
    with clk:
        ms = _event_ms(torch, stream, run, nrep)
        dense_ms = _event_ms(torch, stream, run_dense, nrep)
        route()
        score_ms = _event_ms(torch, stream, score, nrep)
    hbm, kind = _peaks()
    alg = T * (L * d * 2 + h * d * 2 + h * 4)
    res = {"workload": wl.name, "T": T, "L": L, "H_I": wl.H_I, "B": B, "h": h, "topk": kk,
           "step": "route + routed scores + candidate lists and top-k",
           "ms_per_step": ms, "query_tokens_per_s": T * L / (ms / 1000.0), "launches_per_step": 5,
           "roofline": {"bound": "hbm", "kernel": "routed token scoring (score_persist_kernel)",
                        "achieved": alg / (score_ms / 1000.0) / 1e9, "peak": hbm, "peak_kind": kind,
                        "unit": "GB/s", "frac": alg / (score_ms / 1000.0) / 1e9 / hbm,
                        "algorithmic_bytes_per_launch": alg, "avg_launch_ms": score_ms},
           "dense": {"ms_per_call": dense_ms, "query_tokens_per_s": T * L / (dense_ms / 1000.0),
                     "launches_per_call": 4},
           "misa_over_dense_time": ms / dense_ms, "dense_speedup_of_misa": dense_ms / ms,
           "iou_vs_dense": float(np.mean(ious)), "iou_vs_dense_min": float(np.min(ious)),
           "clocks": clk.summary("step, dense and scorer timing passes")}
    del kd, qd, wd, nd, kbar, scores
    return res


def run_ours(args):
    import multiprocessing as mp

    ws, rank, local = _dist()
    wl = _workload(args)
    if wl.n_seq == 1:
        raise SystemExit("shared-cache workloads run through run_prefill")
    gen_pool = mp.get_context("spawn").Pool(_pool_processes())
    try:
        return _run_ours(args, ws, rank, local, wl, gen_pool)
    finally:
        gen_pool.close()
        gen_pool.join()


def _run_ours(args, ws, rank, local, wl, gen_pool):
    big = W.small(wl.cid, n_seq=wl.n_seq * ws, T=wl.T * ws)
    seqs = rank_sequences(rank, ws, wl.T)
    inp = DecodeInputs(big, seqs, gen_pool)

    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if ws > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))
    from long_context_sparse_mean_b200 import binding as M

    kd = inp.k_device(torch, dev)
    T, L, d = inp.shape
    B, h, kp, kk, H_I = wl.B, wl.h, wl.kp, wl.topk, wl.H_I
    stream = torch.cuda.current_stream()
    # q, w and n live in one device staging block, so the end-to-end step fills them (and the newest
    # key of every sequence) with one host-to-device copy
    q_bytes, w_bytes, n_bytes, knew_bytes = T * H_I * d * 2, T * H_I * 4, T * 4, T * d * 2
    offs = np.cumsum([0] + [(x + 255) // 256 * 256 for x in (q_bytes, w_bytes, n_bytes, knew_bytes)])
    stage_d = torch.empty(int(offs[-1]), dtype=torch.uint8, device=dev)
    qd = stage_d[offs[0]:offs[0] + q_bytes].view(torch.bfloat16).view(T, H_I, d)
    wd = stage_d[offs[1]:offs[1] + w_bytes].view(torch.float32).view(T, H_I)
    nd = stage_d[offs[2]:offs[2] + n_bytes].view(torch.int32)
    knew_d = stage_d[offs[3]:offs[3] + knew_bytes].view(torch.bfloat16).view(T, d)
    qd.copy_(torch.from_numpy(inp.q).to(torch.bfloat16))
    wd.copy_(torch.from_numpy(inp.w))
    nd.copy_(torch.from_numpy(inp.n))
    knew_d.copy_(kd[:, L - 1, :])
    wsp = M.Workspace(dev)
    sel_ws = M.Workspace(dev)  # selection state shared by the scoring and top-k' calls
    kbar = M.misa_pool_keys(kd, B)
    heads = torch.empty((T, h), dtype=torch.int32, device=dev)
    scores = torch.empty((T, L), dtype=torch.float32, device=dev)
    cand = torch.empty((T, kp), dtype=torch.int32, device=dev) if kp is not None else None
    idx = torch.empty((T, kk), dtype=torch.int32, device=dev)
    vals = torch.empty((T, kk), dtype=torch.float32, device=dev)
    mode = args.dagger if kp is not None else "unfused"

    def route():
        M.misa_route(qd, wd, kd, kbar, nd, B, h, heads=heads, ws=wsp)

    def score():
        M.misa_token_scores(qd, wd, kd, nd, heads, out=scores)

    def select():
        if kp is not None:  # the k' candidates
            M.misa_topk_select(scores, nd, kp, idx=cand, want_vals=False, ws=sel_ws)
        else:  # MISA: the top-k itself
            M.misa_topk_select(scores, nd, kk, idx=idx, vals=vals, ws=sel_ws)

    def rerank():
        if kp is not None:
            M.misa_hier_rerank(qd, wd, kd, nd, cand, kk, idx=idx, vals=vals, ws=wsp)

    def fused_rest():
        M.misa_hier_topk_fused(qd, wd, kd, nd, heads, kp, kk, idx=idx, vals=vals, ws=sel_ws)

    def step_unfused():
        route()
        score()
        select()
        rerank()

    def step_fused():
        route()
        fused_rest()

    comps = {"unfused": step_unfused}
    if kp is not None:
        comps["fused"] = step_fused
    for _ in range(max(3, args.warmup)):
        for fn in comps.values():
            fn()
    torch.cuda.synchronize()

    clk = ClockSampler(local)
    with clk:
        # each stage alone, replayed back to back as its own graph (the device time of its launches,
        # no host gaps); the routed scoring call is the roofline's kernel
        nrep = max(3, min(args.steps, 20))
        stages_us = {}
        stage_fns = [("route", route), ("routed_scores", score)]
        if kp is not None:
            stage_fns += [("topk_kprime", select), ("rerank", rerank), ("scores_and_selections_fused", fused_rest)]
        else:
            stage_fns += [("topk", select)]
        for nm, fn in stage_fns:
            g = _graphed(torch, fn, not args.no_graph)
            g()
            stages_us[nm] = round(1000 * _event_ms(torch, stream, g, nrep), 2)
            if nm == "routed_scores":
                score_avg = stages_us[nm] / 1000.0
            del g
        # both compositions of the MISA-dagger step (the same selection): the four separate calls, or
        # misa_route + misa_hier_topk_fused; --dagger auto times the step with the faster one here
        comp_ms = {}
        for nm, fn in comps.items():
            g = _graphed(torch, fn, not args.no_graph)
            g()
            comp_ms[nm] = _event_ms(torch, stream, g, nrep)
            del g
        chosen = min(comp_ms, key=comp_ms.get) if mode == "auto" else mode
        step = comps[chosen]
        other_ms = {nm: v for nm, v in comp_ms.items() if nm != chosen}
        # kernels per step.  Fused: router, sampled scores, list cut, routed scorer keeping the dense
        # scores of the tokens at or above the cut, the two selections (one CTA per row).  Unfused:
        # router, routed scorer, list cut, list sweep, top-k' (one CTA per row), re-rank, top-k.
        launches_per_step = 5 if chosen == "fused" else (7 if kp is not None else 5)
        step()  # the stages above reran on the same inputs; leave one whole step's state behind
        torch.cuda.synchronize()

        # the timed region: K whole steps
        run_step = _graphed(torch, step, not args.no_graph)
        for _ in range(3):
            run_step()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if ws > 1:
            dist.barrier()
        torch.cuda.synchronize()
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
    # the paged leg's reference: the same separate calls on the contiguous caches (the fused call's
    # dense scores round differently, so near-ties at the k-th may be ordered otherwise)
    step_unfused()
    torch.cuda.synchronize()
    ref_idx = idx.clone()

    # end to end through the public API with host buffers: per step the new queries q, their head
    # weights w, the prefix lengths n and the newest key of every sequence go host->device in one
    # copy from pinned memory (the key is then written into the cache), the step runs, and the
    # selected indices come back device->host.
    stage_pin = torch.empty(int(offs[-1]), dtype=torch.uint8).pin_memory()
    stage_pin.copy_(stage_d.cpu())
    idx_pin = torch.empty((T, kk), dtype=torch.int32).pin_memory()
    h2d = q_bytes + w_bytes + n_bytes + knew_bytes
    d2h = idx_pin.numel() * 4

    def e2e_step():
        stage_d.copy_(stage_pin, non_blocking=True)
        kd[:, L - 1, :].copy_(knew_d)
        run_step()
        idx_pin.copy_(idx, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    if ws > 1:
        dist.barrier()
    e_ms = _event_ms(torch, stream, e2e_step, args.steps) * args.steps
    if ws > 1:
        e_ms = max_over_ranks(e_ms, dist, dev)
    e2e_value = units_per_step * args.steps / (e_ms / 1000.0)

    # dense DSA on the same inputs (the baseline the pages compare against), not part of the step
    dsa_ms = None
    if not args.no_dense:
        didx = torch.empty((T, kk), dtype=torch.int32, device=dev)
        dvals = torch.empty((T, kk), dtype=torch.float32, device=dev)
        for _ in range(3):
            M.dsa_dense_topk(qd, wd, kd, nd, kk, idx=didx, vals=dvals, ws=wsp)
        torch.cuda.synchronize()
        dsa_ms = _event_ms(torch, stream, lambda: M.dsa_dense_topk(qd, wd, kd, nd, kk, idx=didx, vals=dvals, ws=wsp),
                           min(args.steps, 20))

    single = ws == 1
    bf = block_filter_leg(args, torch, M, qd, wd, kd, kbar, nd, wl, stream, dev, h_d=d) \
        if args.block_filter and single else None
    paged = paged_leg(args, torch, M, qd, wd, kd, nd, wl, stream, dev, ref_idx=ref_idx) \
        if args.paged and wl.kp and single else None

    line = None
    if rank == 0:
        hbm, kind = _peaks()
        alg_bytes = T * (L * d * 2 + h * d * 2 + h * 4)
        achieved = alg_bytes / (score_avg / 1000.0) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": _config(wl, {"parallelism": f"{ws} GPU(s), independent sequences per GPU",
                                   "cuda_graph": not args.no_graph}),
            "roofline": {"bound": "hbm",
                         "kernel": "routed token scoring (score_persist_kernel<1, 0>, the misa_token_scores call; "
                                   "the fused step runs its list-keeping variant <1, 3> over the same key bytes)",
                         "achieved": achieved, "peak": hbm, "peak_kind": kind, "unit": "GB/s",
                         "frac": achieved / hbm,
                         "traffic": _traffic(TRAFFIC, "bytes_per_key", T * L),
                         "algorithmic_bytes_per_launch": alg_bytes, "avg_launch_ms": score_avg,
                         "timing": "the scoring call (one launch) replayed back to back as a CUDA graph, CUDA "
                                   "events on its stream"},
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches_per_step * args.steps,
            "stages_us": stages_us,
            "dagger_step": None if kp is None else
                           ("fused (misa_route + misa_hier_topk_fused)" if chosen == "fused" else
                            "unfused (misa_route, misa_token_scores, misa_topk_select, misa_hier_rerank)") +
                           ("; auto: the faster of the two compositions on this run" if mode == "auto" else ""),
            "other_dagger_step_ms": other_ms,
            "clocks": clk.summary("scorer, stage and timed passes"),
            "dense_dsa_same_inputs": None if dsa_ms is None else {
                "ms_per_call": dsa_ms, "query_tokens_per_s": T * L / (dsa_ms / 1000.0),
                "misa_dagger_step_over_dense_call": (ms / args.steps) / dsa_ms},
        }
        if bf is not None:
            bf["achieved_GBps"] = bf["algorithmic_bytes_per_call"] / (bf["call_ms"] / 1000.0) / 1e9
            bf["frac_of_hbm"] = bf["achieved_GBps"] / hbm
            if not args.no_cpu_baseline:
                dt, thr = cpu_block_filter_sample(wl, [0], args.block_filter,
                                                  inputs=(inp.k_f32([0]), inp.q[:1], inp.w[:1], inp.n[:1]))
                bf["cpu_oracle"] = {"query_tokens_per_s": L / dt, "cores": thr,
                                    "sample": "1 sequence, route + block filter + refinement, double precision"}
            line["block_filter_same_inputs"] = bf
        if paged is not None:
            line["paged_same_inputs"] = paged
        if not args.no_cpu_baseline:
            per = max(1, min(T, os.cpu_count() or 1))
            rows = list(range(per))
            dt, thr = cpu_baseline_sample(wl, rows, inputs=(inp.k_f32(rows), inp.q[:per], inp.w[:per], inp.n[:per]))
            line["cpu_baseline"] = {"value": per * L / dt, "unit": UNIT, "cores": thr, "kind": "oracle",
                                    "sample": f"{per} of {T} sequences, one pass of the whole MISA-dagger path, "
                                              f"double precision, OpenMP over sequences"}
    inp.close()
    if ws > 1:
        dist.destroy_process_group()

    if rank == 0 and single and not args.no_legs:
        # further workloads on the same GPU, outside the timed step
        del kd, stage_d, qd, wd, nd, knew_d, kbar, scores, cand, idx, vals, ref_idx
        wsp = sel_ws = None
        M.release_default_workspaces()
        torch.cuda.empty_cache()
        legs = {}
        try:
            r = prefill_measure(args, W.WORKLOADS[3], dev, gen_pool, max(1, min(args.steps, 5)), 2,
                                want_e2e=False, want_dense=not args.no_dense)
            pre = {"config": _prefill_config(W.WORKLOADS[3], 1, args),
                   "metric": "scored (query, key) pairs per second",
                   "value": r["pairs"] * r["steps"] / (r["ms"] / 1000.0), "ms_per_step": r["ms"] / r["steps"],
                   "steps": r["steps"], "roofline": _prefill_roofline(W.WORKLOADS[3], r),
                   "stages_us": r["stages_us"], "gpu_launches_per_step": r["launches_per_step"],
                   "clocks": r["clocks"]}
            if "dense" in r:
                pre["dense_same_inputs"] = r["dense"]
            if "cpu_baseline" in r:
                pre["cpu_baseline"] = r["cpu_baseline"]
            # the same step with scoring and selection fused (no score rows), on the same inputs
            f = prefill_measure(args, W.WORKLOADS[3], dev, gen_pool, max(1, min(args.steps, 5)), 2,
                                want_e2e=False, want_dense=False, want_cpu=False, fused=True, inputs=r["inputs"])
            same = bool(torch.equal(torch.sort(f["idx"], dim=1).values, torch.sort(r["idx"], dim=1).values))
            pre["fused"] = {"ms_per_step": f["ms"] / f["steps"],
                            "value": f["pairs"] * f["steps"] / (f["ms"] / 1000.0),
                            "scoring_and_selection_ms_per_step": f["score_ms"],
                            "effective_TFLOPs": f["flops"] / (f["score_ms"] / 1000.0) / 1e12,
                            "stages_us": f["stages_us"], "gpu_launches_per_step": f["launches_per_step"],
                            "matches_unfused": same, "clocks": f["clocks"],
                            "speedup_over_unfused_step": r["ms"] / r["steps"] / (f["ms"] / f["steps"])}
            del r, f
            legs["prefill"] = pre
        except Exception as exc:  # a failed leg is reported, the headline stands
            legs["prefill"] = {"error": f"{type(exc).__name__}: {exc}"}
        torch.cuda.empty_cache()
        try:
            legs["glm5_decode"] = misa_decode_leg(args, torch, M, W.WORKLOADS[5], dev, gen_pool, args.steps)
        except Exception as exc:
            legs["glm5_decode"] = {"error": f"{type(exc).__name__}: {exc}"}
        line.update(legs)
    if line is not None:
        print(json.dumps(line), flush=True)
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
    ap.add_argument("--no-legs", action="store_true",
                    help="decode: skip the prefill and GLM-5-shaped decode legs that follow the main line")
    ap.add_argument("--fused", action="store_true",
                    help="prefill main line: score and select each chunk with misa_score_topk_fused (no score rows)")
    ap.add_argument("--dagger", choices=["auto", "fused", "unfused"], default="auto",
                    help="MISA-dagger decode step: one call for scores and both selections (fused), the "
                         "separate scoring, top-k' and re-rank calls (unfused), or the faster of the two as "
                         "timed in the run (auto); the other is reported beside it")
    ap.add_argument("--no-graph", action="store_true", help="launch every call of a step instead of replaying "
                                                              "the step as a CUDA graph")
    ap.add_argument("--paged", type=int, default=64, metavar="PAGE_SIZE",
                    help="decode: also time the MISA-dagger step on the same inputs stored in shuffled pages of "
                         "PAGE_SIZE keys (the *_paged calls), outside the timed step (0: off)")
    ap.add_argument("--block-filter", type=int, default=128, metavar="M",
                    help="decode: also time MISA with the token-axis block filter keeping M blocks per query "
                         "(route + misa_block_filter_topk) on the same inputs, outside the timed step (0: off)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    wl = _workload(args)
    if wl.n_seq == 1:
        return run_prefill(args, wl)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
