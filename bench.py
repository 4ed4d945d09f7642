#!/usr/bin/env python
"""Decode-step throughput of the COBS block-sparse attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cobs|reference]
                    [--stats-format bf16|fp4] [--stats-stream side|same] [--batch B]

One step is one pass of the whole hot path over a batch of synthetic
queries: the statistics of the block that just became complete (one block per
(batch, kv-head)), the second-order block selection (scores + top-k + sink +
local window) and the split-K sparse flash-decode with its log-sum-exp merge —
three C-ABI calls, three kernel launches.  The KV cache and the statistics of
all earlier blocks are resident in HBM before timing starts; L2 is flushed
(256 MiB written, then read) between timed steps and each step is timed with
CUDA events on the stream its kernels run on.  The statistics build runs on a
forked side stream by default (``--stats-stream same`` keeps it in line);
``--stats-format fp4`` stores U in scaled FP4 (E2M1) instead of bf16.  The
line also carries an end-to-end figure through the public calls with host
buffers (``e2e``), the oracle on the host cores (``cpu_baseline``) and the
roofline of the kernel that dominates the step.

Workload (default): batch 32, 32 query / 8 KV heads, head_dim 128, 32768
cached tokens, block 64, rank 8, top-k 16 + sink block + 512-token window,
keys from tight/spread per-block Gaussians with 4 planted needles per
(batch, kv-head) — seeded synthetic data (``workloads``).

Multi-GPU: one process per GPU (torchrun); every rank decodes its own batch
(weak scaling, no collective on the data path); the step time is the max over
ranks and ``value`` counts the queries of all ranks.

``--impl reference`` times the CPU oracle (``oracle/``) on the same workload,
a bounded sample of (batch, kv-head) pairs per step, on rank 0 only.
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
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-decode queries/s and achieved HBM GB/s (% of peak) at 32k context"
UNIT = "queries/s"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=5000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["cobs", "reference"], default="cobs")
    p.add_argument("--workload", default="batched_needles_32k")
    p.add_argument("--batch", type=int, default=0,
                   help="override the workload's batch per GPU (smaller profiling cases)")
    p.add_argument("--gen-workers", type=int, default=0,
                   help="processes drawing the synthetic cache (0 = auto)")
    p.add_argument("--cpu-seconds", type=float, default=10.0,
                   help="time budget of the CPU-oracle baseline sample")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-graph", action="store_true",
                   help="enqueue the timed steps call by call instead of replaying CUDA graphs")
    p.add_argument("--stats-format", choices=["bf16", "fp4", "box", "subspace"], default="bf16",
                   help="block records: mu and U in bf16, U in scaled FP4 (E2M1), the "
                        "per-dimension min/max box (comparison selector), or U projected on "
                        "a query subspace")
    p.add_argument("--subspace-dim", type=int, default=85,
                   help="s of the subspace records (the explainer's adaptive s ~ 85 of 128)")
    p.add_argument("--stats-stream", choices=["side", "same"], default="side",
                   help="run the completed block's stats build on a forked side stream "
                        "(joined before the step ends) or in line before the selection")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# byte model: what the method has to move per launch
# ---------------------------------------------------------------------------

def partition(T, B, sink, local):
    n_blocks = -(-T // B)
    n_full = T // B
    first_local = min(n_full, max(0, T - local) // B)
    sink_end = min(sink, first_local)
    return n_blocks, n_full, sink_end, first_local


def rank_shard(w, rank):
    """The workload one rank decodes: the same shapes, its own seeded batch
    (replicas shard the batch dimension; no data crosses ranks)."""
    return w if rank == 0 else w.scaled(seed=w.seed + 1000003 * rank)


def max_over_ranks(values, dist, device, world):
    """Element-wise maximum of per-rank timings (the slowest rank sets the
    job's time); identity on one rank."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def byte_model(w, n_sel, rec=None):
    """Algorithmic bytes per launch of each kernel for one step (``rec``: bytes
    of one block record; bf16 records by default)."""
    B, d, r = w.block, w.head_dim, w.rank
    pairs = w.batch * w.kv_heads
    nbs, nfull, c0, c1 = partition(w.seq_len, B, w.sink_blocks, w.local_tokens)
    q_bytes = w.batch * w.q_heads * d * 2
    rec = (1 + r) * d * 2 if rec is None else rec
    stats_build = pairs * (B * d * 2 + rec)                 # one block in, one record out
    select = pairs * (c1 - c0) * rec + q_bytes + pairs * (c1 - c0) * 4 + pairs * 4 * (1 + n_sel)
    # valid tokens of the selected blocks (all complete here except a ragged tail)
    kv = 0
    tail = w.seq_len - (nbs - 1) * B
    for_tail = 1 if tail < B else 0
    toks = n_sel * B - (B - tail) * for_tail
    kv = pairs * toks * d * 2 * 2
    decode = kv + q_bytes + pairs * 4 * (1 + n_sel) + w.batch * w.q_heads * (d + 1) * 4
    return {"stats": stats_build, "select": select, "decode": decode}


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for name, flag in zip(names, r[5:9]):
                if flag.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# kernel traffic recorded by ncu (profiles/traffic.json), tied to the source
# ---------------------------------------------------------------------------

def source_hash(name):
    path = os.path.join(ROOT, "block_sparse_long_cobs_b200", "csrc", name)
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def recorded_traffic(kernel_file, workload):
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path)).get(f"{kernel_file}:{workload}")
    if not rec or rec.get("source_sha") != source_hash(kernel_file):
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# the CPU oracle on a bounded sample (baseline and --impl reference)
# ---------------------------------------------------------------------------

class OracleSample:
    """Oracle decode steps for a few (batch, kv-head) pairs of the workload."""

    def __init__(self, w, q_bits, k_bits, v_bits, pairs):
        import oracle.cobs_oracle as O
        from workloads import bits_to_f64
        self.O, self.w = O, w
        self.items = []
        nfull = w.seq_len // w.block
        for (b, h) in pairs:
            keys = bits_to_f64(k_bits[b, h])
            vals = bits_to_f64(v_bits[b, h])
            qg = bits_to_f64(q_bits[b, h * w.group:(h + 1) * w.group])
            recs = O.build_block_records(keys, w.block, w.rank, 0, nfull - 1)
            last = O.build_block_records(keys, w.block, w.rank, nfull - 1, nfull)
            self.items.append((qg, keys, vals, recs, last))

    def step(self, i):
        """One decode step of one pair: selection + attention, and the stats of
        the just-completed block on the pair's steps where a block completes
        (every block-th step of the pair), as in the GPU stream."""
        O, w = self.O, self.w
        n = len(self.items)
        qg, keys, vals, recs, last = self.items[i % n]
        nfull = w.seq_len // w.block
        if (i // n) % w.block == w.block - 1:
            last = O.build_block_records(keys, w.block, w.rank, nfull - 1, nfull)
        allrec = np.concatenate([recs, last])
        O.decode_step(qg, keys, vals, allrec, w.seq_len, w.block, w.top_k,
                      w.sink_blocks, w.local_tokens)
        return w.group                               # queries served


def oracle_pairs(w, n):
    pairs = [(b, h) for b in range(w.batch) for h in range(w.kv_heads)]
    step = max(1, len(pairs) // n)
    return pairs[::step][:n]


def oracle_slices(w, pairs):
    """Only the K/V slices the oracle sample needs (drawn per slice)."""
    from workloads import make_kv_slice, make_queries
    q = make_queries(w)
    K = {}
    V = {}
    for (b, h) in pairs:
        K[(b, h)], V[(b, h)] = make_kv_slice(w, b, h, q if w.needles else None)

    class View:
        def __init__(self, d):
            self.d = d

        def __getitem__(self, key):
            return self.d[key]
    return q, View(K), View(V)


_BARRIER = None


def _oracle_pool_init(barrier):
    global _BARRIER
    _BARRIER = barrier


def _oracle_worker(task):
    """One host core: oracle decode steps of its own (batch, kv-head) pairs,
    started together with the other cores (barrier), for a fixed time or a
    fixed number of steps.  Returns (queries served, seconds, steps)."""
    w, pairs, seconds, steps, warmup = task
    from threadpoolctl import threadpool_limits
    q, K, V = oracle_slices(w, pairs)
    with threadpool_limits(1):
        sample = OracleSample(w, q, K, V, pairs)
        for i in range(max(1, warmup)):
            sample.step(i)
        if _BARRIER is not None:
            _BARRIER.wait(timeout=900)
        t0 = time.perf_counter()
        served = i = 0
        while (i < steps) if steps else (time.perf_counter() - t0 < seconds):
            served += sample.step(i)
            i += 1
        dt = time.perf_counter() - t0
    return served, dt, i


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_rate(w, n_workers, seconds=0.0, steps=0, warmup=1):
    """Throughput of the oracle on ``n_workers`` host cores, one process per
    core (spawn-started, one BLAS thread each), every core decoding its own
    (batch, kv-head) pair of the workload; the cores start their timed loops
    together.  Returns (queries/s, steps per core, seconds, pairs used)."""
    pairs_all = oracle_pairs(w, max(1, n_workers))
    tasks = [(w, [pairs_all[i % len(pairs_all)]], seconds, steps, warmup)
             for i in range(n_workers)]
    if n_workers == 1:
        served, dt, n = _oracle_worker(tasks[0])
        return served / dt, n, dt, pairs_all[:1]
    import multiprocessing as mp
    ctx = mp.get_context("spawn")
    barrier = ctx.Barrier(n_workers)
    with ctx.Pool(n_workers, initializer=_oracle_pool_init, initargs=(barrier,)) as pool:
        res = pool.map(_oracle_worker, tasks, chunksize=1)
    served = sum(r[0] for r in res)
    dt = max(r[1] for r in res)
    return served / dt, min(r[2] for r in res), dt, pairs_all


def oracle_cores():
    """Host cores the oracle legs use: every core this process may run on
    (capped at 128 processes, each holding one pair's cache)."""
    return max(1, min(128, host_cores()))


def run_reference(args, w, rank):
    if rank != 0:
        return
    cores = oracle_cores()
    value, n_steps, dt, pairs = oracle_rate(w, cores, steps=args.steps, warmup=args.warmup)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch_per_gpu": w.batch, "q_heads": w.q_heads,
                   "kv_heads": w.kv_heads, "head_dim": w.head_dim, "seq_len": w.seq_len,
                   "block": w.block, "rank": w.rank, "top_k": w.top_k,
                   "sink_blocks": w.sink_blocks, "local_tokens": w.local_tokens,
                   "parallelism": f"replicas x{args.gpus}",
                   "step": ("one decode token of a pair: select + sparse decode, and the "
                            "stats of the completed block on the pair's steps where a block "
                            "completes (every block-th)")},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: every one of {cores} host cores (one process, "
                                   f"one BLAS thread each) decodes one (batch, kv-head) pair "
                                   f"(selection + attention, and the stats of the "
                                   f"completed block every block-th step of a pair, "
                                   f"fp64 numpy); pairs cycle over {len(pairs)} of "
                                   f"{w.batch * w.kv_heads}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def cpu_baseline(w, seconds):
    """The oracle on every host core, with the one-core figure beside it."""
    cores = oracle_cores()
    one, n1, dt1, p1 = oracle_rate(w, 1, seconds=seconds / 2)
    out = {"value": one, "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"{n1} oracle decode steps of (batch, kv-head) pair {p1[0]} of {w.name} "
                     f"(selection + attention, and the stats of the completed block "
                     f"every block-th step of a pair, fp64 numpy, "
                     f"1 thread), {dt1:.1f} s, scaled to queries/s"}
    if cores > 1:
        try:
            allv, n, dt, pairs = oracle_rate(w, cores, seconds=seconds)
            out = {"value": allv, "unit": UNIT, "cores": cores, "kind": "oracle",
                   "sample": f"{cores} host cores at once, one process and one BLAS thread "
                             f"each, every core decoding its own (batch, kv-head) pair of "
                             f"{w.name} ({len(pairs)} distinct pairs; selection + attention, "
                             f"and the stats of the completed block every block-th step of a "
                             f"pair, fp64 numpy), >= {n} steps per "
                             f"core in {dt:.1f} s, scaled to queries/s",
                   "one_core": {"value": one, "cores": 1, "sample": out["sample"]}}
        except Exception as e:            # the one-core figure still stands
            out["all_cores_error"] = f"{type(e).__name__}: {e}"
    return out


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------

def calibrate_subspace(w, s, steps=8):
    """Query-subspace basis of the subspace records, [kv_heads, s, d] fp32:
    per kv-head, the top-s eigenvectors of the uncentred second moment
    (1/n) sum q q^T of calibration queries -- here seeded draws of the
    workload's own query distribution for `steps` decode steps (there is no
    trained model to calibrate on).  An offline set-up step, like loading a
    calibrated basis; it is not part of the timed path."""
    from workloads import bits_to_f64, make_queries
    d, G = w.head_dim, w.group
    qs = np.stack([bits_to_f64(make_queries(w, 1000 + t)) for t in range(steps)])
    out = np.zeros((w.kv_heads, s, d), dtype=np.float32)
    for h in range(w.kv_heads):
        q = qs[:, :, h * G:(h + 1) * G].reshape(-1, d)
        lam, vec = np.linalg.eigh(q.T @ q / q.shape[0])
        out[h] = vec[:, np.argsort(-lam, kind="stable")[:s]].T
    return out


def run_cobs(args, w, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import block_sparse_long_cobs_b200 as cb
    from workloads import make_kv, make_queries

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    workers = args.gen_workers or max(1, min(16, (os.cpu_count() or 2) // max(1, world) - 1))
    q_bits = make_queries(w)
    k_bits, v_bits = make_kv(w, q_bits if w.needles else None, workers=workers)

    def up(x):
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).to(dev)

    fmt = {"bf16": cb.COBS_STATS_BF16, "fp4": cb.COBS_STATS_FP4, "box": cb.COBS_STATS_BOX,
           "subspace": cb.COBS_STATS_SUBSPACE}[args.stats_format]
    dims = dict(batch=w.batch, num_q_heads=w.q_heads, num_kv_heads=w.kv_heads,
                head_dim=w.head_dim, block_size=w.block, rank=w.rank,
                capacity_tokens=w.cap, stats_format=fmt)
    if args.stats_format == "subspace":
        basis = torch.from_numpy(calibrate_subspace(w, args.subspace_dim)).to(dev)
        dims.update(subspace_dim=args.subspace_dim, subspace_basis=basis)
    k, v = up(k_bits), up(v_bits)
    # one device buffer for a step's inputs (the queries, then the appended
    # token's K and V rows) and one for its results (out, then lse), so that
    # the end-to-end step moves each with a single copy
    nq = w.batch * w.q_heads * w.head_dim
    nkv = w.batch * w.kv_heads * w.head_dim
    inputs = torch.empty(nq + 2 * nkv, dtype=torch.int16, device=dev)
    q = inputs[:nq].view(w.batch, w.q_heads, w.head_dim)
    q.copy_(up(q_bits))
    nb_cap = w.cap // w.block
    nfull = w.seq_len // w.block
    rec_bytes = cb.cobs_stats_record_bytes(dims)
    stats = torch.zeros((w.batch, w.kv_heads, nb_cap, rec_bytes), dtype=torch.uint8,
                        device=dev)
    nsm = cb.cobs_selected_capacity(dims, w.top_k, w.sink_blocks, w.local_tokens)
    idx = torch.zeros((w.batch, w.kv_heads, nsm), dtype=torch.int32, device=dev)
    n_sel = torch.zeros((w.batch, w.kv_heads), dtype=torch.int32, device=dev)
    results = torch.zeros(w.batch * w.q_heads * (w.head_dim + 1), dtype=torch.float32, device=dev)
    out = results[:nq].view(w.batch, w.q_heads, w.head_dim)
    lse = results[nq:].view(w.batch, w.q_heads)
    ws_bytes = cb.cobs_workspace_bytes(dims, w.top_k, w.sink_blocks, w.local_tokens)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
    flush_sink = torch.zeros(1, dtype=torch.int32, device=dev)

    def flush():
        # write a buffer of 2x L2, then read another one: the dirty lines the
        # write leaves are written back here, outside the timed step, and the
        # step starts from a cold, clean L2
        flush_w.zero_()
        torch.amax(flush_r, dim=0, keepdim=True, out=flush_sink)
    stream = torch.cuda.current_stream(dev)
    cb.cobs_workspace_init(ws, ws_bytes, stream)
    scale = 1.0 / math.sqrt(w.head_dim)

    # statistics of every earlier complete block (setup, timed for information)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cb.cobs_build_block_stats(dims, k, 0, nfull - 1, stats, ws, ws_bytes, stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    build_ms = e0.elapsed_time(e1)

    # a workload built by appends: the statistics build of one appended chunk
    # (append_chunk / 64 blocks of every (batch, kv-head)), L2 flushed before
    # each of 20 timed builds
    append = None
    if w.append_chunk:
        per = w.append_chunk // w.block
        j0 = max(0, nfull - 1 - per)
        flush_a = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        times = []
        for i in range(23):
            flush_a.zero_()
            e0.record(stream)
            cb.cobs_build_block_stats(dims, k, j0, j0 + per, stats, ws, ws_bytes, stream)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if i >= 3:
                times.append(e0.elapsed_time(e1))
        del flush_a
        t_app = statistics.median(times)
        heads = w.batch * w.kv_heads * per
        append = {"tokens": w.append_chunk, "block_heads": heads, "ms": t_app,
                  "gbs": heads * (w.block * w.head_dim * 2 + rec_bytes) / (t_app * 1e-3) / 1e9,
                  "note": "statistics build of one appended chunk, median of 20 launches "
                          "after an L2 flush"}

    side = torch.cuda.Stream(dev) if args.stats_stream == "side" else None
    fork_ev, join_ev = torch.cuda.Event(), torch.cuda.Event()

    def step(ev=None, st=None, inner=True, one_stream=False, with_stats=True):
        # ev: [step start, selection start, decode start, step end, stats start, stats end];
        # with inner=False only the step's start and end are recorded (an event
        # between two kernels stops the second from starting its prologue early);
        # with_stats=False leaves the statistics build out (a step in which no
        # block completes)
        st = stream if st is None else st
        evo = ev
        ev = ev if inner else None
        if evo is not None:
            evo[0].record(st)
        use_side = side is not None and not one_stream and with_stats
        if not with_stats:
            pass
        elif use_side:
            # the block completed at this step lies in the local window, so the
            # selection below never reads the record being written
            fork_ev.record(st)
            side.wait_event(fork_ev)
            if ev is not None:
                ev[4].record(side)
            cb.cobs_build_block_stats(dims, k, nfull - 1, nfull, stats, ws, ws_bytes, side)
            if ev is not None:
                ev[5].record(side)
            join_ev.record(side)
        else:
            if ev is not None:
                ev[4].record(st)
            cb.cobs_build_block_stats(dims, k, nfull - 1, nfull, stats, ws, ws_bytes, st)
            if ev is not None:
                ev[5].record(st)
        if ev is None:
            # one call: the decode takes each (batch, kv-head) as soon as its
            # selection is written
            cb.cobs_select_and_decode(dims, q, stats, k, v, w.seq_len, w.top_k, w.sink_blocks,
                                      w.local_tokens, scale, idx, nsm, n_sel, None, out, lse,
                                      ws, ws_bytes, st)
        else:
            # the kernels one by one, with events between them
            ev[1].record(st)
            cb.cobs_select_blocks(dims, q, stats, w.seq_len, w.top_k, w.sink_blocks,
                                  w.local_tokens, idx, nsm, n_sel, None, ws, ws_bytes, st)
            ev[2].record(st)
            cb.cobs_sparse_decode(dims, q, k, v, idx, n_sel, nsm, w.seq_len, scale, out, lse,
                                  ws, ws_bytes, st)
        if use_side:
            st.wait_event(join_ev)
        if evo is not None:
            evo[3].record(st)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize(dev)
    status = cb.cobs_read_device_status(ws, ws_bytes, stream)
    if status != 0:
        raise RuntimeError(f"device status {cb.cobs_status_string(status)} after warm-up")
    sel_counts = n_sel.cpu().numpy()
    n_sel_mean = float(sel_counts.mean())
    quality = None
    if w.needles:
        # needle-block recall of the GPU selection (a quality side-metric):
        # planted needle blocks that made it into each (batch, kv-head) list
        from workloads import needle_block_list
        idx_h = idx.cpu().numpy()
        hits = total = 0
        for b in range(w.batch):
            for h in range(w.kv_heads):
                nb = needle_block_list(w, b, h)
                chosen = set(idx_h[b, h, :sel_counts[b, h]].tolist())
                hits += sum(int(j) in chosen for j in nb)
                total += len(nb)
        quality = {"needle_recall": hits / total if total else None,
                   "needle_blocks": total}

    # timed region: the steps are replayed from CUDA graphs of g_steps steps
    # (L2 flush, stats, selection, decode and the per-step events captured),
    # so that host launch overhead stays out of the device timing; without
    # graphs the same steps are enqueued one call at a time
    g_steps = max(d for d in range(1, min(50, args.steps) + 1) if args.steps % d == 0)
    if args.no_graph:
        g_steps = 1
    # external: recorded inside a graph capture as event-record nodes
    def make_events():
        return [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(6)]
                for _ in range(g_steps)]

    def capture(evs, inner, with_stats=True):
        if args.no_graph:
            return None
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            cs = torch.cuda.current_stream(dev)
            for i in range(g_steps):
                flush()
                step(evs[i], cs, inner, one_stream=inner, with_stats=with_stats)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize(dev)
        return g

    def graph_kernel_nodes(g):
        """Kernel nodes of a captured graph (None when they cannot be read)."""
        try:
            from cuda.bindings import driver as cu
            gr = cu.CUgraph(init_value=int(g.raw_cuda_graph()))
            err, _, n = cu.cuGraphGetNodes(gr, 0)
            err, nodes, n = cu.cuGraphGetNodes(gr, n)
            if err != cu.CUresult.CUDA_SUCCESS:
                return None
            kinds = [cu.cuGraphNodeGetType(nd)[1] for nd in nodes[:n]]
            return sum(k == cu.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL for k in kinds)
        except Exception:
            return None

    def run_timed(evs, graph, n_steps, inner, sums, with_stats=True):
        for _ in range(n_steps // g_steps):
            if graph is not None:
                graph.replay()
            else:
                flush()
                step(evs[0], None, inner, one_stream=inner, with_stats=with_stats)
            torch.cuda.synchronize(dev)
            for e in evs:
                sums[3] += e[0].elapsed_time(e[3])
                if inner:
                    sums[0] += e[4].elapsed_time(e[5])
                    sums[1] += e[1].elapsed_time(e[2])
                    sums[2] += e[2].elapsed_time(e[3])

    # (1) the step time: events at step boundaries only; (2) the per-kernel
    # breakdown: the same steps with all three kernels on one stream and events
    # between them (each kernel timed alone), a fifth as many (at least 250)
    # (3) steps in which no block completes: selection + decode only, events at
    # the step boundaries, as many as the breakdown pass
    evs_step, evs_kern, evs_sd = make_events(), make_events(), make_events()
    graph_step = capture(evs_step, False)
    n_kern = max(min(250, args.steps), args.steps // 5) // g_steps * g_steps or g_steps
    graph_kern = capture(evs_kern, True)
    graph_sd = capture(evs_sd, False, with_stats=False)
    # this library's launches per step (with and without a statistics
    # build): the kernel nodes of a captured step less those of a captured L2
    # flush (torch's kernels); graphs kept uninstantiated for reading, never
    # replayed
    launches = None
    if not args.no_graph:
        counts = []
        for with_stats in (False, True, None):
            g_one = torch.cuda.CUDAGraph(keep_graph=True)
            with torch.cuda.graph(g_one):
                flush()
                if with_stats is not None:
                    step(None, torch.cuda.current_stream(dev), False, with_stats=with_stats)
            counts.append(graph_kernel_nodes(g_one))
            del g_one
        if None not in counts:
            launches = (counts[0] - counts[2], counts[1] - counts[2])

    # the decode stream: every step decodes one token of every sequence
    # (selection + sparse decode); a block completes every `block` steps and
    # on that step its statistics are built as well.  The K timed steps hold
    # round(K / block) such steps (the phase chosen to give that count); each
    # step is replayed from a one-step graph and timed by its own events
    per_block = w.block
    phase = min(per_block - 1, max(0, per_block * round(args.steps / per_block) - args.steps))
    is_build = [(i + phase) % per_block == per_block - 1 for i in range(args.steps)]
    builds = sum(is_build)

    def capture_one(ev, with_stats):
        if args.no_graph:
            return None
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            flush()
            step(ev, torch.cuda.current_stream(dev), False, with_stats=with_stats)
        for _ in range(2):
            g.replay()
        torch.cuda.synchronize(dev)
        return g

    ev_plain = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(6)]
    ev_build = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(6)]
    g_plain, g_build = capture_one(ev_plain, False), capture_one(ev_build, True)

    def run_stream():
        total = 0.0
        for i in range(args.steps):
            ev, g = (ev_build, g_build) if is_build[i] else (ev_plain, g_plain)
            if g is not None:
                g.replay()
            else:
                flush()
                step(ev, None, False, with_stats=is_build[i])
            torch.cuda.synchronize(dev)
            total += ev[0].elapsed_time(ev[3])
        return total / args.steps

    sums_step, sums_kern, sums_sd = [0.0] * 4, [0.0] * 4, [0.0] * 4

    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    # keep the GPU busy while nvidia-smi starts up (~0.2 s), so that its
    # samples all fall under load
    t_pre = time.perf_counter()
    while time.perf_counter() - t_pre < 0.3:
        for _ in range(50):
            flush()
            step()
        torch.cuda.synchronize(dev)
    t_host0 = time.perf_counter()
    t_stream = run_stream()
    t_host = (time.perf_counter() - t_host0) * 1e3 / args.steps   # wall time per step
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    run_timed(evs_step, graph_step, n_kern, False, sums_step)
    torch.cuda.synchronize(dev)
    run_timed(evs_kern, graph_kern, n_kern, True, sums_kern)
    torch.cuda.synchronize(dev)
    run_timed(evs_sd, graph_sd, n_kern, False, sums_sd, with_stats=False)
    torch.cuda.synchronize(dev)
    clock_info = clocks.stop()
    t_every = sums_step[3] / n_kern
    t_stats, t_sel, t_dec, t_step_kern = (x / n_kern for x in sums_kern)
    t_sd = sums_sd[3] / n_kern
    status = cb.cobs_read_device_status(ws, ws_bytes, stream)
    if status != 0:
        raise RuntimeError(f"device status {cb.cobs_status_string(status)} after timing")

    # end to end through the public API with host buffers: queries and the
    # appended token's K/V go host -> device, outputs come back
    e2e = None
    if not args.no_e2e:
        # pinned host images of the input and result buffers: the queries and
        # the appended token's K and V rows in, out and lse back
        inputs_host = torch.from_numpy(np.concatenate([
            q_bits.view(np.int16).reshape(-1),
            np.ascontiguousarray(k_bits[:, :, w.seq_len - 1]).view(np.int16).reshape(-1),
            np.ascontiguousarray(v_bits[:, :, w.seq_len - 1]).view(np.int16).reshape(-1)]))
        inputs_host = inputs_host.pin_memory()
        results_host = torch.empty(results.shape, dtype=results.dtype).pin_memory()
        kn_dev = inputs[nq:nq + nkv].view(w.batch, w.kv_heads, w.head_dim)
        vn_dev = inputs[nq + nkv:].view(w.batch, w.kv_heads, w.head_dim)
        h2d = inputs_host.numel() * 2
        d2h = results_host.numel() * 4
        def e2e_step(pair, st=None, with_stats=True):
            # torch copies go to the current stream: the capture stream inside
            # a graph capture, `stream` otherwise
            st = stream if st is None else st
            pair[0].record(st)
            inputs.copy_(inputs_host, non_blocking=True)
            k[:, :, w.seq_len - 1].copy_(kn_dev)
            v[:, :, w.seq_len - 1].copy_(vn_dev)
            step(None, st, with_stats=with_stats)
            results_host.copy_(results, non_blocking=True)
            pair[1].record(st)

        def time_e2e(use_graph):
            # the same stream of K steps as the device timing: a statistics
            # build on the steps where a block completes
            evp = (torch.cuda.Event(enable_timing=True, external=use_graph),
                   torch.cuda.Event(enable_timing=True, external=use_graph))
            evb = (torch.cuda.Event(enable_timing=True, external=use_graph),
                   torch.cuda.Event(enable_timing=True, external=use_graph))
            graphs = {}
            if use_graph:
                for with_stats, ev in ((False, evp), (True, evb)):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g):
                        flush()
                        e2e_step(ev, torch.cuda.current_stream(dev), with_stats)
                    graphs[with_stats] = g
            for i in range(3):
                if use_graph:
                    graphs[i == 2].replay()
                else:
                    flush()
                    e2e_step(evb if i == 2 else evp, None, i == 2)
            torch.cuda.synchronize(dev)
            total = 0.0
            for i in range(args.steps):
                ev = evb if is_build[i] else evp
                if use_graph:
                    graphs[is_build[i]].replay()
                else:
                    flush()
                    e2e_step(ev, None, is_build[i])
                torch.cuda.synchronize(dev)
                total += ev[0].elapsed_time(ev[1])
            return total / args.steps

        # the public-API calls and the per-step copies, replayed as CUDA
        # graphs (as a decode server drives them); and the same calls made one
        # by one from Python, which adds the host's call overhead
        t_e2e = time_e2e(not args.no_graph)
        t_eager = time_e2e(False)
        t_e2e, t_eager = max_over_ranks([t_e2e, t_eager], dist, dev, world)
        e2e = {"value": world * w.batch * w.q_heads / (t_e2e * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": t_e2e,
               "launch": "one-step CUDA graphs of the API calls and copies" if not args.no_graph
                         else "one call at a time",
               "eager": {"value": world * w.batch * w.q_heads / (t_eager * 1e-3),
                         "ms_per_step": t_eager,
                         "launch": "one call at a time from Python"}}

    t_stream, t_every, t_stats, t_sel, t_dec, t_sd = max_over_ranks(
        [t_stream, t_every, t_stats, t_sel, t_dec, t_sd], dist, dev, world)
    if rank != 0:
        return

    hbm, peak_kind = peaks()
    bm = byte_model(w, round(n_sel_mean), rec_bytes)
    traffic_key = w.name if args.stats_format == "bf16" else f"{w.name}:{args.stats_format}"
    per_kernel = {"stats": (t_stats, bm["stats"],
                            "box.cu" if args.stats_format == "box" else "stats.cu"),
                  "select": (t_sel, bm["select"], "select.cu"),
                  "decode": (t_dec, bm["decode"],
                             "decode_tc.cu" if w.head_dim == 128 else "decode.cu")}
    kernels = {name: {"ms": t, "bytes": b, "gbs": b / (t * 1e-3) / 1e9,
                      "frac_of_hbm": b / (t * 1e-3) / 1e9 / hbm}
               for name, (t, b, _) in per_kernel.items()}
    # the kernel with the largest share of the average stream step: the stats
    # build runs on `builds` of the K steps (and off the critical path when it
    # overlaps on the side stream)
    weight = {"stats": builds / args.steps, "select": 1.0, "decode": 1.0}
    on_path = dict(per_kernel)
    if args.stats_stream == "side" and t_stats < t_sel + t_dec:
        on_path.pop("stats")
    dom = max(on_path, key=lambda n: on_path[n][0] * weight[n])
    t_dom, b_dom, file_dom = per_kernel[dom]
    achieved = b_dom / (t_dom * 1e-3) / 1e9
    # bytes of an average stream step: selection and decode every step, the
    # statistics build on `builds` of the K steps
    step_bytes = bm["select"] + bm["decode"] + bm["stats"] * builds / args.steps
    value = world * w.batch * w.q_heads / (t_stream * 1e-3)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_stream,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch_per_gpu": w.batch, "q_heads": w.q_heads,
                   "kv_heads": w.kv_heads, "head_dim": w.head_dim, "seq_len": w.seq_len,
                   "block": w.block, "rank": w.rank, "top_k": w.top_k,
                   "sink_blocks": w.sink_blocks, "local_tokens": w.local_tokens,
                   "selected_blocks_mean": n_sel_mean, "l2": "flushed between steps: 256 MiB written, then 256 MiB read",
                   "parallelism": f"replicas x{world}",
                   "step": (f"one decode token of every sequence: select + sparse decode, "
                            f"and the stats of the completed block on the steps where a "
                            f"block completes (every {per_block}th)"),
                   "blocks_completed_in_timed_steps": builds,
                   "stats_stream": args.stats_stream,
                   "stats_format": args.stats_format, "record_bytes": rec_bytes,
                   **({"subspace_dim": args.subspace_dim}
                      if args.stats_format == "subspace" else {}),
                   "launch": ("one-step CUDA graphs, one replay per step" if g_plain is not None
                              else "one call at a time")},
        "hbm_gbs_step": step_bytes / (t_stream * 1e-3) / 1e9,
        "hbm_frac_step": step_bytes / (t_stream * 1e-3) / 1e9 / hbm,
        "kernels": kernels,
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm,
                     "unit": "GB/s", "frac": achieved / hbm,
                     "peak_kind": f"{peak_kind} copy bandwidth",
                     "traffic": recorded_traffic(file_dom, traffic_key)},
        "gpu_launches": ((args.steps - builds) * launches[0] + builds * launches[1]
                         if launches is not None else 2 * args.steps + builds),
        "gpu_launches_counted": ("kernel nodes of the captured one-step graphs (with and "
                                 "without the statistics build), less the L2 flush's"
                                 if launches is not None else
                                 "2 per step (select, decode) and 1 per build, not read "
                                 "from a graph"),
        "clocks": clock_info,
        "setup_stats_build_ms": build_ms,
        **({"append_chunk_build": append} if append is not None else {}),
        "wall_ms_per_step": t_host,
        "quality": quality,
        "step_variants": {
            "stats_every_step": {
                "ms_per_step": t_every, "value": world * w.batch * w.q_heads / (t_every * 1e-3),
                "hbm_frac": (bm["select"] + bm["decode"] + bm["stats"]) / (t_every * 1e-3) / 1e9
                            / hbm,
                "note": "every step also builds the statistics of one block per (batch, "
                        f"kv-head) ({n_kern} graph-replayed steps, events at step boundaries)"},
            "select_decode": {
                "ms_per_step": t_sd, "value": world * w.batch * w.q_heads / (t_sd * 1e-3),
                "hbm_frac": (bm["select"] + bm["decode"]) / (t_sd * 1e-3) / 1e9 / hbm,
                "note": "a step in which no block completes: selection + decode only "
                        f"({n_kern} graph-replayed steps, events at step boundaries)"},
            "amortised": {
                "ms_per_step": t_sd + t_stats / w.block,
                "value": world * w.batch * w.q_heads / ((t_sd + t_stats / w.block) * 1e-3),
                "note": f"one decode token per sequence per step completes a block every "
                        f"{w.block} steps: the select + decode step plus 1/{w.block} of the "
                        f"statistics build timed alone"}},
        "kernel_breakdown": {"steps": n_kern, "ms_per_step": t_step_kern,
                             "note": "per-kernel times from a second graph-replayed run, "
                                     "the three kernels on one stream with events between "
                                     "them"},
    }
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.batch:
        w = w.scaled(batch=args.batch)
    if args.impl == "reference":
        run_reference(args, w, rank)
        return
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    w = rank_shard(w, rank)
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_cobs(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
