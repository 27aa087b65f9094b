#!/usr/bin/env python
"""TempCache benchmark: frames/s of the Wan-2.1-1.3B-shaped attention layer.

A step is one full rollout of the workload from an empty cache: 40 chunks of 3
frames (4680 tokens, 12 heads, d = 128, bf16), each chunk one tc_append_chunk
(commit of the previous chunk: append and merge; staging of this one: copy, hash,
bucket search and merge decisions) followed by 4 tc_attend calls. value = frames processed by all ranks / the
slowest rank's device time. Inputs are generated before timing and stay resident
in HBM (3.5 GB of distinct K, V, Q per rollout, far larger than the 126 MB L2).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
  python bench.py --workload annca-wan1.3b     (AnnCA cross-attention, its own line)
  python bench.py --workload annsa-wan1.3b     (AnnSA same-bucket self-attention, its own line)
  python bench.py --workload lvsa-wan1.3b      (LVSA frame-masked attention, its own line)
  python bench.py --key-mode mean              (running-mean keys, its own line)

N > 1 runs under torchrun: each rank runs an independent rollout (its own seed);
there is no collective in the data path, only the max-over-ranks of the timing.
--impl reference times the CPU oracle (fp64 NumPy) on the host instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from synthetic import CONFIGS, CROSS_CONFIGS  # noqa: E402

WORKLOAD = "wan1.3b"
METRIC = "TempCache frames/s (merge+4x attend) at Wan-1.3B shape; attn TFLOP/s vs peak"
UNIT = "frames/s"
MEASURED_PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "attend_bf16_duo_wan1.3b_traffic.json")
ATTN_KERNEL = "attend_bf16_duo_kernel"   # the attention kernel the bf16 path launches
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- plumbing

def dist_info():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def init_dist(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))


def max_over_ranks(x: float, world: int, device) -> float:
    """Largest value of x over all ranks (the step time of the slowest GPU)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units of every rank over the slowest rank's time."""
    return units_per_rank * world / max_seconds


def rank_seed(base: int, rank: int) -> int:
    return base + 7919 * rank


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


def load_peaks():
    if os.path.exists(MEASURED_PEAKS):
        with open(MEASURED_PEAKS) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append((float(p[1]), float(p[2]), p[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, fl in rows for i, v in enumerate(fl) if v.lower() == "active"})
        sm = [r[0] for r in rows]
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------- workload

def generate_inputs(cfg, device, seed):
    from synthetic import Workload

    w = Workload(cfg.replace(seed=seed), device=device)
    chunks = []
    for c in range(cfg.chunks):
        K, V = w.next_chunk()
        Qs = [w.queries(c, a) for a in range(cfg.attends)]
        chunks.append((K, V, Qs))
    return w.hyperplanes().numpy(), chunks


def rollout(tc, chunks, outs, events=None):
    """One rollout from an empty cache. events[c] = (e0, e1, e2) brackets the append
    (e0..e1) and the block of attention calls (e1..e2) of chunk c; no event sits
    between two attention calls, so consecutive calls may overlap on the device."""
    tc.reset()
    for c, (K, V, Qs) in enumerate(chunks):
        if events is not None:
            events[c][0].record()
        tc.append_chunk(K, V)
        if events is not None:
            events[c][1].record()
        for a, Q in enumerate(Qs):
            tc.attend(Q, out=outs[a])
        if events is not None:
            events[c][2].record()


def sizes_per_chunk(tc, chunks, outs, cfg):
    """Committed entries per head seen by the attends of each chunk, and per append call
    the counts its algorithmic bytes depend on: tokens appended, tokens merged and
    entries touched by the commit it runs (of the previous chunk), and the candidates
    the staging search of this chunk visits (the committed entries in each staged
    token's bucket, counted here from the exported codes)."""
    tc.reset()
    sizes, commit = [], []
    for K, V, Qs in chunks:
        tc.append_chunk(K, V)
        sizes.append(tc.cache_size().copy())
        _, match, _ = tc.last_commit()
        staged = tc.staged_codes()
        cand = 0
        for h in range(cfg.H):
            codes = tc.export_cache(h)[3]
            if codes.size:
                u, n = np.unique(codes, return_counts=True)
                pos = np.clip(np.searchsorted(u, staged[h]), 0, u.size - 1)
                cand += int(np.where(u[pos] == staged[h], n[pos], 0).sum())
        if match.size:
            touched = sum(len(np.unique(match[h][match[h] >= 0])) for h in range(cfg.H))
            commit.append((int((match < 0).sum()), int((match >= 0).sum()), touched, match.shape[1], cand))
        else:
            commit.append((0, 0, 0, 0, cand))
        for a, Q in enumerate(Qs):
            tc.attend(Q, out=outs[a])
    return sizes, commit


def attn_flops(cfg, sizes):
    """4 * Tq * (M_h + T) * d summed over heads, for every attend of the rollout."""
    per_chunk = [4.0 * cfg.T * float((s + cfg.T).sum()) * cfg.d for s in sizes]
    return per_chunk  # one attend call of chunk c


def commit_bytes(cfg, commit_counts, b=2):
    """Algorithmic bytes of each tc_append_chunk call, which commits the previous chunk
    and stages this one:
      staging   read K and V, write the head-major copies: 4 T H d b; per token its code,
                decision and bucket head: 12 T H;
      search    per candidate visited, its key row, |k|^2, next link and span: d b + 13;
                per merged token its merge-list link: 8;
      append    per new entry: read the staged K and V rows, write K, V and the fp32 V
                mean: 4 d b + 4 d; its scalars (n, log2 n, code, |k|^2, span, list
                links): 29;
      merge     per merged token its staged V row and list link: d b + 4; per touched
                entry the fp32 mean read and written, the storage copy written and its
                scalars: 8 d + d b + 12;
      exports   per committed token its code, target and entry index: 12 (the commit's
                reads of the staged codes and decisions: 8)."""
    T, H, d = cfg.T, cfg.H, cfg.d
    total = []
    for u, m, e, Tc, cand in commit_counts:
        stage = 4 * T * H * d * b + 12 * T * H
        search = cand * (d * b + 13) + 8 * m
        append = u * (4 * d * b + 4 * d + 29)
        merge = m * (d * b + 4) + e * (8 * d + d * b + 12)
        exports = 20 * Tc * H
        total.append(stage + search + append + merge + exports)
    return total


# ----------------------------------------------------------------------------- CPU oracle leg

def oracle_rollout(cfg, R, chunks, heads, rows_per_call, seed=0):
    """Time the CPU oracle over one whole rollout, on a subset of the heads.

    Heads are independent, so the oracle follows `heads` through every chunk: each
    chunk's full merge path (hash, bucket search, merge, append) is timed, and one of the
    chunk's attention calls on `rows_per_call` sampled query rows, its time scaled to all
    rows and all calls. The sum is scaled to all H heads. Inputs are converted to fp64
    outside the timed sections. Returns (frames/s, description).
    """
    from oracle import OracleTempCache

    f = lambda x: x[:, heads].to(torch.float64).cpu().numpy()  # noqa: E731
    o = OracleTempCache(len(heads), cfg.d, cfg.nbits, cfg.tau, cfg.capacity, R.astype(np.float64))
    rng = np.random.default_rng(seed)
    t_merge = t_attn = 0.0
    for K, V, Qs in chunks:
        k, v = f(K), f(V)
        t0 = time.perf_counter()
        o.append_chunk(k, v)
        t_merge += time.perf_counter() - t0
        rows = np.sort(rng.choice(cfg.T, size=min(rows_per_call, cfg.T), replace=False))
        q = Qs[0][torch.as_tensor(rows, device=Qs[0].device)][:, heads].to(torch.float64).cpu().numpy()
        t1 = time.perf_counter()
        o.attend(q)
        t_attn += (time.perf_counter() - t1) * (cfg.T / len(rows)) * cfg.attends
    total = (t_merge + t_attn) * cfg.H / len(heads)
    desc = (f"one whole {cfg.name} rollout ({len(chunks)} chunks) on heads {list(heads)} of {cfg.H}, scaled to all "
            f"heads: full oracle merge path every chunk; attention timed on {rows_per_call} of {cfg.T} query rows "
            f"of one call per chunk, scaled to all rows and {cfg.attends} calls")
    return cfg.F * len(chunks) / total, desc


def describe(cfg) -> str:
    return (f"{cfg.name}: H={cfg.H} d={cfg.d} P={cfg.P} F={cfg.F} chunks={cfg.chunks} attends={cfg.attends} "
            f"S={cfg.S} p_stay={cfg.p_stay} sigma={cfg.sigma} nbits={cfg.nbits} tau={cfg.tau} {cfg.dtype}")


def run_reference(args):
    rank, world, _ = dist_info()
    if rank != 0:
        return
    cfg = CONFIGS[WORKLOAD]
    R, chunks = generate_inputs(cfg, "cpu", cfg.seed)
    for _ in range(args.warmup):
        oracle_rollout(cfg, R, chunks, [0], 32)
    t = 0.0
    for k in range(args.steps):   # each step: the whole rollout on one head, scaled to all 12
        value_k, desc = oracle_rollout(cfg, R, chunks, [k % cfg.H], 32, seed=k)
        t += cfg.F * cfg.chunks / value_k
    value = cfg.F * cfg.chunks * args.steps / t
    cores = len(os.sched_getaffinity(0))
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(cfg),
                   "step": f"one {cfg.chunks}-chunk rollout ({cfg.F * cfg.chunks} frames) from an empty cache, "
                           "timed on one head (head k mod 12 at step k) and scaled to all heads"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU leg

def time_e2e(tc, cfg, chunks, steps=1):
    """Frames/s through the public API with inputs in pinned host memory: each chunk's
    K, V and Q are copied in and every attention output is read back inside the
    timed region. The API copies host tensors on its side streams, so one chunk's
    transfers overlap another's kernels; the H2D stream waits for the start event and
    the end event waits for both side streams."""
    from kv_cache_attention_tempcache_b200 import host_copy_streams, join_host_copies

    host = [(K.cpu().pin_memory(), V.cpu().pin_memory(), [Q.cpu().pin_memory() for Q in Qs])
            for K, V, Qs in chunks]
    outs_host = [torch.empty(cfg.T, cfg.H, cfg.d, dtype=torch.bfloat16).pin_memory() for _ in range(cfg.attends)]
    h2d, _ = host_copy_streams()

    def one():
        tc.reset()
        for K, V, Qs in host:
            tc.append_chunk(K, V)
            for a, Q in enumerate(Qs):
                tc.attend(Q, out=outs_host[a])

    one()
    join_host_copies()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    h2d.wait_event(e0)
    for _ in range(steps):
        one()
    join_host_copies()
    e1.record()
    torch.cuda.synchronize()
    sec = e0.elapsed_time(e1) / 1000.0 / steps
    per = cfg.T * cfg.H * cfg.d * 2
    h2d = cfg.chunks * (2 + cfg.attends) * per
    d2h = cfg.chunks * cfg.attends * per
    del host
    return sec, h2d, d2h


def run_gpu(args):
    from kv_cache_attention_tempcache_b200 import TempCache

    rank, world, local = dist_info()
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    cfg = CONFIGS[args.workload]
    headline = (args.workload == WORKLOAD and not args.profile and not args.intra_chunk
                and args.key_mode == "representative")
    if args.chunks:
        cfg = cfg.replace(chunks=args.chunks, capacity=min(cfg.capacity, args.chunks * cfg.T))
    R, chunks = generate_inputs(cfg, dev, rank_seed(cfg.seed, rank))
    input_gb = cfg.chunks * cfg.T * cfg.H * cfg.d * 2 * (2 + cfg.attends) / 1e9
    tc = TempCache(cfg.H, cfg.d, cfg.nbits, cfg.tau, cfg.capacity, hyperplanes=R, intra_chunk=args.intra_chunk,
                   key_mode=args.key_mode)
    outs = [torch.empty(cfg.T, cfg.H, cfg.d, dtype=torch.bfloat16, device=dev) for _ in range(cfg.attends)]

    sizes, commit_counts = sizes_per_chunk(tc, chunks, outs, cfg)
    for _ in range(args.warmup):
        rollout(tc, chunks, outs)
    torch.cuda.synchronize()

    # timed region: K rollouts, per-call events for the attention and commit kernels
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    chunk_ev = [[(ev(), ev(), ev()) for _ in range(cfg.chunks)] for _ in range(args.steps)]
    launches0 = tc.launch_count()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = ev(), ev()
    torch.cuda.nvtx.range_push("timed")
    t0.record()
    for k in range(args.steps):
        rollout(tc, chunks, outs, chunk_ev[k])
    t1.record()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    launches = tc.launch_count() - launches0
    sec = t0.elapsed_time(t1) / 1000.0
    sec_max = max_over_ranks(sec, world, dev)
    value = aggregate_rate(cfg.F * cfg.chunks * args.steps, world, sec_max)

    # roofline of the dominant kernel (attention) from the live per-launch events
    flops_per_call = attn_flops(cfg, sizes)
    attn_sec = sum(chunk_ev[k][c][1].elapsed_time(chunk_ev[k][c][2]) for k in range(args.steps)
                   for c in range(cfg.chunks)) / 1000.0
    attn_flops_total = args.steps * cfg.attends * sum(flops_per_call)
    attn_tflops = attn_flops_total / attn_sec / 1e12
    app_sec = sum(chunk_ev[k][c][0].elapsed_time(chunk_ev[k][c][1]) for k in range(args.steps)
                  for c in range(cfg.chunks)) / 1000.0
    cbytes = args.steps * sum(commit_bytes(cfg, commit_counts))
    peaks, peak_kind = load_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    traffic = traffic_earlier = None
    if os.path.exists(TRAFFIC_FILE):
        with open(TRAFFIC_FILE) as f:
            tr = json.load(f)
        # DRAM bytes per unit of work measured by ncu, scaled to an average launch here
        per_launch = tr.get("bytes_per_flop", 0) * (attn_flops_total / (args.steps * cfg.chunks * cfg.attends))
        if tr.get("kernel") == ATTN_KERNEL:
            if tr.get("current", True):
                traffic = per_launch
            else:   # counters of an earlier build of the kernel: context only
                traffic_earlier = per_launch

    # dense baseline: the same attention kernel over the uncompressed history (no merges)
    dense_line = None
    if headline:
        dense = TempCache(cfg.H, cfg.d, cfg.nbits, 2.0, cfg.capacity, hyperplanes=R)
        rollout(dense, chunks, outs)
        torch.cuda.synchronize()
        d0, d1 = ev(), ev()
        d0.record()
        rollout(dense, chunks, outs)
        d1.record()
        torch.cuda.synchronize()
        dense_sec = d0.elapsed_time(d1) / 1000.0
        dense_flops = cfg.attends * sum(4.0 * cfg.T * cfg.H * (c * cfg.T + cfg.T) * cfg.d
                                        for c in range(cfg.chunks))
        dense.close()
        dense_line = {"value": cfg.F * cfg.chunks / dense_sec, "unit": UNIT,
                      "attn_tflops": dense_flops / dense_sec / 1e12,
                      "note": "same kernels, tau > 1 so nothing merges (uncompressed cache)"}

    e2e = None
    if headline:
        e2e_sec, h2d, d2h = time_e2e(tc, cfg, chunks)
        e2e_value = aggregate_rate(cfg.F * cfg.chunks, world, max_over_ranks(e2e_sec, world, dev))
        e2e = {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    if rank != 0:
        return
    cores = len(os.sched_getaffinity(0))
    cpu = None
    if world == 1 and not args.no_cpu_baseline and headline:
        v, desc = oracle_rollout(cfg, R, chunks, [0, cfg.H // 2], 32)
        cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * sec_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": describe(cfg),
                   "step": f"one {cfg.chunks}-chunk rollout ({cfg.F * cfg.chunks} frames) from an empty cache",
                   "l2": f"inputs larger than L2 ({input_gb:.1f} GB of distinct K, V, Q per rollout)",
                   "parallelism": f"independent rollout per rank x{world}",
                   "commit": "matches inside the chunk too" if args.intra_chunk else "snapshot of earlier commits",
                   "keys": "running means of the members' keys" if args.key_mode == "mean"
                           else "the key that created the entry"},
        "roofline": {"bound": "tensor", "kernel": ATTN_KERNEL, "achieved": attn_tflops,
                     "peak": peak, "unit": "TFLOP/s", "frac": attn_tflops / peak,
                     "peak_kind": f"{peak_kind} bf16 dense, sustained", "traffic": traffic,
                     "traffic_earlier_build": traffic_earlier,
                     "flops_per_launch": attn_flops_total / (args.steps * cfg.chunks * cfg.attends),
                     "avg_launch_ms": 1000.0 * attn_sec / (args.steps * cfg.chunks * cfg.attends)},
        "merge": {"kernels": "stage_search_kernel (copy, hash, bucket search) + commit_kernel (append, merge)"
                             + (" + rebucket kernels" if args.key_mode == "mean" else ""),
                  "achieved_gbs": cbytes / app_sec / 1e9, "peak_gbs": float(peaks["hbm_gbs"]),
                  "frac": cbytes / app_sec / 1e9 / float(peaks["hbm_gbs"]),
                  "bytes_per_chunk": cbytes / (args.steps * cfg.chunks),
                  "avg_append_ms": 1000.0 * app_sec / (args.steps * cfg.chunks)},
        "attn_share": attn_sec / sec,
        "dense_baseline": dense_line,
        "cache_entries_per_head_end": float(np.mean(sizes[-1])),
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
    }
    if args.profile:   # per-call FLOPs of each chunk's attends, to pair with an ncu capture
        line["flops_per_chunk"] = flops_per_call
    if args.series:    # per-chunk device time (mean over the timed rollouts)
        line["series"] = {
            "append_ms": [float(np.mean([chunk_ev[k][c][0].elapsed_time(chunk_ev[k][c][1]) for k in range(args.steps)]))
                          for c in range(cfg.chunks)],
            "attend4_ms": [float(np.mean([chunk_ev[k][c][1].elapsed_time(chunk_ev[k][c][2]) for k in range(args.steps)]))
                           for c in range(cfg.chunks)],
            "entries_per_head": [float(np.mean(sz)) for sz in sizes]}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- AnnCA leg

ANNCA_METRIC = "AnnCA cross-attention frames/s at Wan-1.3B shape (512 prompt tokens)"


def annca_bytes(cfg, kept):
    """Algorithmic HBM bytes of one tc_annca_attend: the queries read twice (hash, then
    attention: the kept set of a frame needs all its queries first), the output written
    once, the query codes written, and every kept key and value row read by the packing
    kernel, written packed and read by the attention kernel."""
    q = cfg.T * cfg.H * cfg.d * 2
    return 2 * q + q + cfg.T * cfg.H * 4 + 3 * kept * cfg.d * 2 * 2


def run_annca(args):
    from kv_cache_attention_tempcache_b200 import AnnCA
    from synthetic import CrossWorkload

    rank, world, local = dist_info()
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    cfg = CROSS_CONFIGS[args.workload]
    cfg = cfg.replace(seed=rank_seed(cfg.seed, rank))
    calls = 40   # one rollout's worth of query blocks (120 frames), 0.6 GB: larger than L2
    w = CrossWorkload(cfg, device=dev)
    R = w.hyperplanes().numpy()
    Kp, Vp = w.prompt()
    Qs = [w.queries(c) for c in range(calls)]
    outs = [torch.empty_like(Qs[0]) for _ in range(2)]
    ann = AnnCA(cfg.H, cfg.d, cfg.nbits, hyperplanes=R)
    ann.set_prompt(Kp, Vp)
    kept = []
    for c in range(calls):
        ann.attend(Qs[c], cfg.P, out=outs[0])
        kept.append(int(ann.kept()[0].sum()))

    def step():
        for c in range(calls):
            ann.attend(Qs[c], cfg.P, out=outs[c & 1])

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = ev(), ev()
    t0.record()
    for _ in range(args.steps):
        step()
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    sec = t0.elapsed_time(t1) / 1000.0
    sec_max = max_over_ranks(sec, world, dev)
    value = aggregate_rate(cfg.F * calls * args.steps, world, sec_max)
    call_sec = sec / (args.steps * calls)
    nbytes = float(np.mean([annca_bytes(cfg, k) for k in kept]))
    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])

    # every prompt token kept (1-bit hash, both buckets present): the same kernels
    # over the whole prompt
    dense = AnnCA(cfg.H, cfg.d, 1, hyperplanes=R[:1])
    dense.set_prompt(Kp, Vp)
    for c in range(calls):
        dense.attend(Qs[c], cfg.P, out=outs[c & 1])
    dense_kept = dense.kept()[0].mean()
    torch.cuda.synchronize()
    d0, d1 = ev(), ev()
    d0.record()
    for c in range(calls):
        dense.attend(Qs[c], cfg.P, out=outs[c & 1])
    d1.record()
    torch.cuda.synchronize()
    dense_sec = d0.elapsed_time(d1) / 1000.0
    dense.close()

    # end to end: queries from pinned host memory, outputs read back, per call
    from kv_cache_attention_tempcache_b200 import host_copy_streams, join_host_copies
    h2d, _ = host_copy_streams()
    host_q = [q.cpu().pin_memory() for q in Qs]
    host_o = torch.empty(cfg.T, cfg.H, cfg.d, dtype=torch.bfloat16).pin_memory()
    e0, e1 = ev(), ev()
    e0.record()
    h2d.wait_event(e0)   # (no copy before the start)
    for c in range(calls):
        ann.attend(host_q[c], cfg.P, out=host_o)
    join_host_copies()
    e1.record()
    torch.cuda.synchronize()
    e2e_sec = max_over_ranks(e0.elapsed_time(e1) / 1000.0, world, dev)
    qb = cfg.T * cfg.H * cfg.d * 2

    if rank != 0:
        ann.close()
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        from oracle import annca_cross_attention
        f = lambda x: x.to(torch.float64).cpu().numpy()  # noqa: E731
        Kn, Vn, Qn = f(Kp), f(Vp), f(Qs[0])
        t = time.perf_counter()
        annca_cross_attention(Qn, Kn, Vn, R.astype(np.float64), cfg.P)
        tcpu = time.perf_counter() - t
        cpu = {"value": cfg.F / tcpu, "unit": UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
               "sample": "one query block (3 frames x 1560 tokens, 12 heads) in full"}
    line = {
        "metric": ANNCA_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * sec_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": (f"{cfg.name}: H={cfg.H} d={cfg.d} P={cfg.P} F={cfg.F} L={cfg.L} C={cfg.C} "
                                f"A={cfg.A} sigma={cfg.sigma} nbits={cfg.nbits} bf16"),
                   "step": f"{calls} tc_annca_attend calls ({cfg.F * calls} frames), prompt set once before",
                   "l2": f"inputs larger than L2 ({calls * qb / 1e9:.2f} GB of distinct queries per step)",
                   "parallelism": f"independent layer per rank x{world}"},
        "roofline": {"bound": "hbm", "kernel": "annca_mark_kernel + annca_pack_kernel + attend_bf16_duo_kernel "
                                                "(cross), one call",
                     "achieved": nbytes / call_sec / 1e9, "peak": hbm, "unit": "GB/s",
                     "frac": nbytes / call_sec / 1e9 / hbm, "peak_kind": f"{peak_kind} copy bandwidth",
                     "traffic": None, "bytes_per_call": nbytes, "avg_call_us": 1e6 * call_sec},
        "kept_fraction": float(np.mean(kept)) / (cfg.H * cfg.F * cfg.L),
        "dense_baseline": {"value": cfg.F * calls / dense_sec, "unit": UNIT, "kept_fraction": float(dense_kept),
                           "note": "same kernels with a 1-bit hash: every prompt token kept"},
        "cpu_baseline": cpu,
        "e2e": {"value": aggregate_rate(cfg.F * calls, world, e2e_sec), "unit": UNIT,
                "h2d_bytes_per_step": calls * qb, "d2h_bytes_per_step": calls * qb},
        "gpu_launches": 3 * calls * args.steps,
        "clocks": clk,
    }
    ann.close()
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- AnnSA leg

ANNSA_METRIC = "AnnSA same-bucket self-attention frames/s at Wan-1.3B shape (AnnCA buckets)"


def run_annsa(args):
    from kv_cache_attention_tempcache_b200 import AnnCA, TempCache
    from synthetic import CrossWorkload

    rank, world, local = dist_info()
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    cfg = CROSS_CONFIGS["annca-wan1.3b"]
    cfg = cfg.replace(seed=rank_seed(cfg.seed, rank))
    calls = 40   # 120 frames; 1.7 GB of distinct Q, K, V per step: larger than L2
    w = CrossWorkload(cfg, device=dev)
    R = w.hyperplanes().numpy()
    Kp, Vp = w.prompt()
    Qc = [w.queries(c) for c in range(calls)]
    QKV = [w.self_qkv(c) for c in range(calls)]
    out = torch.empty_like(Qc[0])
    xout = torch.empty_like(Qc[0])
    ann = AnnCA(cfg.H, cfg.d, cfg.nbits, hyperplanes=R)
    ann.set_prompt(Kp, Vp)
    flops = []
    for c in range(calls):   # the algorithmic work: 4 n^2 d per bucket of n tokens, every head
        ann.attend(Qc[c], cfg.P, out=xout)
        _, qcodes, _ = ann.kept()
        flops.append(sum(4.0 * float((np.unique(qcodes[h], return_counts=True)[1].astype(np.float64) ** 2).sum())
                         * cfg.d for h in range(cfg.H)))
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    marks = [[(ev(), ev()) for _ in range(calls)] for _ in range(args.steps)]

    def step(k=None):
        for c in range(calls):
            ann.attend(Qc[c], cfg.P, out=xout)   # the buckets of block c (not timed below)
            if k is not None:
                marks[k][c][0].record()
            ann.self_attend(*QKV[c], out=out)
            if k is not None:
                marks[k][c][1].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    for k in range(args.steps):
        step(k)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    sec = sum(a.elapsed_time(b) for row in marks for a, b in row) / 1000.0
    sec_max = max_over_ranks(sec, world, dev)
    value = aggregate_rate(cfg.F * calls * args.steps, world, sec_max)
    call_sec = sec / (args.steps * calls)
    tflops = args.steps * sum(flops) / sec / 1e12
    peaks, peak_kind = load_peaks()
    peak = float(peaks.get("bf16_tflops", 1590.0))

    # dense baseline: the same attention kernel over the whole block (a TempCache whose
    # only content is the block, staged)
    dense = TempCache(cfg.H, cfg.d, 16, 2.0, cfg.T, hyperplanes=np.zeros((16, cfg.d), np.float32))
    d0, d1 = ev(), ev()
    dense_sec = 0.0
    for c in range(calls):
        Q, K, V = QKV[c]
        dense.reset()
        dense.append_chunk(K, V)
        d0.record()
        dense.attend(Q, out=out)
        d1.record()
        torch.cuda.synchronize()
        dense_sec += d0.elapsed_time(d1) / 1000.0
    dense.close()

    # end to end: Q, K, V from pinned host memory and the output read back, per call (the
    # AnnCA call that finds the buckets stays outside the events)
    hq = [tuple(x.cpu().pin_memory() for x in qkv) for qkv in QKV[:8]]
    ho = torch.empty(cfg.T, cfg.H, cfg.d, dtype=torch.bfloat16).pin_memory()
    from kv_cache_attention_tempcache_b200 import host_copy_streams, join_host_copies
    h2d, _ = host_copy_streams()
    for c in range(8):   # warm-up: the allocator's device blocks for host inputs
        ann.attend(Qc[c], cfg.P, out=xout)
        ann.self_attend(*hq[c], out=ho)
    join_host_copies()
    torch.cuda.synchronize()
    e2e_sec = 0.0
    for c in range(8):
        ann.attend(Qc[c], cfg.P, out=xout)
        a0, a1 = ev(), ev()
        a0.record()
        h2d.wait_event(a0)   # (no copy before the start)
        ann.self_attend(*hq[c], out=ho)
        join_host_copies()
        a1.record()
        torch.cuda.synchronize()
        e2e_sec += a0.elapsed_time(a1) / 1000.0
    e2e_sec = max_over_ranks(e2e_sec, world, dev)
    blk = cfg.T * cfg.H * cfg.d * 2

    if rank != 0:
        ann.close()
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        from oracle import annsa_attention
        f = lambda x: x.to(torch.float64).cpu().numpy()  # noqa: E731
        ann.attend(Qc[0], cfg.P, out=xout)
        _, qcodes, _ = ann.kept()
        t = time.perf_counter()
        annsa_attention(*(f(x) for x in QKV[0]), qcodes)
        cpu = {"value": cfg.F / (time.perf_counter() - t), "unit": UNIT, "cores": len(os.sched_getaffinity(0)),
               "kind": "oracle", "sample": "one block (3 frames x 1560 tokens, 12 heads) in full"}
    line = {
        "metric": ANNSA_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * sec_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": (f"annsa-wan1.3b: H={cfg.H} d={cfg.d} T={cfg.T} (F={cfg.F} x P={cfg.P}), buckets "
                                f"= {cfg.nbits}-bit AnnCA query codes (annca-wan1.3b), Q K V ~ N(0,1) bf16"),
                   "step": f"{calls} tc_annsa_attend calls ({cfg.F * calls} frames); the AnnCA call that "
                           "finds each block's buckets runs before it, outside the timed events",
                   "l2": f"inputs larger than L2 ({calls * 3 * cfg.T * cfg.H * cfg.d * 2 / 1e9:.2f} GB of "
                         "distinct Q, K, V per step)",
                   "parallelism": f"independent layer per rank x{world}"},
        "roofline": {"bound": "tensor", "kernel": "annsa_bcount_kernel + annsa_bplace_kernel + annsa_pack_kernel + "
                                                  "attend_bf16_duo_kernel (sparse), one call",
                     "achieved": tflops, "peak": peak, "unit": "TFLOP/s", "frac": tflops / peak,
                     "peak_kind": f"{peak_kind} bf16 dense, burst", "traffic": None,
                     "flops_per_call": float(np.mean(flops)), "avg_call_us": 1e6 * call_sec},
        "dense_baseline": {"value": cfg.F * calls / dense_sec, "unit": UNIT,
                           "note": "same attention kernel over the whole block (every token sees every token)"},
        "cpu_baseline": cpu,
        "e2e": {"value": aggregate_rate(cfg.F * 8, world, e2e_sec), "unit": UNIT,
                "h2d_bytes_per_step": 3 * blk * calls, "d2h_bytes_per_step": blk * calls},
        "gpu_launches": 3 * calls * args.steps,
        "clocks": clk,
    }
    ann.close()
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- LVSA leg

LVSA_METRIC = "LVSA frame-masked attention frames/s at Wan-1.3B shape, 6x horizon (126 frames, C = 21)"


def run_lvsa(args):
    """One step = one tc_lvsa_attend call (one denoising step s = k) over a 126-frame
    latent video of the Wan-2.1-1.3B layer shape (6x its 21-frame training horizon):
    every query frame attends to C = 21 frames (rotating anchors every T_per = 21
    frames plus its expanded window)."""
    from kv_cache_attention_tempcache_b200 import LVSA
    from oracle import attended_frames

    rank, world, local = dist_info()
    torch.cuda.set_device(local)
    init_dist(world, "nccl")
    dev = torch.device("cuda", local)
    T, P, H, d, T_per, C = 126, 1560, 12, 128, 21, 21
    g = torch.Generator(device=dev).manual_seed(rank_seed(2024, rank))
    Q, K, V = (torch.randn(T * P, H, d, generator=g, device=dev).to(torch.bfloat16) for _ in range(3))
    out = torch.empty_like(Q)
    lv = LVSA(H, d, P, T_per, C)
    dense = LVSA(H, d, P, 1, T)   # every frame attends to every frame: the same kernel, dense

    def flops_of(Cb, Tp, s):
        return 4.0 * P * P * d * H * sum(len(a) for a in attended_frames(T, Tp, Cb, s))

    for k in range(args.warmup):
        lv.attend(Q, K, V, k, out=out)
    torch.cuda.synchronize()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    marks = [(ev(), ev()) for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = ev(), ev()
    t0.record()
    for k in range(args.steps):
        marks[k][0].record()
        lv.attend(Q, K, V, k, out=out)
        marks[k][1].record()
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    sec = t0.elapsed_time(t1) / 1000.0
    sec_max = max_over_ranks(sec, world, dev)
    value = aggregate_rate(T * args.steps, world, sec_max)
    call_sec = sum(a.elapsed_time(b) for a, b in marks) / 1000.0 / args.steps
    flops = float(np.mean([flops_of(C, T_per, k) for k in range(args.steps)]))
    peaks, peak_kind = load_peaks()
    peak = float(peaks.get("bf16_tflops_sustained", peaks.get("bf16_tflops")))
    # dense baseline: the same kernel with every frame attended
    dense.attend(Q, K, V, 0, out=out)
    torch.cuda.synchronize()
    d0, d1 = ev(), ev()
    d0.record()
    dense.attend(Q, K, V, 0, out=out)
    d1.record()
    torch.cuda.synchronize()
    dense_sec = d0.elapsed_time(d1) / 1000.0
    dense_flops = flops_of(T, 1, 0)
    # end to end: Q, K, V from pinned host memory, the output read back
    from kv_cache_attention_tempcache_b200 import host_copy_streams, join_host_copies
    h2d, _ = host_copy_streams()
    hq, hk, hv = (x.cpu().pin_memory() for x in (Q, K, V))
    ho = torch.empty_like(hq).pin_memory()
    lv.attend(hq, hk, hv, 0, out=ho)
    join_host_copies()
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    e0.record()
    h2d.wait_event(e0)   # (no copy before the start)
    lv.attend(hq, hk, hv, 1, out=ho)
    join_host_copies()
    e1.record()
    torch.cuda.synchronize()
    e2e_sec = max_over_ranks(e0.elapsed_time(e1) / 1000.0, world, dev)
    nb = T * P * H * d * 2
    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        from oracle import biased_attention
        A = attended_frames(T, T_per, C, 0)
        t, h = T // 2, 0
        keys = np.concatenate([np.arange(f * P, (f + 1) * P) for f in A[t]])
        f64 = lambda x: x.to(torch.float64).cpu().numpy()  # noqa: E731
        q, kk, vv = f64(Q[t * P:(t + 1) * P, h]), f64(K[keys, h]), f64(V[keys, h])
        tc0 = time.perf_counter()
        biased_attention(q, kk, vv, np.zeros(keys.size), 1.0 / math.sqrt(d))
        tcpu = (time.perf_counter() - tc0) * T * H
        cpu = {"value": T / tcpu, "unit": UNIT, "cores": len(os.sched_getaffinity(0)), "kind": "oracle",
               "sample": f"query frame {t} of head {h} in full (its {len(A[t])} frames of keys), scaled to "
                         f"{T} frames x {H} heads"}
    line = {
        "metric": LVSA_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * sec_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"lvsa-wan1.3b: T={T} frames x P={P} tokens, H={H} d={d}, T_per={T_per}, C={C}, "
                               "Q K V ~ N(0,1) bf16",
                   "step": "one tc_lvsa_attend call (denoising step s = k)",
                   "l2": f"inputs larger than L2 ({3 * nb / 1e9:.2f} GB of Q, K, V)",
                   "parallelism": f"independent layer per rank x{world}"},
        "roofline": {"bound": "tensor", "kernel": "attend_bf16_duo_kernel (frame mode)", "achieved": flops / call_sec / 1e12,
                     "peak": peak, "unit": "TFLOP/s", "frac": flops / call_sec / 1e12 / peak,
                     "peak_kind": f"{peak_kind} bf16 dense, sustained", "traffic": None,
                     "flops_per_call": flops, "avg_call_ms": 1000.0 * call_sec},
        "dense_baseline": {"value": T / dense_sec, "unit": UNIT, "attn_tflops": dense_flops / dense_sec / 1e12,
                           "note": "same kernel with C = T (every frame attends to every frame)"},
        "cpu_baseline": cpu,
        "e2e": {"value": aggregate_rate(T, world, e2e_sec), "unit": UNIT, "h2d_bytes_per_step": 3 * nb,
                "d2h_bytes_per_step": nb},
        "gpu_launches": 2 * args.steps,
        "clocks": clk,
    }
    lv.close()
    dense.close()
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", action="store_true",
                    help="timed rollouts only (no dense baseline, end-to-end or CPU legs), for profilers")
    ap.add_argument("--chunks", type=int, default=0,
                    help="rollout length in chunks (default: the workload's); profiling runs use fewer")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=[k for k, v in CONFIGS.items() if v.dtype == "bf16"] + ["annca-wan1.3b",
                                                                                      "annsa-wan1.3b",
                                                                                      "lvsa-wan1.3b"],
                    help="synthetic workload; only the default one adds the dense, end-to-end and CPU legs "
                         "(annca-wan1.3b: AnnCA cross-attention, with its own legs)")
    ap.add_argument("--series", action="store_true", help="add per-chunk commit and attention times")
    ap.add_argument("--intra-chunk", action="store_true",
                    help="commits also match tokens against entries created earlier in the same commit")
    ap.add_argument("--key-mode", default="representative", choices=["representative", "mean"],
                    help="mean: an entry's key is the running mean of its members' keys")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload in CROSS_CONFIGS:
        run_annca(args)
    elif args.workload == "annsa-wan1.3b":
        run_annsa(args)
    elif args.workload == "lvsa-wan1.3b":
        run_lvsa(args)
    else:
        run_gpu(args)
    if torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
