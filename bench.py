#!/usr/bin/env python
"""Benchmark of the paged decode step on B200: KV-read GB/s and decode tokens/s per layer.

One step = one pass of the whole decode path over one batch: the new-token
KV write (one token per sequence), then paged decode attention (partition
pass + split-context reduce), and -- for workloads with shared prefixes --
the copy-on-write block copies first.  Inputs are synthetic and seeded
(paged_kv_cache_450_b200.workloads) and already resident in HBM when the
timed region starts; the KV stream per step (1.14 GB for the default
workload) is larger than the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

N > 1 runs under torchrun, one process per GPU; every rank processes its own
independent batch (different seed), there is no data-path collective, and the
time is the max over ranks ("scaling": "weak").  ``--impl reference`` times
the CPU oracle (fp64 C) on the host cores instead.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_450_b200 import workloads as W  # noqa: E402

METRIC = "paged decode attention KV-read GB/s (% of B200 HBM peak); decode tokens/s per layer"
DEFAULT_WORKLOAD = W.LLAMA7B.name
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0
DTYPE_NAMES = {torch.float32: "f32", torch.bfloat16: "bf16", torch.float8_e4m3fn: "fp8_e4m3"}


# --------------------------------------------------------------------------- #
# host-side multi-rank logic (covered by CPU gloo tests)
# --------------------------------------------------------------------------- #

def dist_env():
    """(rank, world_size, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws its own independent batch (weak scaling)."""
    return base_seed + 1000 * rank


def max_over_ranks(x: float, device=None) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# --------------------------------------------------------------------------- #
# peaks, clocks, profiles
# --------------------------------------------------------------------------- #

def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device: torch.device):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            self.ident = None

    def start(self):
        if self.ident is None:
            return
        self.path = f"/tmp/pkv_clocks_{os.getpid()}.csv"
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.ident}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
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
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def profile_traffic(kernel_file: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if it was taken on
    the current kernel source (sha256 of the files it names); else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel_file}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*(\d+)", text)
    h = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    w = re.search(r"workload:\s*(\S+)", text)
    if not (m and h and w) or w.group(1) != workload:
        return None
    if h.group(1) != kernel_source_hash():
        return None
    return int(m.group(1))


def kernel_source_hash() -> str:
    d = os.path.join(ROOT, "paged_kv_cache_450_b200", "csrc")
    hsh = hashlib.sha256()
    for name in ("common.cuh", "decode.cuh", "decode_mma.cuh", "decode_mma_bf16.cuh", "decode_launch.cuh"):
        with open(os.path.join(d, name), "rb") as f:
            hsh.update(f.read())
    return hsh.hexdigest()


# --------------------------------------------------------------------------- #
# the GPU arm
# --------------------------------------------------------------------------- #

def kernel_name(spec) -> str:
    """The decode partition kernel that serves this workload (mirrors the library's dispatch)."""
    g = spec.num_q_heads // spec.num_kv_heads
    if spec.head_dim == 128 and spec.block_size in (16, 32):
        if spec.cache_dtype == torch.float8_e4m3fn and g == 8:
            return "paged_decode_gqa8_fp8_mma_kernel"
        if spec.cache_dtype == torch.bfloat16 and g in (2, 4, 8):
            return "paged_decode_mma_bf16_kernel"
    return "paged_decode_partition_kernel"


def step_inputs_bytes(w) -> tuple[int, int]:
    """Bytes of one step's per-step inputs (host -> device) and result (device -> host)."""
    ts = [w.q, w.new_k, w.new_v, w.slot_mapping, w.block_tables, w.context_lens, w.copy_pairs]
    h2d = sum(t.numel() * t.element_size() for t in ts if t is not None)
    return h2d, w.q.numel() * w.q.element_size()


def run_gpu(args, rank, world, local_rank):
    import paged_kv_cache_450_b200 as pk

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    spec = workload_spec(args)
    w = W.make_decode_workload(spec, seed=rank_seed(args.seed, rank), device=dev)
    s = spec
    kv_bytes = w.kv_bytes()
    MB = w.block_tables.shape[1]
    pt = pk.decode_partition_tokens(s.num_seqs, s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size, MB,
                                    s.cache_dtype, args.partition_tokens)
    ws_bytes = pk.decode_workspace_bytes(s.num_seqs, s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size, MB,
                                         s.cache_dtype, pt)
    workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    out = torch.empty_like(w.q)
    kc, vc = w.key_cache, w.value_cache
    stream = torch.cuda.current_stream(dev)

    fused = w.new_k is not None and not args.unfused

    def step(ev_mid=None, ev_end=None):
        if w.copy_pairs is not None and len(w.copy_pairs):
            pk.kv_block_copy(w.copy_pairs, kc, vc, stream=stream)
        if fused:  # the new token (one per sequence, at ctx - 1) is written inside the decode launch
            if ev_mid is not None:
                ev_mid.record(stream)
            pk.paged_decode_append(w.q, w.new_k, w.new_v, kc, vc, w.block_tables, w.context_lens, w.scale,
                                   k_scale=w.k_scale, v_scale=w.v_scale, out=out, workspace=workspace,
                                   partition_tokens=pt, stream=stream)
        else:
            if w.new_k is not None:
                pk.paged_kv_write(w.new_k, w.new_v, w.slot_mapping, kc, vc, k_scale=w.k_scale, v_scale=w.v_scale,
                                  stream=stream)
            if ev_mid is not None:
                ev_mid.record(stream)
            pk.paged_attention_decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, k_scale=w.k_scale,
                                      v_scale=w.v_scale, out=out, workspace=workspace, partition_tokens=pt,
                                      stream=stream)
        if ev_end is not None:
            ev_end.record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    # ---- timed region: device-resident inputs, K whole steps ------------------
    # No events between the kernels of a step (they would stop the launch of
    # one kernel from overlapping the tail of the previous one).
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(dev)
    barrier(dev)
    torch.cuda.synchronize(dev)
    clocks.start()
    launches0 = pk.launch_count()
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    launches = pk.launch_count() - launches0
    barrier(dev)
    clk = clocks.stop()
    elapsed_ms = t0.elapsed_time(t1)

    # ---- the decode kernels alone (roofline): events around each decode call --
    n_inst = max(1, min(args.steps, 1000))
    mids = [torch.cuda.Event(enable_timing=True) for _ in range(n_inst)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(n_inst)]
    for i in range(n_inst):
        step(mids[i], ends[i])
    torch.cuda.synchronize(dev)
    decode_ms = sum(m.elapsed_time(e) for m, e in zip(mids, ends)) / n_inst

    # ---- end to end through the public API with pinned host buffers ----------
    host = {k: (getattr(w, k).cpu().pin_memory() if getattr(w, k) is not None else None)
            for k in ("q", "new_k", "new_v", "slot_mapping", "block_tables", "context_lens", "copy_pairs")}
    # two steps in flight: the copies in of step i+1 overlap the kernels of step i
    pipe = pk.HostStepPipeline(host["q"], host["new_k"], kc, host["block_tables"], host["copy_pairs"],
                               partition_tokens=pt, depth=2, compute_stream=stream)

    def e2e_step():
        pipe.step(host["q"], host["new_k"], host["new_v"], host["slot_mapping"], host["block_tables"],
                  host["context_lens"], kc, vc, w.scale, copy_pairs=host["copy_pairs"], k_scale=w.k_scale,
                  v_scale=w.v_scale)

    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    for _ in range(min(args.warmup, 10)):
        e2e_step()
    pipe.synchronize()
    torch.cuda.synchronize(dev)
    barrier(dev)
    # the timed region opens on the copy-in stream (before the first copy) and closes on the
    # copy-out stream after the last step's output has landed in host memory
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(pipe.copy_in)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(pipe.copy_out)
    e1.synchronize()
    torch.cuda.synchronize(dev)
    barrier(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    # ---- cross-rank aggregation ------------------------------------------------
    step_ms = max_over_ranks(elapsed_ms / args.steps, dev)
    e2e_ms = max_over_ranks(e2e_ms, dev)
    decode_ms = max_over_ranks(decode_ms, dev)
    total_kv = sum_over_ranks(kv_bytes, dev)
    total_seqs = sum_over_ranks(s.num_seqs, dev)
    h2d, d2h = step_inputs_bytes(w)

    peak, peak_kind = hbm_peak()
    value = total_kv / (step_ms * 1e-3) / 1e9
    achieved = kv_bytes / (decode_ms * 1e-3) / 1e9
    res = None
    if rank == 0:
        cpu = cpu_baseline(w, args) if (world == 1 and not args.no_cpu_baseline) else None
        res = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(step_ms, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": DTYPE_NAMES[s.cache_dtype], "data": "synthetic",
            "config": {"workload": s.name, "num_seqs_per_gpu": s.num_seqs, "num_q_heads": s.num_q_heads,
                       "num_kv_heads": s.num_kv_heads, "head_dim": s.head_dim, "block_size": s.block_size,
                       "q_dtype": DTYPE_NAMES[s.q_dtype], "kv_dtype": DTYPE_NAMES[s.cache_dtype],
                       "context_lens": list(s.ctx), "pool": list(s.pool),
                       "kv_bytes_per_step_per_gpu": kv_bytes, "partition_tokens": pt,
                       "new_tokens_per_step": 0 if w.new_k is None else int(w.new_k.shape[0]),
                       "new_token_write": "fused into the decode launch" if fused else "separate launch",
                       "cow_pairs_per_step": 0 if w.copy_pairs is None else int(len(w.copy_pairs)),
                       "l2": "inputs larger than L2 (KV stream per step > 126 MB); no flush",
                       "parallelism": f"dp{world} (independent batch per GPU, no collective)"},
            "pct_of_hbm_peak": {"measured_copy": round(100 * value / peak, 2) if peak_kind == "measured" else None,
                                "spec_8tbs": round(100 * value / SPEC_HBM_GBS, 2)},
            "tokens_per_s_per_layer": round(total_seqs / (step_ms * 1e-3), 1),
            "roofline": {"kernel": kernel_name(s) + " + paged_decode_reduce_kernel",
                         "bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                         "peak_kind": f"{peak_kind} (burst copy bandwidth)", "frac": round(achieved / peak, 4),
                         "algorithmic_bytes_per_launch": kv_bytes, "decode_ms": round(decode_ms, 5),
                         "timing": f"CUDA events around each decode call on its stream, {n_inst} steps after the timed region",
                         "traffic": profile_traffic("paged_decode_" + s.name, s.name)},
            "e2e": {"value": round(total_kv / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s", "steps": e2e_steps,
                    "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "api": "paged_kv_cache_450_b200.HostStepPipeline -> pkv_decode_step_host_async (pinned host inputs and output every step; two steps in flight: copies in, kernels, copies out on three streams)"},
            "gpu_launches": int(launches),
            "clocks": clk,
            "cpu_baseline": cpu,
        }
    return res


# --------------------------------------------------------------------------- #
# the CPU oracle (cpu_baseline leg and --impl reference)
# --------------------------------------------------------------------------- #

def _host_state(w):
    import oracle

    def to_np(t):
        t = t.detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            return t.view(torch.int16).numpy().view(np.uint16)
        if t.dtype == torch.float8_e4m3fn:
            return t.view(torch.uint8).numpy()
        return t.numpy()

    code = {torch.float32: oracle.F32, torch.bfloat16: oracle.BF16, torch.float8_e4m3fn: oracle.E4M3}
    s = w.spec
    st = {"q": to_np(w.q), "kc": to_np(w.key_cache).copy(), "vc": to_np(w.value_cache).copy(),
          "tables": to_np(w.block_tables), "lens": to_np(w.context_lens), "qd": code[s.q_dtype],
          "cd": code[s.cache_dtype]}
    if w.copy_pairs is not None and len(w.copy_pairs):
        oracle.kv_block_copy(to_np(w.copy_pairs), st["kc"], st["vc"])
    if w.new_k is not None:
        oracle.paged_kv_write(to_np(w.new_k), to_np(w.new_v), to_np(w.slot_mapping), st["kc"], st["vc"],
                              in_dtype=code[s.q_dtype], cache_dtype=code[s.cache_dtype], k_scale=w.k_scale,
                              v_scale=w.v_scale)
    return st


def _row_bytes(w):
    """Logical KV bytes attributed to each (sequence, query head) row."""
    s = w.spec
    ctx = np.repeat(np.array(w.ctx_list, np.float64), s.num_q_heads)
    return ctx * s.head_dim * W.elem_size(s.cache_dtype) * 2 * s.num_kv_heads / s.num_q_heads


def _oracle_rows(w, st, rows, threads):
    import oracle
    return oracle.paged_attention_decode(st["q"], st["kc"], st["vc"], st["tables"], st["lens"], scale=w.scale,
                                         q_dtype=st["qd"], cache_dtype=st["cd"], k_scale=w.k_scale,
                                         v_scale=w.v_scale, rows=rows, num_threads=threads)


def cpu_baseline(w, args, budget_s: float = 15.0):
    """The oracle as it stands, on this host's cores, over a bounded sample of
    the same workload: whole rows (sequence, query head) in a seeded order
    until about `budget_s` seconds of work or the whole batch."""
    threads = os.cpu_count() or 1
    st = _host_state(w)
    rb = _row_bytes(w)
    order = np.random.default_rng(0).permutation(len(rb))
    done, t_used, nbytes, i = 0, 0.0, 0.0, 0
    chunk = max(threads, 8)
    while i < len(order) and t_used < budget_s:
        rows = order[i:i + chunk]
        t = time.perf_counter()
        _oracle_rows(w, st, rows, threads)
        t_used += time.perf_counter() - t
        nbytes += rb[rows].sum()
        done += len(rows)
        i += len(rows)
        chunk = min(chunk * 2, 4096)
    return {"value": round(nbytes / t_used / 1e9, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{done} of {len(rb)} (sequence, query head) rows of {w.spec.name} "
                      f"({nbytes / 1e9:.3f} GB of logical KV) in {t_used:.1f} s, fp64 C oracle, OpenMP"}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle timed on the host cores, K steps, each a
    bounded sample (whole rows) of the same workload; rank 0 only."""
    if rank != 0:
        return None
    spec = workload_spec(args)
    w = W.make_decode_workload(spec, seed=rank_seed(args.seed, 0), device="cpu")
    threads = os.cpu_count() or 1
    st = _host_state(w)
    rb = _row_bytes(w)
    order = np.random.default_rng(0).permutation(len(rb))
    # size the per-step sample so that warmup + steps take about args.ref_budget seconds
    t = time.perf_counter()
    _oracle_rows(w, st, order[:threads], threads)
    per_row = max((time.perf_counter() - t) / threads, 1e-6)
    total_steps = args.steps + args.warmup
    rows_per_step = int(max(1, min(len(rb), args.ref_budget / total_steps / per_row)))
    pos = 0

    def take():
        nonlocal pos
        r = np.take(order, np.arange(pos, pos + rows_per_step), mode="wrap")
        pos = (pos + rows_per_step) % len(order)
        return r

    for _ in range(args.warmup):
        _oracle_rows(w, st, take(), threads)
    t_total, nbytes = 0.0, 0.0
    for _ in range(args.steps):
        r = take()
        t = time.perf_counter()
        _oracle_rows(w, st, r, threads)
        t_total += time.perf_counter() - t
        nbytes += rb[r].sum()
    value = nbytes / t_total / 1e9
    sample = (f"{rows_per_step} (sequence, query head) rows per step of {spec.name}, "
              f"fp64 C oracle with OpenMP on {threads} threads")
    return {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * t_total / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": spec.name}, "impl": "reference",
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# --------------------------------------------------------------------------- #

def workload_spec(args):
    spec = W.SPECS[args.workload]
    if args.num_seqs:
        if spec.sampling is not None:
            raise SystemExit("--num-seqs does not apply to the parallel-sampling workload")
        spec = spec.with_(name=f"{spec.name}@b{args.num_seqs}", num_seqs=args.num_seqs)
    return spec


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.SPECS) + sorted(W.MQ_SPECS))
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--partition-tokens", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=1000)
    ap.add_argument("--ref-budget", type=float, default=90.0, help="seconds of oracle work for --impl reference")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--unfused", action="store_true",
                    help="write the new tokens with a separate paged_kv_write launch instead of inside the decode")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="override the workload's batch (a smaller case of the same shape, for profiling)")
    return ap.parse_args(argv)


def run_multiquery(args, rank, world, local_rank):
    """Multi-query attention (draft verification / chunked prefill) timed alone."""
    import paged_kv_cache_450_b200 as pk

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    spec, n = W.MQ_SPECS[args.workload]
    if args.num_seqs:
        spec = spec.with_(name=f"{spec.name}@b{args.num_seqs}", num_seqs=args.num_seqs)
    mw = W.make_multiquery_workload(spec, [n] * spec.num_seqs, seed=rank_seed(args.seed, rank), device=dev)
    w = mw.base
    s = spec
    kv_bytes = w.kv_bytes()
    flops = mw.flops()
    stream = torch.cuda.current_stream(dev)
    out = torch.empty_like(mw.q)
    MB = w.block_tables.shape[1]
    lib = pk._lib.load()
    T = int(mw.query_start_loc[-1])
    need = int(lib.pkv_multiquery_workspace_bytes(s.num_seqs, T, n, s.num_q_heads, s.num_kv_heads, s.head_dim,
                                                  s.block_size, MB, args.partition_tokens))
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)

    def call():
        pk.paged_attention_multiquery(mw.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens,
                                      mw.query_start_loc, w.scale, max_q_len=n, out=out, workspace=ws,
                                      partition_tokens=args.partition_tokens, stream=stream)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dev)
    clocks = ClockSampler(dev)
    clocks.start()
    launches0 = pk.launch_count()
    t0.record(stream)
    for _ in range(args.steps):
        call()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    launches = pk.launch_count() - launches0
    clk = clocks.stop()
    step_ms = max_over_ranks(t0.elapsed_time(t1) / args.steps, dev)
    total_kv = sum_over_ranks(kv_bytes, dev)
    total_flops = sum_over_ranks(flops, dev)
    if rank != 0:
        return None
    peak_gbs, peak_kind = hbm_peak()
    gbs = kv_bytes / (step_ms * 1e-3) / 1e9
    tflops = flops / (step_ms * 1e-3) / 1e12
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak_tf = float(json.load(f)["bf16_tflops"])
    except Exception:
        peak_tf = 1590.0
    tensor_bound = flops / max(kv_bytes, 1) > peak_tf * 1e12 / (peak_gbs * 1e9)
    return {
        "metric": METRIC, "value": round(total_kv / (step_ms * 1e-3) / 1e9, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": s.name, "op": "paged_attention_multiquery (causal, queries = last q_len positions)",
                   "num_seqs_per_gpu": s.num_seqs, "q_len": n, "num_q_heads": s.num_q_heads,
                   "num_kv_heads": s.num_kv_heads, "head_dim": s.head_dim, "block_size": s.block_size,
                   "context_lens": list(s.ctx), "kv_bytes_per_step_per_gpu": kv_bytes, "flops_per_step": flops},
        "tflops": round(total_flops / (step_ms * 1e-3) / 1e12, 2),
        "roofline": {"kernel": ("paged_multiquery_tc_kernel" if n * (s.num_q_heads // s.num_kv_heads) > 16
                                else "paged_multiquery_bf16_kernel")
                               + (" + paged_multiquery_reduce_kernel" if need else ""),
                     "bound": "tensor" if tensor_bound else "hbm",
                     "achieved": round(tflops if tensor_bound else gbs, 2),
                     "peak": peak_tf if tensor_bound else peak_gbs,
                     "unit": "TFLOP/s" if tensor_bound else "GB/s",
                     "frac": round((tflops / peak_tf) if tensor_bound else (gbs / peak_gbs), 4),
                     "traffic": None},
        "gpu_launches": int(launches), "clocks": clk, "cpu_baseline": None,
    }


def main(argv=None):
    args = parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    rank, world, local_rank = dist_env()
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}: launch N>1 with torchrun")
    if args.impl == "reference":
        # rank 0 alone times the oracle; the other ranks exit without work
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.workload in W.MQ_SPECS:
            res = run_multiquery(args, rank, world, local_rank)
        else:
            res = run_gpu(args, rank, world, local_rank)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
