#!/usr/bin/env python
"""Benchmark of the paged decode step on B200: KV-read GB/s and decode tokens/s per layer.

One step = one pass of the whole decode path over one batch: the new-token
KV write (one token per sequence, fused into the decode launch), paged decode
attention (partition pass + split-context reduce) and -- for workloads with
shared prefixes -- the copy-on-write block copies first.  Inputs are
synthetic and seeded (paged_kv_cache_450_b200.workloads) and already resident
in HBM when the timed region starts; every workload's KV stream per step is
larger than the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--configs auto|all|none]
                  [--impl reference]

The headline line is the LLaMA-13B-shaped batch-256 workload (the largest
single-GPU configuration).  At N = 1 the same line carries a ``configs``
object with the same measurements for the other decode configurations and a
``multiquery`` object for the multi-query workloads, all from this one run.
N > 1 runs under torchrun, one process per GPU; every rank processes its own
independent batch (different seed), there is no data-path collective, and the
time is the max over ranks ("scaling": "weak").  ``--impl reference`` times
the CPU oracle (fp64 C) on the host cores instead.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import gc
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_450_b200 import workloads as W  # noqa: E402

METRIC = "paged decode attention KV-read GB/s (% of B200 HBM peak); decode tokens/s per layer"
DEFAULT_WORKLOAD = W.LLAMA13B.name
# the other decode configurations measured in the same run (N = 1)
SECONDARY = ["llama13b_decode_b256_bf16_bs32", W.PARALLEL_SAMPLING.name, W.GQA_LONG.name, W.GQA_BATCH.name,
             W.LLAMA7B.name]
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
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

def _peaks_file():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f)
    except Exception:
        return None


def hbm_peak():
    p = _peaks_file()
    try:
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def bf16_peak():
    p = _peaks_file()
    try:
        return float(p["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


# NVML clock-event reason bits and the names the bench line reports
_REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting", 0x10: "sync_boost"}
REJECT_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


class ClockSampler:
    """SM clock and clock-event reasons of this GPU, sampled by a background
    thread through NVML every ~2 ms for the whole run; ``window(t0, t1)``
    summarises the samples taken between two host timestamps (a timed region).
    Reading clocks changes no setting of the GPU."""

    def __init__(self, device: torch.device, period_s: float = 0.002):
        self.period = period_s
        self.samples = []          # (host time, sm MHz, reason bits)
        self.handle = None
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            self.nvml = pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device)
            try:
                uuid = str(props.uuid)
                self.handle = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else f"GPU-{uuid}")
            except Exception:  # the same GPU by its PCI address
                bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
                self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM))
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception as e:  # no NVML: the line says so
            self.error = f"{type(e).__name__}: {e}"
            self.handle = None

    def _run(self):
        nv, h = self.nvml, self.handle
        while not self._stop.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                bits = int(self._reasons(h))
                self.samples.append((time.perf_counter(), mhz, bits))
            except Exception as e:
                self.error = f"{type(e).__name__}: {e}"
                return
            time.sleep(self.period)

    def start(self):
        if self.handle is not None and self._thread is None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
            t_end = time.perf_counter() + 1.0
            while not self.samples and time.perf_counter() < t_end and self._thread.is_alive():
                time.sleep(0.001)

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def window(self, t0: float, t1: float):
        if self.handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "source": f"NVML unavailable ({self.error})"}
        rows = [s for s in list(self.samples) if t0 <= s[0] <= t1]
        where = "inside the timed region"
        if not rows:  # a region shorter than the sampling period: the samples just around it
            near = sorted(list(self.samples), key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
            rows = near
            where = "the samples nearest the timed region (region shorter than the 2 ms sampling period)"
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "source": "NVML, no sample"}
        reasons = sorted({name for _, _, b in rows for bit, name in _REASONS.items() if b & bit})
        med = statistics.median(r[1] for r in rows)
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(rows),
                "source": f"NVML every {self.period * 1e3:.0f} ms, {where}",
                "rejected": bool(set(reasons) & REJECT_REASONS) or (self.max_mhz is not None and not reasons
                                                                     and med < 0.8 * self.max_mhz)}


def profile_traffic(profile: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (sha256 recorded in the summary); else None."""
    path = os.path.join(ROOT, "profiles", f"{profile}.md")
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
    """sha256 of the decode kernel sources (what a recorded DRAM byte count depends on)."""
    d = os.path.join(ROOT, "paged_kv_cache_450_b200", "csrc")
    hsh = hashlib.sha256()
    for name in ("common.cuh", "decode.cuh", "decode_mma.cuh", "decode_mma_bf16.cuh", "decode_launch.cuh"):
        with open(os.path.join(d, name), "rb") as f:
            hsh.update(f.read())
    return hsh.hexdigest()


# --------------------------------------------------------------------------- #
# byte accounting
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


def unique_kv_bytes(w) -> int:
    """KV bytes of the distinct (physical block, row) pairs one decode pass reads:
    a block shared by several sequences counts once (prefix sharing)."""
    s = w.spec
    bs = s.block_size
    tables = w.block_tables.cpu().numpy()
    rows = {}
    for b, c in enumerate(w.ctx_list):
        for j in range(-(-c // bs)):
            pid = int(tables[b, j])
            rows[pid] = max(rows.get(pid, 0), min(bs, c - j * bs))
    return int(sum(rows.values())) * s.num_kv_heads * s.head_dim * W.elem_size(s.cache_dtype) * 2


def step_inputs_bytes(w, grouped: bool = False) -> tuple[int, int]:
    """Bytes of one step's per-step inputs (host -> device) and result (device -> host)."""
    ts = [w.q, w.new_k, w.new_v, w.block_tables, w.context_lens, w.copy_pairs]
    ts += [w.group_start, w.shared_blocks] if grouped else [w.slot_mapping]
    h2d = sum(t.numel() * t.element_size() for t in ts if t is not None)
    return h2d, w.q.numel() * w.q.element_size()


def _events(n=2):
    return [torch.cuda.Event(enable_timing=True) for _ in range(n)]


# --------------------------------------------------------------------------- #
# the GPU arm: one decode workload
# --------------------------------------------------------------------------- #

def measure_decode(spec, args, dev, rank, world, clocks, *, headline: bool):
    """Step, decode-kernel, end-to-end and oracle timings of one decode workload."""
    import paged_kv_cache_450_b200 as pk

    w = W.make_decode_workload(spec, seed=rank_seed(args.seed, rank), device=dev)
    s = spec
    kv_bytes = w.kv_bytes()
    kv_unique = unique_kv_bytes(w) if w.copy_pairs is not None else kv_bytes
    MB = w.block_tables.shape[1]
    pt = pk.decode_partition_tokens(s.num_seqs, s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size, MB,
                                    s.cache_dtype, args.partition_tokens)
    ws_bytes = pk.decode_workspace_bytes(s.num_seqs, s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size, MB,
                                         s.cache_dtype, pt)
    fused = w.new_k is not None and not args.unfused
    # groups sharing their prompt's blocks (parallel sampling): each shared block read once per group
    grouped = w.group_start is not None and fused and not args.no_shared_prefix
    if grouped:
        n_groups = int(w.group_start.shape[0]) - 1
        max_group = int((w.group_start[1:] - w.group_start[:-1]).max().item())
        pt = pk.decode_shared_prefix_partition_tokens(n_groups, s.num_kv_heads, s.block_size, MB,
                                                      args.partition_tokens)
        ws_bytes = pk.decode_shared_prefix_workspace_bytes(s.num_seqs, n_groups, s.num_q_heads, s.num_kv_heads,
                                                           s.head_dim, s.block_size, MB, pt)
    workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    out = torch.empty_like(w.q)
    stream = torch.cuda.current_stream(dev)

    def decode(kc, vc, tables):
        if grouped:
            pk.paged_attention_decode_shared_prefix(w.q, kc, vc, tables, w.context_lens, w.group_start,
                                                    w.shared_blocks, w.scale, k_new=w.new_k, v_new=w.new_v,
                                                    max_group_size=max_group, out=out, workspace=workspace,
                                                    partition_tokens=pt, stream=stream)
        elif fused:  # the new token (one per sequence, at ctx - 1) is written inside the decode launch
            pk.paged_decode_append(w.q, w.new_k, w.new_v, kc, vc, tables, w.context_lens, w.scale,
                                   k_scale=w.k_scale, v_scale=w.v_scale, out=out, workspace=workspace,
                                   partition_tokens=pt, stream=stream)
        else:
            if w.new_k is not None:
                pk.paged_kv_write(w.new_k, w.new_v, w.slot_mapping, kc, vc, k_scale=w.k_scale, v_scale=w.v_scale,
                                  stream=stream)
            pk.paged_attention_decode(w.q, kc, vc, tables, w.context_lens, w.scale, k_scale=w.k_scale,
                                      v_scale=w.v_scale, out=out, workspace=workspace, partition_tokens=pt,
                                      stream=stream)

    def step():
        if w.copy_pairs is not None and len(w.copy_pairs):
            pk.kv_block_copy(w.copy_pairs, w.key_cache, w.value_cache, stream=stream)
        decode(w.key_cache, w.value_cache, w.block_tables)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    # ---- timed region: device-resident inputs, K whole steps ------------------
    # No events between the kernels of a step (they would stop the launch of
    # one kernel from overlapping the tail of the previous one).
    t0, t1 = _events()
    barrier(dev)
    torch.cuda.synchronize(dev)
    launches0 = pk.launch_count()
    h0 = time.perf_counter()
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    h1 = time.perf_counter()
    launches = pk.launch_count() - launches0
    barrier(dev)
    clk = clocks.window(h0, h1)
    step_ms = t0.elapsed_time(t1) / args.steps

    # ---- the decode launches alone (roofline): one event pair around N -------
    # back-to-back decode calls (partition pass + merge; the fused append
    # rewrites the same token each time), on the launching stream.
    n_dec = max(args.steps, 20)
    d0, d1 = _events()
    d0.record(stream)
    for _ in range(n_dec):
        decode(w.key_cache, w.value_cache, w.block_tables)
    d1.record(stream)
    torch.cuda.synchronize(dev)
    decode_ms = d0.elapsed_time(d1) / n_dec

    ablation = placement_ablation(w, args, dev, stream, decode, pt, n_dec) if headline and world == 1 else None

    # ---- end to end through the public API with pinned host buffers ----------
    host = {k: (getattr(w, k).cpu().pin_memory() if getattr(w, k) is not None else None)
            for k in ("q", "new_k", "new_v", "slot_mapping", "block_tables", "context_lens", "copy_pairs",
                      "group_start", "shared_blocks")}
    # two steps in flight: the copies in of step i+1 overlap the kernels of step i
    if grouped:  # the same shared-prefix decode, its inputs and output in host memory
        pipe = pk.SharedPrefixHostStepPipeline(host["q"], w.key_cache, host["block_tables"], host["group_start"],
                                               host["copy_pairs"], partition_tokens=pt, depth=2,
                                               compute_stream=stream)

        def e2e_step():
            pipe.step(host["q"], host["new_k"], host["new_v"], host["block_tables"], host["context_lens"],
                      host["group_start"], host["shared_blocks"], w.key_cache, w.value_cache, w.scale,
                      max_group_size=max_group, copy_pairs=host["copy_pairs"])
    else:
        pipe = pk.HostStepPipeline(host["q"], host["new_k"], w.key_cache, host["block_tables"], host["copy_pairs"],
                                   partition_tokens=pt, depth=2, compute_stream=stream)

        def e2e_step():
            pipe.step(host["q"], host["new_k"], host["new_v"], host["slot_mapping"], host["block_tables"],
                      host["context_lens"], w.key_cache, w.value_cache, w.scale, copy_pairs=host["copy_pairs"],
                      k_scale=w.k_scale, v_scale=w.v_scale)

    e2e_steps = max(1, args.e2e_steps)  # its own count: the two-deep pipeline's fill and drain amortised
    for _ in range(min(args.warmup, 10)):
        e2e_step()
    pipe.synchronize()
    torch.cuda.synchronize(dev)
    barrier(dev)
    # the timed region opens on the copy-in stream (before the first copy) and closes on the
    # copy-out stream after the last step's output has landed in host memory
    e0, e1 = _events()
    e0.record(pipe.copy_in)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(pipe.copy_out)
    e1.synchronize()
    torch.cuda.synchronize(dev)
    barrier(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    del pipe

    # ---- cross-rank aggregation ------------------------------------------------
    step_ms = max_over_ranks(step_ms, dev)
    e2e_ms = max_over_ranks(e2e_ms, dev)
    decode_ms = max_over_ranks(decode_ms, dev)
    total_kv = sum_over_ranks(kv_bytes, dev)
    total_seqs = sum_over_ranks(s.num_seqs, dev)
    h2d, d2h = step_inputs_bytes(w, grouped)
    peak, peak_kind = hbm_peak()
    value = total_kv / (step_ms * 1e-3) / 1e9
    shared = w.copy_pairs is not None
    # algorithmic bytes of the decode launch: the logical KV stream, or for shared
    # prefixes the distinct blocks (the rest is served from L2)
    alg = kv_unique if shared else kv_bytes
    achieved = alg / (decode_ms * 1e-3) / 1e9
    traffic = profile_traffic("paged_decode_" + s.name, s.name)
    res = {
        "value": round(value, 2), "unit": "GB/s", "ms_per_step": round(step_ms, 5),
        "tokens_per_s_per_layer": round(total_seqs / (step_ms * 1e-3), 1),
        "pct_of_hbm_peak": {"measured_copy": round(100 * value / peak, 2) if peak_kind == "measured" else None,
                            "fallback_copy": round(100 * value / peak, 2) if peak_kind == "fallback" else None,
                            "spec_8tbs": round(100 * value / SPEC_HBM_GBS, 2)},
        "config": {"workload": s.name, "num_seqs_per_gpu": s.num_seqs, "num_q_heads": s.num_q_heads,
                   "num_kv_heads": s.num_kv_heads, "head_dim": s.head_dim, "block_size": s.block_size,
                   "q_dtype": DTYPE_NAMES[s.q_dtype], "kv_dtype": DTYPE_NAMES[s.cache_dtype],
                   "context_lens": list(s.ctx), "pool": list(s.pool),
                   "kv_bytes_per_step_per_gpu": kv_bytes, "partition_tokens": pt,
                   "new_tokens_per_step": 0 if w.new_k is None else int(w.new_k.shape[0]),
                   "new_token_write": "fused into the decode launch" if fused else "separate launch",
                   "decode": ("shared prefix: each group's shared blocks read once for all its members, own "
                              "blocks per sequence, partials merged" if grouped else "per sequence"),
                   "cow_pairs_per_step": 0 if w.copy_pairs is None else int(len(w.copy_pairs)),
                   "l2": "inputs larger than L2 (KV stream per step > 126 MB); no flush",
                   "parallelism": f"dp{world} (independent batch per GPU, no collective)"},
        "roofline": {"kernel": ("paged_decode_mma_bf16_kernel (shared-prefix units)" if grouped else kernel_name(s))
                               + " + paged_decode_reduce_kernel",
                     "bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                     "peak_kind": f"{peak_kind} (burst copy bandwidth)", "frac": round(achieved / peak, 4),
                     "algorithmic_bytes_per_launch": alg, "decode_ms": round(decode_ms, 5),
                     "timing": f"one CUDA event pair around {n_dec} back-to-back decode launches on their stream",
                     "traffic": traffic},
        "e2e": {"value": round(total_kv / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s", "steps": e2e_steps,
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "api": ("paged_kv_cache_450_b200.SharedPrefixHostStepPipeline -> "
                        "pkv_decode_step_host_shared_prefix_async" if grouped else
                        "paged_kv_cache_450_b200.HostStepPipeline -> pkv_decode_step_host_async")
                       + " (pinned host inputs and output every step; two steps in flight: copies in, kernels, "
                         "copies out on three streams)"},
        "gpu_launches": int(launches),
        "clocks": clk,
    }
    if shared:
        res["kv_bytes_unique_per_step"] = kv_unique
        res["value_unique"] = round(kv_unique / (step_ms * 1e-3) / 1e9, 2)
        res["roofline"]["algorithmic_bytes_note"] = (
            "distinct (block, row) pairs read: the shared prompt blocks count once; the logical stream "
            f"({kv_bytes} B) re-reads them from L2")
        if traffic:
            res["roofline"]["dram_rate"] = round(traffic / (decode_ms * 1e-3) / 1e9, 2)
    if ablation is not None:
        res["placement_ablation"] = ablation
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, args.cpu_budget if headline else args.cpu_budget / 2)
    else:
        res["cpu_baseline"] = None
    del w, workspace, out, host
    gc.collect()
    torch.cuda.empty_cache()
    return res


def placement_ablation(w, args, dev, stream, decode, pt, n):
    """Context for the pages' "the paged kernel is 20-26% slower than a contiguous
    one" ("vLLM — 把操作系统的分页搬进 GPU KV cache", 踩过的坑): the same decode on
    the same bytes with every sequence's blocks laid out contiguously (identity
    order), the block-table reads alone (pkv_decode_table_scan, the decode grid),
    each timed with one event pair around n back-to-back launches."""
    import paged_kv_cache_450_b200 as pk
    s = w.spec
    tables = w.block_tables.cpu().numpy()
    order, new_tab = [], np.zeros_like(tables)
    for b, c in enumerate(w.ctx_list):
        nb = -(-c // s.block_size)
        new_tab[b, :nb] = np.arange(len(order), len(order) + nb)
        order.extend(int(x) for x in tables[b, :nb])
    idx = torch.tensor(order, dtype=torch.int64, device=dev)
    kc, vc = w.key_cache.index_select(0, idx), w.value_cache.index_select(0, idx)
    tab = torch.from_numpy(new_tab).to(dev)
    res = {}
    for name, (k_, v_, t_) in (("random_placement", (w.key_cache, w.value_cache, w.block_tables)),
                               ("contiguous_placement", (kc, vc, tab))):
        for _ in range(3):
            decode(k_, v_, t_)
        a, b = _events()
        a.record(stream)
        for _ in range(n):
            decode(k_, v_, t_)
        b.record(stream)
        torch.cuda.synchronize(dev)
        res[f"{name}_decode_ms"] = round(a.elapsed_time(b) / n, 5)
    sink = pk.decode_table_scan(w.block_tables, w.context_lens, s.num_kv_heads, s.block_size, w.num_blocks, pt,
                                stream=stream)
    a, b = _events()
    a.record(stream)
    for _ in range(n):
        pk.decode_table_scan(w.block_tables, w.context_lens, s.num_kv_heads, s.block_size, w.num_blocks, pt,
                             sink=sink, stream=stream)
    b.record(stream)
    torch.cuda.synchronize(dev)
    res["table_scan_ms"] = round(a.elapsed_time(b) / n, 5)
    res["table_scan_share_of_decode"] = round(res["table_scan_ms"] / res["random_placement_decode_ms"], 4)
    res["random_over_contiguous"] = round(res["random_placement_decode_ms"] / res["contiguous_placement_decode_ms"],
                                          4)
    res["note"] = ("same kernel and bytes; contiguous = each sequence's blocks at consecutive physical ids. "
                   "table_scan = the decode grid reading only its block ids (an upper bound: in the decode "
                   "those reads overlap the KV stream)")
    del kc, vc, tab, sink
    return res


# --------------------------------------------------------------------------- #
# the GPU arm: one multi-query workload
# --------------------------------------------------------------------------- #

def measure_multiquery(name, args, dev, rank, world, clocks):
    """Multi-query attention (draft verification / chunked prefill) timed alone."""
    import paged_kv_cache_450_b200 as pk

    spec, n = W.MQ_SPECS[name]
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
    T = int(mw.query_start_loc[-1])
    need = pk.multiquery_workspace_bytes(s.num_seqs, T, n, s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size,
                                         MB, s.cache_dtype, args.partition_tokens)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)

    def call():
        pk.paged_attention_multiquery(mw.q, w.key_cache, w.value_cache, w.block_tables, w.context_lens,
                                      mw.query_start_loc, w.scale, k_scale=w.k_scale, v_scale=w.v_scale, max_q_len=n,
                                      out=out, workspace=ws, partition_tokens=args.partition_tokens, stream=stream)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    steps = max(args.steps, 20)
    t0, t1 = _events()
    barrier(dev)
    launches0 = pk.launch_count()
    h0 = time.perf_counter()
    t0.record(stream)
    for _ in range(steps):
        call()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    h1 = time.perf_counter()
    launches = pk.launch_count() - launches0
    clk = clocks.window(h0, h1)
    step_ms = max_over_ranks(t0.elapsed_time(t1) / steps, dev)
    total_kv = sum_over_ranks(kv_bytes, dev)
    total_flops = sum_over_ranks(flops, dev)
    peak_gbs, gkind = hbm_peak()
    peak_tf, tkind = bf16_peak()
    gbs = kv_bytes / (step_ms * 1e-3) / 1e9
    tflops = flops / (step_ms * 1e-3) / 1e12
    tensor_bound = flops / max(kv_bytes, 1) > peak_tf * 1e12 / (peak_gbs * 1e9)
    tc = n * (s.num_q_heads // s.num_kv_heads) > 16  # the library's kernel split (both cache types)
    res = {
        "value": round(total_kv / (step_ms * 1e-3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(step_ms, 5),
        "steps": steps, "dtype": DTYPE_NAMES[s.cache_dtype],
        "tflops": round(total_flops / (step_ms * 1e-3) / 1e12, 2),
        "config": {"workload": s.name, "op": "paged_attention_multiquery (causal, queries = last q_len positions)",
                   "num_seqs_per_gpu": s.num_seqs, "q_len": n, "num_q_heads": s.num_q_heads,
                   "num_kv_heads": s.num_kv_heads, "head_dim": s.head_dim, "block_size": s.block_size,
                   "context_lens": list(s.ctx), "kv_bytes_per_step_per_gpu": kv_bytes, "flops_per_step": flops},
        "roofline": {"kernel": ("paged_multiquery_tc_kernel" if tc else "paged_multiquery_mma_kernel")
                               + (" + paged_multiquery_reduce_kernel" if need else ""),
                     "bound": "tensor" if tensor_bound else "hbm",
                     "achieved": round(tflops if tensor_bound else gbs, 2),
                     "peak": peak_tf if tensor_bound else peak_gbs,
                     "unit": "TFLOP/s" if tensor_bound else "GB/s",
                     "peak_kind": (f"{tkind} (burst bf16 GEMM)" if tensor_bound else f"{gkind} (burst copy bandwidth)"),
                     "frac": round((tflops / peak_tf) if tensor_bound else (gbs / peak_gbs), 4),
                     "timing": f"one CUDA event pair around {steps} back-to-back calls on their stream",
                     "traffic": None},
        "gpu_launches": int(launches), "clocks": clk,
    }
    del mw, w, out, ws
    gc.collect()
    torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------------------- #
# one companion operation alone (--op), for its own rate and its ncu summary
# --------------------------------------------------------------------------- #

OPS = ("kv_write", "block_copy", "swap", "amax", "table_scan")


def measure_op(op, args, dev):
    """Times one library call on the workload's tensors: K back-to-back calls
    captured in a CUDA graph and replayed between one CUDA event pair (device
    time; the eager loop of K calls is reported beside it, host launch cost
    included).  Bytes are the call's algorithmic bytes: read + written for the
    copies and the write, read for amax and the table scan."""
    import paged_kv_cache_450_b200 as pk

    spec = workload_spec(args)
    w = W.make_decode_workload(spec, seed=rank_seed(args.seed, 0), device=dev)
    s = spec
    stream = torch.cuda.current_stream(dev)
    blk = W.block_bytes(s.block_size, s.num_kv_heads, s.head_dim, s.cache_dtype)
    extra = {}
    if op == "kv_write":
        T = int(w.new_k.shape[0])
        row = s.num_kv_heads * s.head_dim
        nbytes = 2 * T * row * (W.elem_size(s.q_dtype) + W.elem_size(s.cache_dtype)) + T * 8

        def call():
            pk.paged_kv_write(w.new_k, w.new_v, w.slot_mapping, w.key_cache, w.value_cache, k_scale=w.k_scale,
                              v_scale=w.v_scale, stream=torch.cuda.current_stream(dev))
        kernel = "paged_kv_write_kernel"
    elif op == "block_copy":
        if w.copy_pairs is None:
            raise SystemExit("--op block_copy needs a workload with copy-on-write pairs")
        n = int(len(w.copy_pairs))
        nbytes = 2 * 2 * n * blk  # K and V, read + written

        def call():
            pk.kv_block_copy(w.copy_pairs, w.key_cache, w.value_cache, stream=torch.cuda.current_stream(dev))
        kernel = "kv_block_copy_kernel"
    elif op == "swap":
        n = min(args.swap_blocks, w.num_blocks)
        ids = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(args.seed))[:n]
        pairs_out = torch.stack([ids, torch.arange(n)], 1).to(dev)
        host_k = torch.empty((n,) + tuple(w.key_cache.shape[1:]), dtype=w.key_cache.dtype, pin_memory=True)
        host_v = torch.empty_like(host_k, pin_memory=True)
        nbytes = 2 * n * blk  # K and V over the host link, one direction

        def call():
            pk.swap_blocks(pairs_out, w.key_cache, w.value_cache, host_k, host_v, stream=torch.cuda.current_stream(dev))
        kernel = "kv_block_copy_kernel (device -> pinned host)"
        extra = {"blocks": n, "direction": "device to pinned host (swap out)"}
    elif op == "amax":
        if s.cache_dtype not in (torch.bfloat16, torch.float32):
            raise SystemExit("--op amax reads a bf16 or f32 tensor")
        x = w.key_cache.view(-1)
        nbytes = x.numel() * x.element_size()
        scale = torch.empty((1,), dtype=torch.float32, device=dev)

        def call():
            pk.fp8_scale_from_amax(x, out=scale, stream=torch.cuda.current_stream(dev))
        kernel = "amax_kernel + fp8_scale_finish_kernel"
    elif op == "table_scan":
        MB = w.block_tables.shape[1]
        pt = pk.decode_partition_tokens(s.num_seqs, s.num_q_heads, s.num_kv_heads, s.head_dim, s.block_size, MB,
                                        s.cache_dtype, args.partition_tokens)
        sink = pk.decode_table_scan(w.block_tables, w.context_lens, s.num_kv_heads, s.block_size, w.num_blocks, pt,
                                    stream=stream)
        nbytes = sum(-(-c // s.block_size) for c in w.ctx_list) * 4 * s.num_kv_heads  # id reads, all CTAs

        def call():
            pk.decode_table_scan(w.block_tables, w.context_lens, s.num_kv_heads, s.block_size, w.num_blocks, pt,
                                 sink=sink, stream=torch.cuda.current_stream(dev))
        kernel = "decode_table_scan_kernel"
        extra = {"partition_tokens": pt, "bytes_note": "block-id reads of every CTA (each KV head's CTAs re-read "
                                                      "the sequence's ids)"}
    else:
        raise SystemExit(f"unknown --op {op}")
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    a, b = _events()
    a.record(stream)
    for _ in range(args.steps):
        call()
    b.record(stream)
    torch.cuda.synchronize(dev)
    eager_ms = a.elapsed_time(b) / args.steps
    timing = "CUDA graph of the calls, replayed between one event pair"
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(args.steps):
                call()
        g.replay()
        torch.cuda.synchronize(dev)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms = a.elapsed_time(b) / args.steps
        del g
    except Exception as e:  # capture not possible here: the eager loop stands
        ms, timing = eager_ms, f"eager loop (graph capture failed: {type(e).__name__})"
    assert pk.device_status(clear=True) == 0
    return {"metric": f"{op} GB/s", "op": op, "kernel": kernel, "value": round(nbytes / (ms * 1e-3) / 1e9, 2),
            "unit": "GB/s", "ms_per_call": round(ms, 5), "eager_ms_per_call": round(eager_ms, 5),
            "timing": timing, "bytes_per_call": int(nbytes), "steps": args.steps, "warmup": args.warmup,
            "config": {"workload": s.name, **extra}}


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
    st = {"q": to_np(w.q), "kc": to_np(w.key_cache), "vc": to_np(w.value_cache),
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


def _oracle_rate(w, st, rb, order, threads, budget_s):
    """Whole rows in the seeded order until about budget_s seconds of oracle work."""
    done, t_used, nbytes, i = 0, 0.0, 0.0, 0
    chunk = max(threads, 2)
    while i < len(order) and t_used < budget_s:
        rows = order[i:i + chunk]
        t = time.perf_counter()
        _oracle_rows(w, st, rows, threads)
        t_used += time.perf_counter() - t
        nbytes += rb[rows].sum()
        done += len(rows)
        i += len(rows)
        chunk = min(chunk * 2, 4096)
    return nbytes / max(t_used, 1e-9) / 1e9, done, nbytes, t_used


def cpu_baseline(w, budget_s: float = 16.0):
    """The oracle as it stands, on this host's cores, over a bounded sample of
    the same workload: whole (sequence, query head) rows in a seeded order,
    with OpenMP over all cores and on one thread (each about budget_s / 2)."""
    threads = os.cpu_count() or 1
    st = _host_state(w)
    rb = _row_bytes(w)
    order = np.random.default_rng(0).permutation(len(rb))
    v_all, n_all, b_all, t_all = _oracle_rate(w, st, rb, order, threads, budget_s / 2)
    v_one, n_one, b_one, t_one = _oracle_rate(w, st, rb, order, 1, budget_s / 2)
    del st
    gc.collect()
    return {"value": round(v_all, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{n_all} of {len(rb)} (sequence, query head) rows of {w.spec.name} "
                      f"({b_all / 1e9:.3f} GB of logical KV) in {t_all:.1f} s, fp64 C oracle, OpenMP on "
                      f"{threads} threads",
            "single_thread": {"value": round(v_one, 4), "unit": "GB/s", "cores": 1,
                              "sample": f"{n_one} rows ({b_one / 1e9:.3f} GB of logical KV) in {t_one:.1f} s, "
                                        "the same oracle on one thread"}}


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
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.SPECS) + sorted(W.MQ_SPECS))
    ap.add_argument("--configs", default="auto", choices=["auto", "all", "none"],
                    help="also measure the other decode and multi-query workloads in this run (N = 1): "
                         "auto = when the headline is the default workload")
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--op", default="step", choices=("step",) + OPS,
                    help="time one companion operation alone on the workload's tensors instead of the step")
    ap.add_argument("--swap-blocks", type=int, default=4096, help="blocks moved by --op swap")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--partition-tokens", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=200, help="steps of the end-to-end (host buffers) timing")
    ap.add_argument("--cpu-budget", type=float, default=16.0,
                    help="seconds of oracle work for the headline's cpu_baseline (half for the other configs)")
    ap.add_argument("--ref-budget", type=float, default=90.0, help="seconds of oracle work for --impl reference")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-shared-prefix", action="store_true",
                    help="decode parallel-sampling workloads per sequence instead of reading shared prefixes once")
    ap.add_argument("--unfused", action="store_true",
                    help="write the new tokens with a separate paged_kv_write launch instead of inside the decode")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="override the workload's batch (a smaller case of the same shape, for profiling)")
    return ap.parse_args(argv)


def run_gpu(args, rank, world, local_rank):
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    clocks = ClockSampler(dev)
    clocks.start()
    try:
        common = {"metric": METRIC, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                  "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "data": "synthetic"}
        if args.workload in W.MQ_SPECS:
            r = measure_multiquery(args.workload, args, dev, rank, world, clocks)
            return {**common, "dtype": "bf16", **r, "cpu_baseline": None}
        spec = workload_spec(args)
        head = measure_decode(spec, args, dev, rank, world, clocks, headline=True)
        res = {**common, "dtype": DTYPE_NAMES[spec.cache_dtype], **head}
        run_configs = world == 1 and (args.configs == "all" or (args.configs == "auto" and
                                                                 args.workload == DEFAULT_WORKLOAD
                                                                 and not args.num_seqs))
        if run_configs:
            res["configs"] = {}
            for name in SECONDARY + ([DEFAULT_WORKLOAD] if args.workload != DEFAULT_WORKLOAD else []):
                if name == args.workload:
                    continue
                r = measure_decode(W.SPECS[name], args, dev, rank, world, clocks, headline=False)
                r["dtype"] = DTYPE_NAMES[W.SPECS[name].cache_dtype]
                res["configs"][name] = r
            res["multiquery"] = {name: measure_multiquery(name, args, dev, rank, world, clocks)
                                 for name in sorted(W.MQ_SPECS)}
        return res
    finally:
        clocks.stop()


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
    if args.op != "step":
        if world != 1:
            raise SystemExit("--op runs on one GPU")
        torch.cuda.set_device(0)
        print(json.dumps(measure_op(args.op, args, torch.device("cuda", 0))), flush=True)
        return
    try:
        res = run_gpu(args, rank, world, local_rank)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
