"""Benchmark of the absorbed-MLA hot path on B200.

One step = one full call of the path (q_norm → wq_b+RoPE → W_UK absorption → latent attention over
the cache → split merge → W_UV) on synthetic seeded inputs resident in HBM.  The default run times
every configuration of the method in turn:
  ragged_decode  B=64, H=128, cache lengths L_b ~ U{1024..32768}, residual RMSNorm  (headline:
                 the largest single-GPU configuration; top-level value / config)
  tiny_decode    B=2,  H=16,  L=128
  v32_decode     B=32, H=128, L=4096
  prefill_chunk  B=1,  T=2048 new tokens after 2048 cached, H=128 (causal), reported in TFLOP/s
  kimi_decode    B=128, H=64, L=2048
and prints ONE JSON line: the headline's numbers at top level and the others under "workloads".
Between timed steps L2 is flushed by writing a 256 MiB buffer and then reading another 256 MiB
buffer (both untimed): every step starts with none of its data in L2.  The timed steps replay a
CUDA graph of one C-ABI call on a dedicated stream (--no-graph: the eager call); the per-kernel
breakdown (roofline) and the end-to-end number use eager calls through the C ABI.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
        [--workload all|ragged_decode|tiny_decode|v32_decode|prefill_chunk|kimi_decode]
For N > 1 launch one process per GPU with torch.distributed.run; every rank runs its own replica
batch (the path shards by sequence with no exchange: weak scaling) and rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mla_synth import keys_per_row, make_inputs, workload  # noqa: E402

METRIC = "MLA decode queries/s + HBM GB/s (% peak); prefill-chunk TFLOP/s (% peak)"
FLUSH_BYTES = 256 << 20
HEADLINE = "ragged_decode"
WORKLOAD_ORDER = ("ragged_decode", "tiny_decode", "v32_decode", "prefill_chunk", "kimi_decode")
# variants of the path measured beside the configurations: name -> (workload, variant)
VARIANTS = {"v32_decode_fp8": ("v32_decode", "fp8"),
            "ragged_decode_top2048": ("ragged_decode", "top2048")}


# ------------------------------------------------------------------------------------------
# Algorithmic work of one step (bytes the method must move, flops it must do)
# ------------------------------------------------------------------------------------------
def algorithmic_work(w, start_pos: np.ndarray, fp8: bool = False, topk_len=None) -> dict:
    """Bytes and flops of one step.  ``fp8``: weights are one-byte codes plus one fp32 scale per
    128 x 128 block.  ``topk_len``: index-mask decode, row b attends topk_len[b] keys."""
    d = w.dims
    H, R, C, Dn, Dr, Dv = d.n_heads, d.q_lora_rank, d.kv_lora_rank, d.qk_nope_head_dim, d.qk_rope_head_dim, d.v_head_dim
    rows = w.batch * w.tokens
    keys = keys_per_row(w, start_pos)                      # [B, T] visible keys per query row
    if topk_len is not None:
        keys = np.asarray(topk_len, np.int64)[:, None]
    if w.mode == "decode":
        cache_rows = int(keys.sum())                       # each decode row reads its own keys
    else:
        cache_rows = int(keys[:, -1].sum())                # a chunk reads its cache prefix once
    act = rows * R * 2 * (3 if w.residual else 1) + rows * R * 2   # x (+res r/w) + y
    if fp8:
        weights = (H * (Dn + Dr) * R + H * (Dn + Dv) * C
                   + (H * (Dn + Dr) * R + H * (Dn + Dv) * C) // (128 * 128) * 4 + R * 4)
    else:
        weights = H * (Dn + Dr) * R * 2 + H * (Dn + Dv) * C * 2 + R * 4
    cache = cache_rows * (C + Dr) * 2
    out = rows * H * Dv * 2
    flops = (2 * rows * R * H * (Dn + Dr) + 2 * rows * H * Dn * C
             + 2 * int(keys.sum()) * H * ((C + Dr) + C) + 2 * rows * H * C * Dv)
    # the attention kernel's roofline counts only what the method must move: every cache row a
    # query attends crosses HBM once (the absorbed query and o_lat are intermediates of this build)
    attn_bytes = cache
    attn_flops = 2 * int(keys.sum()) * H * ((C + Dr) + C)
    return dict(bytes=act + weights + cache + out, flops=flops, cache_bytes=cache,
                weight_bytes=weights, attn_bytes=attn_bytes, attn_flops=attn_flops,
                keys=int(keys.sum()), rows=rows)


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# The attention kernel's part of k_attn.cu: everything before the combine kernel's section (the
# combine is a separate launch and does not change the attention's traffic).
ATTN_SOURCE_END = b"// Combine: rows cut between pairs merge"


def attention_source_sha256() -> str:
    """sha256 of the attention kernel's source region of k_attn.cu."""
    import hashlib
    src = os.path.join(ROOT, "head_latent_attention_11_b200", "csrc", "k_attn.cu")
    with open(src, "rb") as f:
        text = f.read()
    cut = text.find(ATTN_SOURCE_END)
    return hashlib.sha256(text[:cut] if cut >= 0 else text).hexdigest()


def profiled_traffic(workload_name: str):
    """DRAM bytes (read + write) of one attention launch from the committed ncu summary, or None
    when there is none for this workload or the kernel source changed since it was captured."""
    prof = os.path.join(ROOT, "profiles", f"latent_attention_{workload_name}.json")
    if not os.path.exists(prof):
        return None
    with open(prof) as f:
        d = json.load(f)
    if not attention_source_sha256().startswith(d.get("source_sha256_prefix", "-")):
        return None
    return int(d["dram_bytes_read"]) + int(d["dram_bytes_write"])


# ------------------------------------------------------------------------------------------
# Multi-rank aggregation (replicas: every rank runs its own batch, no data exchange)
# ------------------------------------------------------------------------------------------
def max_over_ranks(values, device="cpu"):
    """Element-wise max of per-rank float values over the default process group (a no-op when
    torch.distributed is not initialised).  Only timings cross ranks; the data path has no
    collective."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def aggregate_throughput(units_per_rank: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: all ranks' units over the slowest rank's timed region."""
    return world * units_per_rank * steps / (max_ms / 1e3)


# ------------------------------------------------------------------------------------------
# Clock sampling during the timed region
# ------------------------------------------------------------------------------------------
class ClockSampler:
    """Samples the SM clock and the clock-event reasons of one GPU from a background thread.

    NVML is polled every 5 ms (read-only queries); where NVML is unavailable, nvidia-smi's
    100 ms loop is used instead.  `mark(name)` stamps host times so that the summary can say
    how many samples fell inside the timed region proper."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.samples: list[tuple[float, float, set]] = []   # (host time, SM MHz, reasons)
        self.sm_max = None
        self.marks: dict[str, float] = {}
        self.source = None
        self._stop = threading.Event()
        self._t = None
        self.proc = None

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
        h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        return pynvml, h

    def start(self):
        try:
            nv, h = self._nvml_handle()
            bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                    "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                    "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                    "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            self.sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))

            def poll():
                while not self._stop.is_set():
                    mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                    mask = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                    self.samples.append((time.perf_counter(), mhz,
                                         {n for n, b in bits.items() if mask & b}))
                    time.sleep(0.005)

            self.source = "nvml, 5 ms"
            self._t = threading.Thread(target=poll, daemon=True)
            self._t.start()
            return
        except Exception:
            pass
        try:
            gpu = os.environ.get("CUDA_VISIBLE_DEVICES", str(self.dev)).split(",")[self.dev] or "0"
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi, 100 ms"
            self._t = threading.Thread(target=self._read_smi, daemon=True)
            self._t.start()
        except (FileNotFoundError, OSError, IndexError):
            self.proc = None

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz, self.sm_max = float(parts[1]), float(parts[2])
            except ValueError:
                continue
            self.samples.append((time.perf_counter(), mhz,
                                 {n for n, v in zip(self.REASONS, parts[5:9]) if v.lower() == "active"}))

    def mark(self, name: str) -> None:
        self.marks[name] = time.perf_counter()

    def stop(self) -> dict:
        if self.source is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["clock query unavailable"]}
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self._t is not None:
            self._t.join(timeout=5)
        lo = self.marks.get("load", float("-inf"))
        t0, t1 = self.marks.get("timed0", lo), self.marks.get("timed1", float("inf"))
        under_load = [s for s in self.samples if lo <= s[0] <= t1]
        timed = [s for s in under_load if s[0] >= t0]
        reasons = set().union(*[s[2] for s in under_load]) if under_load else set()
        return {"sm_mhz": statistics.median([s[1] for s in under_load]) if under_load else None,
                "sm_max_mhz": self.sm_max, "reasons": sorted(reasons),
                "samples": len(under_load), "samples_timed": len(timed),
                "source": self.source,
                "window": "untimed load steps (0.5 s) directly before the timed steps, then the timed steps"}


# ------------------------------------------------------------------------------------------
# Our arm
# ------------------------------------------------------------------------------------------
def run_workload(name: str, args, rank: int, world: int, local_rank: int,
                 variant: str | None = None, entry: str | None = None) -> dict | None:
    """Times one configuration on this rank's GPU; returns its JSON entry on rank 0 (None on the
    other ranks).  Every rank takes the same collective steps (two barriers, one all-reduce).
    ``variant``: "fp8" (FP8 block-scaled weights) or "top2048" (index-mask decode, 2048 seeded
    selected keys per sequence)."""
    import torch
    import torch.distributed as dist

    dev = f"cuda:{local_rank}"
    from head_latent_attention_11_b200 import (mla_enable_stage_timing, mla_last_launch_count,
                                               mla_stage_times)
    from head_latent_attention_11_b200.runtime import MLARuntime
    from mla_synth import make_fp8_weights, make_topk

    w = workload(name)
    inp = make_inputs(w, seed=args.seed + rank)
    topk = make_topk(inp["start_pos"], 2048, seed=args.seed + rank) if variant == "top2048" else None
    work = algorithmic_work(w, inp["start_pos"], fp8=variant == "fp8",
                            topk_len=None if topk is None else topk[1])
    B, T, H = w.batch, w.tokens, w.dims.n_heads

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    q_latent = bf16(inp["q_latent"])
    if w.mode == "decode":
        q_latent = q_latent.reshape(B, -1)
    residual = bf16(inp["residual"]) if inp["residual"] is not None else None
    if residual is not None and w.mode == "decode":
        residual = residual.reshape(B, -1)
    gamma = torch.from_numpy(inp["gamma"]).to(dev)
    cache = bf16(inp["cache"])
    start_pos = torch.from_numpy(inp["start_pos"].astype(np.int32)).to(dev)
    scales = {}
    if variant == "fp8":
        f8 = make_fp8_weights(w, seed=args.seed + rank)
        wq_b, wkv_b = torch.from_numpy(f8["wq_b"]).to(dev), torch.from_numpy(f8["wkv_b"]).to(dev)
        scales = dict(wq_b_scale=torch.from_numpy(f8["wq_b_scale"]).to(dev),
                      wkv_b_scale=torch.from_numpy(f8["wkv_b_scale"]).to(dev))
    else:
        wq_b, wkv_b = bf16(inp["wq_b"]), bf16(inp["wkv_b"])
    t_idx = t_len = None
    if topk is not None:
        t_idx, t_len = torch.from_numpy(topk[0]).to(dev), torch.from_numpy(topk[1]).to(dev)
    del inp
    rt = MLARuntime(gamma, wq_b, wkv_b, n_heads=H, max_rows=B * T, max_seq_len=cache.shape[1],
                    rope_theta=w.rope_theta, rms_eps=w.rms_eps, **scales)
    # the set-up kernels (workspace zeroing, W_UK^T copy) ran on the current stream; the timed
    # calls use a pool stream that does not wait for it
    torch.cuda.synchronize()
    out_shape = (B, H, 128) if w.mode == "decode" else (B, T, H, 128)
    out = torch.empty(out_shape, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    # a dedicated stream (the legacy default stream serialises with every other stream); torch's
    # flush kernels run on it too
    stream = torch.cuda.Stream(device=dev)
    prev_stream = torch.cuda.current_stream(dev)
    torch.cuda.set_stream(stream)

    def flush_l2(i: int) -> None:
        flush.fill_(float(i))   # evict everything the previous step left in L2 ...
        flush_rd.sum()          # ... and leave L2 holding clean lines of an unrelated buffer

    def step(q_in=None, sp=None):
        q_in = q_latent if q_in is None else q_in
        sp = start_pos if sp is None else sp
        if topk is not None:
            rt.decode_sparse(q_in, sp, t_idx, t_len, cache, residual=residual, out=out,
                             stream=stream)
        elif w.mode == "decode":
            rt.decode(q_in, sp, cache, residual=residual, out=out, stream=stream)
        else:
            rt.prefill(q_in, w.prefill_start, cache, residual=residual, out=out, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if rt.sync_status(stream) != 0:
        raise RuntimeError(f"{name}: device status set during warm-up")
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        graph.replay()
        torch.cuda.synchronize()
        if rt.sync_status(stream) != 0:
            raise RuntimeError(f"{name}: device status set by the captured step")
    run_step = graph.replay if graph is not None else step

    # ---- timed region: K steps, L2 flushed before each (flush not timed)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    clocks.start()
    # keep the GPU busy for ~0.5 s right before the timed steps (same flush + step, untimed) so
    # that the clock record holds samples taken under this load
    clocks.mark("load")
    t_load = time.perf_counter()
    while time.perf_counter() - t_load < 0.5:
        for i in range(16):
            flush_l2(i)
            run_step()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark("timed0")
    for i in range(args.steps):
        flush_l2(i)
        starts[i].record(stream)
        run_step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    clocks.mark("timed1")
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    launches = mla_last_launch_count(rt.ctx)
    if rt.sync_status(stream) != 0:
        raise RuntimeError(f"{name}: device status set during the timed steps")
    total_ms = float(sum(s.elapsed_time(e) for s, e in zip(starts, ends)))

    # ---- per-kernel breakdown: a separate pass of eager calls on the same stream with CUDA
    # events around every kernel (not part of `value`)
    mla_enable_stage_timing(rt.ctx, True)
    stage_acc: dict[str, list[float]] = {}
    for i in range(max(3, min(args.steps, 20))):
        flush_l2(i)
        step()
        for kname, ms in mla_stage_times(rt.ctx):
            stage_acc.setdefault(kname, []).append(ms)
    mla_enable_stage_timing(rt.ctx, False)
    stages = {k: float(np.mean(v)) for k, v in stage_acc.items()}

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the timed region
    h_q = torch.empty(q_latent.shape, dtype=torch.bfloat16, pin_memory=True)
    h_q.copy_(q_latent.cpu())
    h_sp = torch.empty(start_pos.shape, dtype=torch.int32, pin_memory=True)
    h_sp.copy_(start_pos.cpu())
    h_out = torch.empty(out.shape, dtype=torch.bfloat16, pin_memory=True)
    d_q = torch.empty_like(q_latent)
    d_sp = torch.empty_like(start_pos)
    e2e_ms = []
    for i in range(args.steps):
        flush_l2(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        d_q.copy_(h_q, non_blocking=True)
        d_sp.copy_(h_sp, non_blocking=True)
        step(d_q, d_sp)
        h_out.copy_(out, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        e2e_ms.append(e0.elapsed_time(e1))
    h2d = h_q.numel() * 2 + h_sp.numel() * 4
    d2h = h_out.numel() * 2

    # ---- max over ranks
    total_ms, e2e_total = max_over_ranks([total_ms, float(np.sum(e2e_ms))], device=dev)
    rt.close()
    torch.cuda.set_stream(prev_stream)
    del graph, rt, cache, wq_b, wkv_b, flush, flush_rd
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if rank != 0:
        return None

    peaks = measured_peaks()
    ms_per_step = total_ms / args.steps
    if w.mode == "decode":
        value = aggregate_throughput(B * T, args.steps, world, total_ms)
        unit = "queries/s"
        e2e_value = aggregate_throughput(B * T, args.steps, world, e2e_total)
    else:
        value = world * work["flops"] * args.steps / (total_ms / 1e3) / 1e12
        unit = "TFLOP/s"
        e2e_value = world * work["flops"] * args.steps / (e2e_total / 1e3) / 1e12
    attn_ms = stages.get("latent_attention")
    if w.mode == "decode":
        achieved = work["attn_bytes"] / (attn_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": profiled_traffic(entry or w.name), "kernel": "latent_attention",
                "algorithmic_bytes_per_launch": work["attn_bytes"],
                "algorithmic_bytes_rule": "cache rows attended x 1152 B (576 bf16)",
                "kernel_ms": round(attn_ms, 5),
                "peak_source": peaks["source"] + " (hbm_gbs, copy burst)"}
    else:
        achieved = work["attn_flops"] / (attn_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                "traffic": profiled_traffic(w.name), "kernel": "latent_attention",
                "algorithmic_flops_per_launch": work["attn_flops"],
                "algorithmic_flops_rule": "2 x visible (query, key) pairs x H x (576 + 512)",
                "kernel_ms": round(attn_ms, 5),
                "peak_source": peaks["source"] + " (bf16_tflops, burst: a kernel of a few ms)"}
    step_gbs = work["bytes"] / (ms_per_step / 1e3) / 1e9
    return {
        "value": round(value, 2), "unit": unit, "ms_per_step": round(ms_per_step, 5),
        "config": {"workload": entry or w.name, "batch": B, "tokens": T, "n_heads": H,
                   "weights": "fp8 e4m3, 128x128 block scales" if variant == "fp8" else "bf16",
                   "keys": "2048 selected per sequence (index mask)" if topk is not None else "all",
                   "cache_keys_per_step": work["keys"], "q_lora": 1536, "kv_lora": 512,
                   "rope": 64, "v": 128, "residual": bool(w.residual),
                   "l2": "flushed before every timed step: 256 MiB write, then 256 MiB read of another buffer (untimed)",
                   "launch": "eager C-ABI call" if args.no_graph else "CUDA graph of one C-ABI call, replayed on a dedicated stream",
                   "parallelism": f"replicas x{world} (sequence-sharded, no collective)"},
        "hbm": {"step_bytes": work["bytes"], "step_gbs": round(step_gbs, 1),
                "frac_of_peak": round(step_gbs / peaks["hbm_gbs"], 4)},
        "tflops_step": round(work["flops"] / (ms_per_step / 1e3) / 1e12, 2),
        "tensor_frac_of_peak": round(work["flops"] / (ms_per_step / 1e3) / 1e12 / peaks["bf16_tflops"], 4),
        "roofline": roof,
        "stages_ms": {k: round(v, 5) for k, v in stages.items()},
        "clocks": clk,
        "e2e": {"value": round(e2e_value, 2), "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_total / args.steps, 5)},
        "gpu_launches": launches * args.steps,
        "kernels_per_step": launches,
    }


# ------------------------------------------------------------------------------------------
# The cache producer (wq_a, wkv_a → kv_norm / key RoPE → cache rows), upstream of the path
# ------------------------------------------------------------------------------------------
PRODUCER_RUNS = {"cache_producer_decode": "v32_decode", "cache_producer_chunk": "prefill_chunk"}


def producer_work(w, dim: int) -> dict:
    d = w.dims
    rows = w.batch * w.tokens
    weights = (d.q_lora_rank + d.cache_width) * dim * 2 + d.kv_lora_rank * 4
    x = rows * dim * 2
    q_out = rows * d.q_lora_rank * 2
    cache_rows = rows * d.cache_width * 2
    flops = 2 * rows * dim * (d.q_lora_rank + d.cache_width)
    wq_a_bytes = d.q_lora_rank * dim * 2 + x + q_out           # the dominant (first) GEMM
    wq_a_flops = 2 * rows * dim * d.q_lora_rank
    return dict(bytes=weights + x + q_out + cache_rows, flops=flops, rows=rows,
                wq_a_bytes=wq_a_bytes, wq_a_flops=wq_a_flops)


def run_producer(name: str, args, rank: int, world: int, local_rank: int) -> dict | None:
    import torch
    import torch.distributed as dist
    from mla_synth import MODEL_DIM, make_producer_inputs

    dev = f"cuda:{local_rank}"
    from head_latent_attention_11_b200 import (mla_enable_stage_timing, mla_last_launch_count,
                                               mla_stage_times)
    from head_latent_attention_11_b200.runtime import MLARuntime

    w = workload(PRODUCER_RUNS[name])
    inp = make_inputs(w, seed=args.seed + rank)
    pin = make_producer_inputs(w, seed=args.seed + rank, dim=MODEL_DIM)
    work = producer_work(w, MODEL_DIM)
    B, T = w.batch, w.tokens

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    gamma = torch.from_numpy(inp["gamma"]).to(dev)
    wq_b, wkv_b, cache = bf16(inp["wq_b"]), bf16(inp["wkv_b"]), bf16(inp["cache"])
    start_pos = torch.from_numpy(inp["start_pos"].astype(np.int32)).to(dev)
    x = bf16(pin["x"])
    wq_a, wkv_a = bf16(pin["wq_a"]), bf16(pin["wkv_a"])
    kv_gain = torch.from_numpy(pin["kv_gain"]).to(dev)
    del inp, pin
    rt = MLARuntime(gamma, wq_b, wkv_b, n_heads=w.dims.n_heads, max_rows=B * T,
                    max_seq_len=cache.shape[1], rope_theta=w.rope_theta, rms_eps=w.rms_eps)
    rt.attach_producer(wq_a, wkv_a, kv_gain)
    torch.cuda.synchronize()   # set-up kernels ran on the current stream (see run_workload)
    q_lat = torch.empty(B, T, 1536, dtype=torch.bfloat16, device=dev)
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    prev_stream = torch.cuda.current_stream(dev)
    torch.cuda.set_stream(stream)

    def flush_l2(i: int) -> None:
        flush.fill_(float(i))
        flush_rd.sum()

    def step(xin=x, sp=start_pos):
        if w.mode == "decode":
            rt.produce(xin, cache, start_pos=sp, q_latent=q_lat, stream=stream)
        else:
            rt.produce(xin, cache, start_pos_host=w.prefill_start, q_latent=q_lat, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if rt.sync_status(stream) != 0:
        raise RuntimeError(f"{name}: device status set during warm-up")
    graph = None
    if not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        graph.replay()
        torch.cuda.synchronize()
    run_step = graph.replay if graph is not None else step
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    clocks.start()
    clocks.mark("load")
    t_load = time.perf_counter()
    while time.perf_counter() - t_load < 0.5:
        for i in range(16):
            flush_l2(i)
            run_step()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark("timed0")
    for i in range(args.steps):
        flush_l2(i)
        starts[i].record(stream)
        run_step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    clocks.mark("timed1")
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    launches = mla_last_launch_count(rt.ctx)
    if rt.sync_status(stream) != 0:
        raise RuntimeError(f"{name}: device status set during the timed steps")
    total_ms = float(sum(s_.elapsed_time(e) for s_, e in zip(starts, ends)))
    mla_enable_stage_timing(rt.ctx, True)
    stage_acc: dict[str, list[float]] = {}
    for i in range(max(3, min(args.steps, 20))):
        flush_l2(i)
        step()
        for kname, ms in mla_stage_times(rt.ctx):
            stage_acc.setdefault(kname, []).append(ms)
    mla_enable_stage_timing(rt.ctx, False)
    stages = {k: float(np.mean(v)) for k, v in stage_acc.items()}
    # end to end: x and positions from pinned host memory, the query latent back to the host
    h_x = torch.empty(x.shape, dtype=torch.bfloat16, pin_memory=True)
    h_x.copy_(x.cpu())
    h_sp = torch.empty(start_pos.shape, dtype=torch.int32, pin_memory=True)
    h_sp.copy_(start_pos.cpu())
    h_q = torch.empty(q_lat.shape, dtype=torch.bfloat16, pin_memory=True)
    d_x, d_sp = torch.empty_like(x), torch.empty_like(start_pos)
    e2e_ms = []
    for i in range(args.steps):
        flush_l2(i)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        d_x.copy_(h_x, non_blocking=True)
        d_sp.copy_(h_sp, non_blocking=True)
        step(d_x, d_sp)
        h_q.copy_(q_lat, non_blocking=True)
        e1.record(stream)
        e1.synchronize()
        e2e_ms.append(e0.elapsed_time(e1))
    h2d = h_x.numel() * 2 + h_sp.numel() * 4
    d2h = h_q.numel() * 2
    total_ms, e2e_total = max_over_ranks([total_ms, float(np.sum(e2e_ms))], device=dev)
    rt.close()
    torch.cuda.set_stream(prev_stream)
    del graph, rt, cache, wq_b, wkv_b, wq_a, wkv_a, flush, flush_rd
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    if rank != 0:
        return None
    peaks = measured_peaks()
    ms_per_step = total_ms / args.steps
    rows = work["rows"]
    value = aggregate_throughput(rows, args.steps, world, total_ms)
    e2e_value = aggregate_throughput(rows, args.steps, world, e2e_total)
    k_ms = stages.get("wq_a")
    if w.mode == "decode":
        achieved = work["wq_a_bytes"] / (k_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": None,
                "kernel": "wq_a GEMM", "algorithmic_bytes_per_launch": work["wq_a_bytes"],
                "algorithmic_bytes_rule": "wq_a weights + x + q_latent out",
                "kernel_ms": round(k_ms, 5),
                "peak_source": peaks["source"] + " (hbm_gbs, copy burst)"}
    else:
        achieved = work["wq_a_flops"] / (k_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4),
                "traffic": None, "kernel": "wq_a GEMM",
                "algorithmic_flops_per_launch": work["wq_a_flops"],
                "algorithmic_flops_rule": "2 x tokens x 7168 x 1536",
                "kernel_ms": round(k_ms, 5),
                "peak_source": peaks["source"] + " (bf16_tflops, burst)"}
    step_gbs = work["bytes"] / (ms_per_step / 1e3) / 1e9
    return {
        "value": round(value, 2), "unit": "tokens/s", "ms_per_step": round(ms_per_step, 5),
        "config": {"workload": name, "batch": B, "tokens": T, "dim": MODEL_DIM,
                   "writes": "kv_cache / pe_cache rows at each token's position",
                   "l2": "flushed before every timed step (untimed)",
                   "launch": "CUDA graph of one C-ABI call" if not args.no_graph else "eager C-ABI call",
                   "parallelism": f"replicas x{world}"},
        "hbm": {"step_bytes": work["bytes"], "step_gbs": round(step_gbs, 1),
                "frac_of_peak": round(step_gbs / peaks["hbm_gbs"], 4)},
        "tflops_step": round(work["flops"] / (ms_per_step / 1e3) / 1e12, 2),
        "roofline": roof,
        "stages_ms": {k: round(v, 5) for k, v in stages.items()},
        "clocks": clk,
        "e2e": {"value": round(e2e_value, 2), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_total / args.steps, 5)},
        "gpu_launches": launches * args.steps,
        "kernels_per_step": launches,
    }


def producer_oracle_sample(name: str, budget_s: float) -> dict:
    from mla_synth import MODEL_DIM, bf16_bits_to_f64, make_producer_inputs
    import oracle
    w = workload(PRODUCER_RUNS[name])
    pin = make_producer_inputs(w, seed=0, dim=MODEL_DIM)
    x = bf16_bits_to_f64(pin["x"]).reshape(w.batch * w.tokens, -1)
    wq_a, wkv_a = bf16_bits_to_f64(pin["wq_a"]), bf16_bits_to_f64(pin["wkv_a"])
    gain = pin["kv_gain"].astype(np.float64)
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        cores = 1
    done, t0 = 0, time.perf_counter()
    while True:
        r = done % x.shape[0]
        oracle.produce_latents(x[r:r + 1], wq_a, wkv_a, gain, np.array([r]))
        done += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    return dict(value=round(done / el, 4), unit="tokens/s", cores=cores, kind="oracle",
                sample=f"{done} single-token producer calls (cycling over {x.shape[0]} tokens) in {el:.1f} s")


# ------------------------------------------------------------------------------------------
# CPU legs: the fp64 oracle on the host cores (bounded sample)
# ------------------------------------------------------------------------------------------
def oracle_sample(w, inp, budget_s: float, max_rows: int | None = None) -> dict:
    """Run the oracle on query rows 0, 1, ... (cycling over the batch) until ~budget_s of CPU
    time; returns the rate in the workload's unit."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from mla_cases import oracle_decode, oracle_prefill
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        cores = 1
    done, t0 = 0, time.perf_counter()
    if w.mode == "decode":
        while True:
            oracle_decode(inp, w, rows=[done % w.batch])
            done += 1
            if time.perf_counter() - t0 >= budget_s or (max_rows and done >= max_rows):
                break
        el = time.perf_counter() - t0
        return dict(value=done / el, unit="queries/s", cores=cores,
                    sample=f"{done} decode rows (cycling over the {w.batch} sequences, all "
                           f"{w.dims.n_heads} heads) in {el:.1f} s")
    T = w.tokens
    work = algorithmic_work(w, inp["start_pos"])
    per_token = work["flops"] / T
    while True:
        oracle_prefill(inp, w, tokens=[(done * 97) % T])
        done += 1
        if time.perf_counter() - t0 >= budget_s or (max_rows and done >= max_rows):
            break
    el = time.perf_counter() - t0
    return dict(value=done * per_token / el / 1e12, unit="TFLOP/s", cores=cores,
                sample=f"{done} chunk tokens (of {T}, all {w.dims.n_heads} heads; flops "
                       f"credited at the chunk's mean per token) in {el:.1f} s")


def run_reference(args) -> dict:
    name = HEADLINE if args.workload == "all" else args.workload
    w = workload(name)
    inp = make_inputs(w, seed=args.seed)
    per_step = []
    res = None
    for _ in range(args.warmup):
        oracle_sample(w, inp, budget_s=0.0, max_rows=1)
    # each step is a bounded sample; the whole run stays within about two minutes of oracle time
    step_s = min(args.ref_step_seconds, max(0.5, 120.0 / max(1, args.steps)))
    for _ in range(args.steps):
        res = oracle_sample(w, inp, budget_s=step_s)
        per_step.append(res["value"])
    value = float(np.mean(per_step))
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": res["unit"],
        "n_gpus": 0, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "tokens": w.tokens,
                   "n_heads": w.dims.n_heads},
        "cpu_baseline": {"kind": "oracle", "cores": res["cores"], "sample": res["sample"],
                         "value": round(value, 4), "unit": res["unit"]},
        "e2e": {"value": round(value, 4), "unit": res["unit"], "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="all", choices=("all",) + WORKLOAD_ORDER)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--cpu-seconds", type=float, default=8.0,
                    help="budget of each workload's oracle CPU-baseline sample")
    ap.add_argument("--ref-step-seconds", type=float, default=6.0,
                    help="oracle time per step of --impl reference (capped so that all steps "
                         "together take about two minutes)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time the eager C-ABI call instead of a CUDA-graph replay of it")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    import torch
    torch.cuda.set_device(local_rank)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    from head_latent_attention_11_b200 import build
    build.build()

    names = WORKLOAD_ORDER if args.workload == "all" else (args.workload,)
    entries = {n: run_workload(n, args, rank, world, local_rank) for n in names}
    if args.workload == "all":
        # the variants and the producer are measured beside the configurations; a failure in one
        # of them is reported in its entry instead of voiding the line
        def guarded(fn, *a, **kw):
            try:
                return fn(*a, **kw)
            except Exception as e:  # noqa: BLE001
                return {"error": f"{type(e).__name__}: {e}"[:300], "gpu_launches": 0}
        for n, (base, variant) in VARIANTS.items():
            entries[n] = guarded(run_workload, base, args, rank, world, local_rank,
                                 variant=variant, entry=n)
        for n in PRODUCER_RUNS:
            entries[n] = guarded(run_producer, n, args, rank, world, local_rank)
    if rank == 0:
        head_name = names[0]
        head = entries[head_name]
        if not args.no_cpu_baseline and world == 1:
            for n in names:
                w = workload(n)
                cb = oracle_sample(w, make_inputs(w, seed=args.seed), budget_s=args.cpu_seconds)
                entries[n]["cpu_baseline"] = {"value": round(cb["value"], 4), "unit": cb["unit"],
                                              "cores": cb["cores"], "kind": "oracle",
                                              "sample": cb["sample"]}
        line = {
            "metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) latents/caches/residual, N(0,1/fan_in) weights, "
                    "U(0.5,1.5) gain)",
        }
        line.update({k: v for k, v in head.items() if k not in ("value", "unit", "ms_per_step")})
        line["gpu_launches"] = sum(e["gpu_launches"] for e in entries.values() if e)
        line["gpu_launches_note"] = ("kernels of this library launched in the timed steps of "
                                     "every workload below (headline included)")
        if not args.no_cpu_baseline and world == 1 and args.workload == "all":
            for n in PRODUCER_RUNS:
                if entries[n] and "error" not in entries[n]:
                    entries[n]["cpu_baseline"] = producer_oracle_sample(n, min(4.0, args.cpu_seconds))
        if len(names) > 1:
            line["workloads"] = {n: entries[n] for n in entries if n != head_name}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
