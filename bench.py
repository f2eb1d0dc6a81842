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


# ------------------------------------------------------------------------------------------
# Algorithmic work of one step (bytes the method must move, flops it must do)
# ------------------------------------------------------------------------------------------
def algorithmic_work(w, start_pos: np.ndarray) -> dict:
    d = w.dims
    H, R, C, Dn, Dr, Dv = d.n_heads, d.q_lora_rank, d.kv_lora_rank, d.qk_nope_head_dim, d.qk_rope_head_dim, d.v_head_dim
    rows = w.batch * w.tokens
    keys = keys_per_row(w, start_pos)                      # [B, T] visible keys per query row
    if w.mode == "decode":
        cache_rows = int(keys.sum())                       # each decode row reads its own keys
    else:
        cache_rows = int(keys[:, -1].sum())                # a chunk reads its cache prefix once
    act = rows * R * 2 * (3 if w.residual else 1) + rows * R * 2   # x (+res r/w) + y
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


def profiled_traffic(workload_name: str):
    """DRAM bytes (read + write) of one attention launch from the committed ncu summary, or None
    when there is none for this workload or the kernel source changed since it was captured."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", f"latent_attention_{workload_name}.json")
    src = os.path.join(ROOT, "head_latent_attention_11_b200", "csrc", "k_attn.cu")
    if not (os.path.exists(prof) and os.path.exists(src)):
        return None
    with open(prof) as f:
        d = json.load(f)
    with open(src, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    if not sha.startswith(d.get("source_sha256_prefix", "-")):
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
def run_workload(name: str, args, rank: int, world: int, local_rank: int) -> dict | None:
    """Times one configuration on this rank's GPU; returns its JSON entry on rank 0 (None on the
    other ranks).  Every rank takes the same collective steps (two barriers, one all-reduce)."""
    import torch
    import torch.distributed as dist

    dev = f"cuda:{local_rank}"
    from head_latent_attention_11_b200 import (mla_enable_stage_timing, mla_last_launch_count,
                                               mla_stage_times)
    from head_latent_attention_11_b200.runtime import MLARuntime

    w = workload(name)
    inp = make_inputs(w, seed=args.seed + rank)
    work = algorithmic_work(w, inp["start_pos"])
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
    wq_b, wkv_b, cache = bf16(inp["wq_b"]), bf16(inp["wkv_b"]), bf16(inp["cache"])
    start_pos = torch.from_numpy(inp["start_pos"].astype(np.int32)).to(dev)
    del inp
    rt = MLARuntime(gamma, wq_b, wkv_b, n_heads=H, max_rows=B * T, max_seq_len=cache.shape[1],
                    rope_theta=w.rope_theta, rms_eps=w.rms_eps)
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

    def step():
        if w.mode == "decode":
            rt.decode(q_latent, start_pos, cache, residual=residual, out=out, stream=stream)
        else:
            rt.prefill(q_latent, w.prefill_start, cache, residual=residual, out=out,
                       stream=stream)

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
        if w.mode == "decode":
            rt.decode(d_q, d_sp, cache, residual=residual, out=out, stream=stream)
        else:
            rt.prefill(d_q, w.prefill_start, cache, residual=residual, out=out, stream=stream)
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
                "traffic": profiled_traffic(w.name), "kernel": "latent_attention",
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
        "config": {"workload": w.name, "batch": B, "tokens": T, "n_heads": H,
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
        line["gpu_launches"] = sum(e["gpu_launches"] for e in entries.values())
        line["gpu_launches_note"] = ("kernels of this library launched in the timed steps of "
                                     "every workload below (headline included)")
        if len(names) > 1:
            line["workloads"] = {n: entries[n] for n in names[1:]}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
