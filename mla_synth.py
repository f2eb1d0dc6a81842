"""Seeded synthetic inputs for the absorbed multi-head latent attention (MLA) path.

This module is shared by the CPU oracle's tests, the GPU parity tests, ``bench.py`` and the smoke
entry.  It holds no arithmetic of the method itself: it draws random numbers, rounds them to
bfloat16 bit patterns (round-to-nearest-even) and lays them out in the tensors the method reads.

Tensors follow the pages' names (DeepSeek-V3.2-Exp "Query heads" and "Attention update" pages,
Kimi-K2 "value_states" page):

* ``q_latent``  [B, T, q_lora]            bf16   the query latent c^Q (input of q_norm)
* ``residual``  [B, T, q_lora]            bf16   optional residual fused into q_norm
* ``gamma``     [q_lora]                  fp32   q_norm gain
* ``wq_b``      [H*(nope+rope), q_lora]   bf16   nn.Linear layout [out, in]
* ``wkv_b``     [H*(nope+v), kv_lora]     bf16   nn.Linear layout [out, in]; per head, the first
                                                 ``nope`` rows are W_UK, the last ``v`` rows W_UV
* ``cache``     [B, max_t, kv_lora+rope]  bf16   packed latent cache: columns [0, kv_lora) are the
                                                 kv_cache latents, [kv_lora, kv_lora+rope) the
                                                 (already rotated) pe_cache key
* ``start_pos`` [B] int32 — decode: the new token sits at cache row start_pos[b] and attends keys
                 0..start_pos[b]; prefill: one shared start position, tokens at start_pos + t.

Distributions (one seed per workload): q_latent, residual, cache ~ N(0, 1); gamma ~ U(0.5, 1.5);
wq_b ~ N(0, 1/q_lora); wkv_b ~ N(0, 1/kv_lora) (variance 1/fan_in).  Cache rows past the last key
a sequence may attend are filled with ``tail`` ("zero" or "nan"), so a kernel that reads past the
boundary shows up as a parity failure.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = [
    "MLADims", "Workload", "WORKLOADS", "workload", "make_inputs", "make_producer_inputs",
    "make_topk", "make_fp8_weights", "make_wo",
    "f32_to_bf16_bits", "bf16_bits_to_f32", "bf16_bits_to_f64", "MODEL_DIM",
]

# Model width of the pages' models (the attention update is [B, 1, 7168] on the V3.2 page; the
# Kimi-K2 hidden size is the same): the input width of the cache producer.
MODEL_DIM = 7168


# --------------------------------------------------------------------------------------------
# bfloat16 bit-pattern conversion (data marshalling, not part of the method)
# --------------------------------------------------------------------------------------------
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even) and return the uint16 patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    r = ((u + np.uint32(0x7FFF) + ((u >> 16) & np.uint32(1))) >> 16).astype(np.uint16)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 patterns to float64."""
    return bf16_bits_to_f32(b).astype(np.float64)


# --------------------------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class MLADims:
    n_heads: int
    q_lora_rank: int = 1536
    kv_lora_rank: int = 512
    qk_nope_head_dim: int = 128
    qk_rope_head_dim: int = 64
    v_head_dim: int = 128

    @property
    def qk_head_dim(self) -> int:
        return self.qk_nope_head_dim + self.qk_rope_head_dim

    @property
    def cache_width(self) -> int:
        return self.kv_lora_rank + self.qk_rope_head_dim


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload.  ``mode`` is "decode" (T = 1, per-sequence start_pos) or "prefill"
    (T new tokens appended after one shared start_pos, causal)."""
    name: str
    dims: MLADims
    batch: int
    mode: str                       # "decode" | "prefill"
    tokens: int = 1                 # T
    cache_len: int | None = None    # decode: L, the new token's row (uniform lengths)
    ragged: tuple[int, int] | None = None   # decode: L_b ~ U{lo..hi} drawn from the seed
    prefill_start: int = 0          # prefill: start_pos
    residual: bool = False
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6

    @property
    def softmax_scale(self) -> float:
        return float(self.dims.qk_head_dim) ** -0.5


WORKLOADS: dict[str, Workload] = {
    # Tiny MLA decode: B=2, cache L=128 (keys 0..128), H=16.
    "tiny_decode": Workload("tiny_decode", MLADims(16), batch=2, mode="decode", cache_len=128),
    # DeepSeek-V3.2-shaped decode: B=32, H=128, L=4096.
    "v32_decode": Workload("v32_decode", MLADims(128), batch=32, mode="decode", cache_len=4096),
    # Ragged long-context decode: B=64, H=128, L_b ~ U{1024..32768}, residual-add RMSNorm.
    "ragged_decode": Workload("ragged_decode", MLADims(128), batch=64, mode="decode",
                              ragged=(1024, 32768), residual=True),
    # Prefill chunk: B=1, T=2048 after start_pos=2048, H=128 (causal over 4096 keys).
    "prefill_chunk": Workload("prefill_chunk", MLADims(128), batch=1, mode="prefill",
                              tokens=2048, prefill_start=2048),
    # Kimi-K2-shaped decode: B=128, H=64, L=2048.
    "kimi_decode": Workload("kimi_decode", MLADims(64), batch=128, mode="decode", cache_len=2048),
}


def workload(name: str, **overrides) -> Workload:
    """A named workload, optionally with fields replaced (e.g. a smaller batch for a test)."""
    w = WORKLOADS[name]
    return dataclasses.replace(w, **overrides) if overrides else w


# --------------------------------------------------------------------------------------------
# Generation
# --------------------------------------------------------------------------------------------
def _normal_bf16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    a = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return f32_to_bf16_bits(a)


def _start_positions(w: Workload, rng: np.random.Generator) -> np.ndarray:
    if w.mode == "prefill":
        return np.full(w.batch, w.prefill_start, dtype=np.int32)
    if w.ragged is not None:
        lo, hi = w.ragged
        return rng.integers(lo, hi + 1, size=w.batch, dtype=np.int64).astype(np.int32)
    return np.full(w.batch, int(w.cache_len), dtype=np.int32)


def keys_per_row(w: Workload, start_pos: np.ndarray) -> np.ndarray:
    """Number of keys each query row attends: [B, T] (start_pos + t + 1)."""
    t = np.arange(w.tokens, dtype=np.int64)
    return start_pos.astype(np.int64)[:, None] + t[None, :] + 1


def make_inputs(w: Workload, seed: int = 0, tail: str = "zero", max_t: int | None = None,
                threads: int | None = None) -> dict:
    """Draw every input of workload ``w`` from ``seed``.

    Returns a dict of numpy arrays (bf16 tensors as uint16 bit patterns) plus ``n_keys`` [B]
    (keys visible to the last token of each sequence) and ``max_t`` (cache rows per sequence).
    """
    d = w.dims
    root = np.random.SeedSequence(seed)
    s_pos, s_q, s_r, s_g, s_wq, s_wkv, s_cache = root.spawn(7)
    start_pos = _start_positions(w, np.random.default_rng(s_pos))
    n_keys = start_pos.astype(np.int64) + w.tokens           # keys of the last query of each row
    if max_t is None:
        max_t = max(64, int(n_keys.max()))   # the library wants at least 64 cache rows
    if max_t < int(n_keys.max()):
        raise ValueError("max_t smaller than the longest sequence")

    B, T = w.batch, w.tokens
    out = {
        "start_pos": start_pos,
        "n_keys": n_keys,
        "max_t": max_t,
        "q_latent": _normal_bf16(np.random.default_rng(s_q), (B, T, d.q_lora_rank)),
        "residual": (_normal_bf16(np.random.default_rng(s_r), (B, T, d.q_lora_rank))
                     if w.residual else None),
        "gamma": np.random.default_rng(s_g).uniform(0.5, 1.5, d.q_lora_rank).astype(np.float32),
        "wq_b": _normal_bf16(np.random.default_rng(s_wq),
                             (d.n_heads * d.qk_head_dim, d.q_lora_rank), d.q_lora_rank ** -0.5),
        "wkv_b": _normal_bf16(np.random.default_rng(s_wkv),
                              (d.n_heads * (d.qk_nope_head_dim + d.v_head_dim), d.kv_lora_rank),
                              d.kv_lora_rank ** -0.5),
    }

    cache = np.empty((B, max_t, d.cache_width), dtype=np.uint16)
    fill = {"zero": 0x0000, "nan": 0x7FC0}[tail]
    child = s_cache.spawn(B)

    def fill_row(b: int) -> None:
        n = int(n_keys[b])
        cache[b, :n] = _normal_bf16(np.random.default_rng(child[b]), (n, d.cache_width))
        cache[b, n:] = fill

    nthreads = threads or min(B, os.cpu_count() or 1)
    if nthreads > 1 and B > 1:
        with ThreadPoolExecutor(nthreads) as ex:
            list(ex.map(fill_row, range(B)))
    else:
        for b in range(B):
            fill_row(b)
    out["cache"] = cache
    return out


def make_producer_inputs(w: Workload, seed: int = 0, dim: int = MODEL_DIM) -> dict:
    """Inputs of the cache producer for workload ``w``'s new tokens, from their own seed stream
    (so ``make_inputs`` is unchanged): ``x`` [B, T, dim] bf16 ~ N(0, 1); ``wq_a`` [q_lora, dim] and
    ``wkv_a`` [kv_lora + rope, dim] bf16 ~ N(0, 1/dim) (nn.Linear [out, in]); ``kv_gain``
    [kv_lora] fp32 ~ U(0.5, 1.5)."""
    d = w.dims
    s_x, s_q, s_kv, s_g = np.random.SeedSequence([seed, 0x70726F64]).spawn(4)
    return {
        "dim": dim,
        "x": _normal_bf16(np.random.default_rng(s_x), (w.batch, w.tokens, dim)),
        "wq_a": _normal_bf16(np.random.default_rng(s_q), (d.q_lora_rank, dim), dim ** -0.5),
        "wkv_a": _normal_bf16(np.random.default_rng(s_kv), (d.cache_width, dim), dim ** -0.5),
        "kv_gain": np.random.default_rng(s_g).uniform(0.5, 1.5, d.kv_lora_rank).astype(np.float32),
    }


def make_topk(start_pos: np.ndarray, k: int, seed: int = 0):
    """A seeded stand-in for an indexer's top-k: for sequence b, min(k, start_pos[b] + 1)
    distinct key indices drawn uniformly from [0, start_pos[b]], in random order.  Returns
    (idx [B, k] int32 padded with -1, lengths [B] int32)."""
    B = len(start_pos)
    idx = np.full((B, k), -1, dtype=np.int32)
    lens = np.empty(B, dtype=np.int32)
    children = np.random.SeedSequence([seed, 0x746F706B]).spawn(B)
    for b in range(B):
        n = int(start_pos[b]) + 1
        m = min(k, n)
        rng = np.random.default_rng(children[b])
        idx[b, :m] = rng.choice(n, size=m, replace=False)
        lens[b] = m
    return idx, lens


def make_fp8_weights(w: Workload, seed: int = 0) -> dict:
    """wq_b and wkv_b of workload ``w`` as a checkpoint would store them in FP8: E4M3 codes
    (uint8, nn.Linear layout [out, in]) with one fp32 scale per 128 x 128 block.  Codes: N(0, 1)
    draws times 16 rounded to E4M3 (torch's float8_e4m3fn conversion, round to nearest even);
    scales U(0.75, 1.25) / (16 sqrt(fan_in)), so the dequantised weights have about the variance
    1/fan_in of the bf16 weights."""
    import torch
    d = w.dims
    out = {}
    for tag, (name, rows, cols) in enumerate((
            ("wq_b", d.n_heads * d.qk_head_dim, d.q_lora_rank),
            ("wkv_b", d.n_heads * (d.qk_nope_head_dim + d.v_head_dim), d.kv_lora_rank))):
        rng = np.random.default_rng(np.random.SeedSequence([seed, 0x66703800 + tag]))
        v = rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(16.0)
        out[name] = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        out[name + "_scale"] = (rng.uniform(0.75, 1.25, (rows // 128, cols // 128))
                                / (16.0 * np.sqrt(cols))).astype(np.float32)
    return out


def make_wo(w: Workload, seed: int = 0, dim: int = MODEL_DIM) -> np.ndarray:
    """The output projection wo [dim, H*v] bf16 ~ N(0, 1/(H*v)) (nn.Linear [out, in])."""
    d = w.dims
    fan_in = d.n_heads * d.v_head_dim
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x776F]))
    return _normal_bf16(rng, (dim, fan_in), fan_in ** -0.5)
