"""Helpers shared by the GPU parity tests: move seeded inputs to the device, run the library
through the C ABI, run the oracle on the same bf16 values and compare within the stated bounds.

Tolerances (stated for the path): bf16 outputs |err| <= 1e-2 * max|ref| + 1e-3; softmax
probabilities within 1e-3 absolute.
"""
from __future__ import annotations

import numpy as np

import oracle
from mla_synth import bf16_bits_to_f64, make_inputs, workload

REL_TOL = 1e-2
ABS_TOL = 1e-3
PROB_TOL = 1e-3
# lse is compared with the oracle run on the same bf16-rounded queries ("bf16" query mode): what
# is left is fp32 arithmetic on the GPU — scores accumulated in fp32 from bf16 operands (relative
# error <= 576 * 2^-24 of sum|q_c k_c| * scale, about 4e-4 for these inputs), the hardware exp2 /
# log2 (relative error ~2^-22) and the fp32 split merge — so 2e-3 absolute is a bound with margin.
LSE_ATOL = 2e-3
LSE_RTOL = 0.0


def assert_close_bf16(got: np.ndarray, ref: np.ndarray, what: str, rel=REL_TOL, abs_=ABS_TOL):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} vs {ref.shape}"
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    bound = rel * float(np.max(np.abs(ref))) + abs_
    err = float(np.max(np.abs(got - ref)))
    assert err <= bound, f"{what}: max|err| {err:.3e} > bound {bound:.3e}"
    return err, bound


def to_device(inp: dict, device="cuda"):
    import torch

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)

    d = {
        "q_latent": bf16(inp["q_latent"]),
        "residual": None if inp["residual"] is None else bf16(inp["residual"]),
        "gamma": torch.from_numpy(inp["gamma"]).to(device),
        "wq_b": bf16(inp["wq_b"]),
        "wkv_b": bf16(inp["wkv_b"]),
        "cache": bf16(inp["cache"]),
        "start_pos": torch.from_numpy(inp["start_pos"].astype(np.int32)).to(device),
    }
    return d


def bf16_to_np(t) -> np.ndarray:
    import torch
    return t.detach().to("cpu").view(torch.int16).numpy().view(np.uint16)


def f64(t) -> np.ndarray:
    return bf16_bits_to_f64(bf16_to_np(t))


def oracle_decode(inp: dict, w, rows=None, **kw):
    d = w.dims
    return oracle.decode(
        bf16_bits_to_f64(inp["q_latent"][:, 0]), inp["gamma"].astype(np.float64),
        bf16_bits_to_f64(inp["wq_b"]), bf16_bits_to_f64(inp["wkv_b"]), _CacheView(inp["cache"]),
        inp["start_pos"], d.n_heads,
        residual=None if inp["residual"] is None else bf16_bits_to_f64(inp["residual"][:, 0]),
        theta=w.rope_theta, eps=w.rms_eps, rows=rows, **kw)


def oracle_prefill(inp: dict, w, tokens=None, **kw):
    d = w.dims
    # the chunk's cache prefix is small: widen it once instead of per token
    n = int(inp["start_pos"][0]) + w.tokens
    cache = bf16_bits_to_f64(inp["cache"][:, :n])
    return oracle.prefill(
        bf16_bits_to_f64(inp["q_latent"]), inp["gamma"].astype(np.float64),
        bf16_bits_to_f64(inp["wq_b"]), bf16_bits_to_f64(inp["wkv_b"]), cache,
        int(inp["start_pos"][0]), d.n_heads,
        residual=None if inp["residual"] is None else bf16_bits_to_f64(inp["residual"]),
        theta=w.rope_theta, eps=w.rms_eps, tokens=tokens, **kw)


# ------------------------------------------------------------------------------------------
# The oracle over many rows / tokens in worker processes (spawned, so safe after CUDA has been
# initialised in the test process; each worker uses one BLAS thread)
# ------------------------------------------------------------------------------------------
_P_STATE = {}


def _pool_init(inp, w):
    _P_STATE["inp"], _P_STATE["w"] = inp, w
    try:
        from threadpoolctl import threadpool_limits
        _P_STATE["limits"] = threadpool_limits(1)
    except Exception:  # pragma: no cover
        pass


def _pool_call(task):
    kind, items, kw = task
    fn = oracle_decode if kind == "decode" else oracle_prefill
    key = "rows" if kind == "decode" else "tokens"
    return fn(_P_STATE["inp"], _P_STATE["w"], **{key: items}, **kw)


def _merge(parts, axis):
    out = {}
    for k in parts[0]:
        v = parts[0][k]
        if isinstance(v, np.ndarray):
            out[k] = np.concatenate([p[k] for p in parts], axis=axis)
        elif isinstance(v, list):
            out[k] = [x for p in parts for x in p[k]]
        elif v is None:
            out[k] = None
        else:
            raise TypeError(k)
    return out


def oracle_parallel(kind: str, inp: dict, w, items=None, workers=None, **kw):
    """``oracle_decode`` (kind "decode", items = rows) or ``oracle_prefill`` (kind "prefill",
    items = tokens) split over worker processes; the result is the same dict the single call
    returns for all items."""
    import multiprocessing as mp
    import os
    from concurrent.futures import ProcessPoolExecutor
    n = w.batch if kind == "decode" else w.tokens
    items = list(range(n)) if items is None else list(items)
    workers = workers or max(1, min(16, os.cpu_count() or 1, len(items)))
    chunk = max(1, (len(items) + 4 * workers - 1) // (4 * workers))
    tasks = [(kind, items[i:i + chunk], kw) for i in range(0, len(items), chunk)]
    if workers == 1 or len(tasks) == 1:
        parts = [_pool_call_local(inp, w, t) for t in tasks]
    else:
        with ProcessPoolExecutor(workers, mp_context=mp.get_context("spawn"),
                                 initializer=_pool_init, initargs=(inp, w)) as ex:
            parts = list(ex.map(_pool_call, tasks))
    if kind == "decode":
        return _merge(parts, 0)
    merged = {"out": np.concatenate([p["out"] for p in parts], axis=1),
              "lse": np.concatenate([p["lse"] for p in parts], axis=1)}
    return merged


def _pool_call_local(inp, w, task):
    kind, items, kw = task
    if kind == "decode":
        return oracle_decode(inp, w, rows=items, **kw)
    return oracle_prefill(inp, w, tokens=items, **kw)


class _CacheView:
    """Widens rows of the bf16 cache to float64 lazily (indexing [b, :n, cols])."""

    def __init__(self, bits: np.ndarray):
        self.bits = bits

    def __getitem__(self, idx):
        return bf16_bits_to_f64(self.bits[idx])


__all__ = ["assert_close_bf16", "to_device", "bf16_to_np", "f64", "oracle_decode",
           "oracle_prefill", "make_inputs", "workload", "REL_TOL", "ABS_TOL", "PROB_TOL",
           "LSE_ATOL", "LSE_RTOL", "oracle_parallel"]
