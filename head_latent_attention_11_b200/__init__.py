"""Python binding of the B200 absorbed-MLA C ABI (``include/mla.h``).

Argument marshalling only: every function forwards to the entry point of the same name in
``libmla_b200.so`` through ctypes and raises :class:`MLAError` on a non-OK status.  Pointer
arguments accept plain integers (device addresses) or any object with ``data_ptr()`` (e.g. a
CUDA ``torch.Tensor``); ``None`` passes NULL.  Streams are raw ``cudaStream_t`` handles (an int, or
an object with a ``cuda_stream`` attribute).

The library must have been built (``python -m head_latent_attention_11_b200.build``); there is no
fallback: importing a function when the library is missing raises immediately.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "MLAError", "MLAConfig", "load", "lib_path", "mla_status_string", "mla_workspace_size",
    "mla_init", "mla_destroy", "mla_rmsnorm", "mla_decode", "mla_prefill_chunk", "mla_sync_status",
    "mla_enable_stage_timing", "mla_stage_times", "mla_debug_copy", "mla_last_launch_count",
    "EXPORTED_SYMBOLS", "STATUS", "mla_latent_attention_noalloc", "mla_attach_producer",
    "mla_produce", "mla_decode_sparse", "mla_init_fp8", "mla_mha_scratch_size",
    "mla_prefill_chunk_mha", "mla_set_wait_limit",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "libmla_b200.so"

STATUS = {
    0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_WORKSPACE",
    4: "MLA_ERR_CUDA", 5: "MLA_ERR_DEVICE_TIMEOUT", 6: "MLA_ERR_DEVICE_ARG",
}

EXPORTED_SYMBOLS = (
    "mla_status_string", "mla_workspace_size", "mla_init", "mla_destroy", "mla_rmsnorm",
    "mla_decode", "mla_prefill_chunk", "mla_sync_status", "mla_enable_stage_timing",
    "mla_stage_times", "mla_debug_copy", "mla_last_launch_count",
    "mla_latent_attention_noalloc", "mla_attach_producer", "mla_produce", "mla_decode_sparse",
    "mla_init_fp8", "mla_mha_scratch_size", "mla_prefill_chunk_mha", "mla_set_wait_limit",
)


class MLAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")


class MLAConfig(ctypes.Structure):
    """Mirror of ``mla_config``."""
    _fields_ = [
        ("n_heads", ctypes.c_int32), ("q_lora_rank", ctypes.c_int32),
        ("kv_lora_rank", ctypes.c_int32), ("qk_nope_head_dim", ctypes.c_int32),
        ("qk_rope_head_dim", ctypes.c_int32), ("v_head_dim", ctypes.c_int32),
        ("rope_theta", ctypes.c_float), ("softmax_scale", ctypes.c_float),
        ("rms_eps", ctypes.c_float), ("max_rows", ctypes.c_int32), ("max_seq_len", ctypes.c_int32),
    ]

    @classmethod
    def make(cls, n_heads: int, max_rows: int, max_seq_len: int, *, rope_theta: float = 10000.0,
             softmax_scale: float = 0.0, rms_eps: float = 1e-6, q_lora_rank: int = 1536,
             kv_lora_rank: int = 512, qk_nope_head_dim: int = 128, qk_rope_head_dim: int = 64,
             v_head_dim: int = 128) -> "MLAConfig":
        return cls(n_heads, q_lora_rank, kv_lora_rank, qk_nope_head_dim, qk_rope_head_dim,
                   v_head_dim, rope_theta, softmax_scale, rms_eps, max_rows, max_seq_len)


_lib = None


def lib_path() -> str:
    return os.path.join(_HERE, _LIB_NAME)


def load() -> ctypes.CDLL:
    """Load ``libmla_b200.so`` (once) and declare the signatures of its entry points."""
    global _lib
    if _lib is not None:
        return _lib
    path = lib_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{_LIB_NAME} is not built ({path}); run "
                           "`python -m head_latent_attention_11_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(path)
    P, I32, I64, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    sig = {
        "mla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "mla_workspace_size": (SZ, [ctypes.POINTER(MLAConfig)]),
        "mla_init": (ctypes.c_int, [ctypes.POINTER(MLAConfig), P, P, P, P, SZ, P,
                                    ctypes.POINTER(P)]),
        "mla_destroy": (None, [P]),
        "mla_rmsnorm": (ctypes.c_int, [P, P, P, I32, I32, F, P, P]),
        "mla_decode": (ctypes.c_int, [P, P, P, P, P, I64, I64, P, I64, I64, I32, P, P, P, P]),
        "mla_prefill_chunk": (ctypes.c_int, [P, P, P, I32, I32, P, I64, I64, P, I64, I64, I32, P,
                                             P, P]),
        "mla_sync_status": (ctypes.c_int, [P, P]),
        "mla_enable_stage_timing": (ctypes.c_int, [P, I32]),
        "mla_stage_times": (ctypes.c_int, [P, ctypes.POINTER(ctypes.c_float),
                                           ctypes.POINTER(ctypes.c_char_p), I32,
                                           ctypes.POINTER(I32)]),
        "mla_debug_copy": (ctypes.c_int, [P, I32, P, SZ, P]),
        "mla_last_launch_count": (I32, [P]),
        "mla_latent_attention_noalloc": (ctypes.c_int, [P, P, I32, I32, F, P, I64, I64, P, I64,
                                                        I64, I32, P, P, P, P]),
        "mla_attach_producer": (ctypes.c_int, [P, I32, P, P, P]),
        "mla_mha_scratch_size": (SZ, [P, I32, I32, I32]),
        "mla_set_wait_limit": (ctypes.c_int, [P, ctypes.c_uint64]),
        "mla_prefill_chunk_mha": (ctypes.c_int, [P, P, P, I32, I32, P, I64, I64, P, I64, I64, I32,
                                                 P, SZ, P, P, P, I32, P, P]),
        "mla_init_fp8": (ctypes.c_int, [ctypes.POINTER(MLAConfig), P, P, P, P, P, P, SZ, P,
                                        ctypes.POINTER(P)]),
        "mla_decode_sparse": (ctypes.c_int, [P, P, P, P, P, P, I32, P, I64, I64, P, I64, I64, I32,
                                             P, P, P]),
        "mla_produce": (ctypes.c_int, [P, P, P, I32, I32, I32, P, I64, I64, P, I64, I64, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, ctypes.c_void_p):
        return x.value
    raise TypeError(f"cannot pass {type(x).__name__} as a pointer")


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return getattr(s, "cuda_stream")


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise MLAError(fn, status)


def mla_status_string(status: int) -> str:
    return load().mla_status_string(status).decode()


def mla_workspace_size(cfg: MLAConfig) -> int:
    return int(load().mla_workspace_size(ctypes.byref(cfg)))


def mla_init(cfg: MLAConfig, q_norm_gain, wq_b, wkv_b, workspace, workspace_bytes: int,
             stream=None) -> ctypes.c_void_p:
    ctx = ctypes.c_void_p()
    _check("mla_init", load().mla_init(ctypes.byref(cfg), _ptr(q_norm_gain), _ptr(wq_b),
                                       _ptr(wkv_b), _ptr(workspace), workspace_bytes,
                                       _stream(stream), ctypes.byref(ctx)))
    return ctx


def mla_destroy(ctx) -> None:
    load().mla_destroy(ctx)


def mla_rmsnorm(x, residual, gain, rows: int, dim: int, eps: float, y, stream=None) -> None:
    _check("mla_rmsnorm", load().mla_rmsnorm(_ptr(x), _ptr(residual), _ptr(gain), rows, dim, eps,
                                             _ptr(y), _stream(stream)))


def mla_decode(ctx, q_latent, residual, start_pos, kv_cache, kv_stride_b: int, kv_stride_t: int,
               pe_cache, pe_stride_b: int, pe_stride_t: int, B: int, out, lse=None, logits=None,
               stream=None) -> None:
    _check("mla_decode", load().mla_decode(
        ctx, _ptr(q_latent), _ptr(residual), _ptr(start_pos), _ptr(kv_cache), kv_stride_b,
        kv_stride_t, _ptr(pe_cache), pe_stride_b, pe_stride_t, B, _ptr(out), _ptr(lse),
        _ptr(logits), _stream(stream)))


def mla_prefill_chunk(ctx, q_latent, residual, start_pos: int, T: int, kv_cache, kv_stride_b: int,
                      kv_stride_t: int, pe_cache, pe_stride_b: int, pe_stride_t: int, B: int, out,
                      lse=None, stream=None) -> None:
    _check("mla_prefill_chunk", load().mla_prefill_chunk(
        ctx, _ptr(q_latent), _ptr(residual), start_pos, T, _ptr(kv_cache), kv_stride_b,
        kv_stride_t, _ptr(pe_cache), pe_stride_b, pe_stride_t, B, _ptr(out), _ptr(lse),
        _stream(stream)))


def mla_sync_status(ctx, stream=None) -> int:
    """Returns the status code (does not raise: device-side errors are data)."""
    return int(load().mla_sync_status(ctx, _stream(stream)))


def mla_enable_stage_timing(ctx, enable: bool = True) -> None:
    _check("mla_enable_stage_timing", load().mla_enable_stage_timing(ctx, int(enable)))


def mla_stage_times(ctx, cap: int = 8) -> list[tuple[str, float]]:
    ms = (ctypes.c_float * cap)()
    names = (ctypes.c_char_p * cap)()
    n = ctypes.c_int32()
    _check("mla_stage_times", load().mla_stage_times(ctx, ms, names, cap, ctypes.byref(n)))
    return [(names[i].decode(), float(ms[i])) for i in range(min(n.value, cap))]


def mla_debug_copy(ctx, which: int, dst, nbytes: int, stream=None) -> None:
    _check("mla_debug_copy", load().mla_debug_copy(ctx, which, _ptr(dst), nbytes,
                                                   _stream(stream)))


def mla_last_launch_count(ctx) -> int:
    return int(load().mla_last_launch_count(ctx))


def mla_latent_attention_noalloc(q_abs, start_pos, rows: int, n_heads: int, softmax_scale: float,
                                 kv_cache, kv_stride_b: int, kv_stride_t: int, pe_cache,
                                 pe_stride_b: int, pe_stride_t: int, max_seq_len: int, o_lat,
                                 lse=None, status=None, stream=None) -> None:
    """Attention over the cache for given absorbed queries using no memory beyond the arguments
    and the library's fixed scratch array (see include/mla.h for limits and set-up)."""
    _check("mla_latent_attention_noalloc", load().mla_latent_attention_noalloc(
        _ptr(q_abs), _ptr(start_pos), rows, n_heads, softmax_scale, _ptr(kv_cache), kv_stride_b,
        kv_stride_t, _ptr(pe_cache), pe_stride_b, pe_stride_t, max_seq_len, _ptr(o_lat),
        _ptr(lse), _ptr(status), _stream(stream)))


def mla_attach_producer(ctx, dim: int, wq_a, wkv_a, kv_norm_gain) -> None:
    _check("mla_attach_producer", load().mla_attach_producer(ctx, dim, _ptr(wq_a), _ptr(wkv_a),
                                                             _ptr(kv_norm_gain)))


def mla_produce(ctx, x, start_pos, start_pos_host: int, T: int, B: int, kv_cache, kv_stride_b: int,
                kv_stride_t: int, pe_cache, pe_stride_b: int, pe_stride_t: int, q_latent,
                stream=None) -> None:
    _check("mla_produce", load().mla_produce(
        ctx, _ptr(x), _ptr(start_pos), start_pos_host, T, B, _ptr(kv_cache), kv_stride_b,
        kv_stride_t, _ptr(pe_cache), pe_stride_b, pe_stride_t, _ptr(q_latent), _stream(stream)))


def mla_decode_sparse(ctx, q_latent, residual, start_pos, topk_idx, topk_len, k: int, kv_cache,
                      kv_stride_b: int, kv_stride_t: int, pe_cache, pe_stride_b: int,
                      pe_stride_t: int, B: int, out, lse=None, stream=None) -> None:
    _check("mla_decode_sparse", load().mla_decode_sparse(
        ctx, _ptr(q_latent), _ptr(residual), _ptr(start_pos), _ptr(topk_idx), _ptr(topk_len), k,
        _ptr(kv_cache), kv_stride_b, kv_stride_t, _ptr(pe_cache), pe_stride_b, pe_stride_t, B,
        _ptr(out), _ptr(lse), _stream(stream)))


def mla_init_fp8(cfg: MLAConfig, q_norm_gain, wq_b_fp8, wq_b_scale, wkv_b_fp8, wkv_b_scale,
                 workspace, workspace_bytes: int, stream=None) -> ctypes.c_void_p:
    ctx = ctypes.c_void_p()
    _check("mla_init_fp8", load().mla_init_fp8(
        ctypes.byref(cfg), _ptr(q_norm_gain), _ptr(wq_b_fp8), _ptr(wq_b_scale), _ptr(wkv_b_fp8),
        _ptr(wkv_b_scale), _ptr(workspace), workspace_bytes, _stream(stream), ctypes.byref(ctx)))
    return ctx


def mla_mha_scratch_size(ctx, B: int, T: int, start_pos: int) -> int:
    return int(load().mla_mha_scratch_size(ctx, B, T, start_pos))


def mla_prefill_chunk_mha(ctx, q_latent, residual, start_pos: int, T: int, kv_cache,
                          kv_stride_b: int, kv_stride_t: int, pe_cache, pe_stride_b: int,
                          pe_stride_t: int, B: int, kv_scratch, scratch_bytes: int, out, lse=None,
                          wo=None, dim: int = 0, y=None, stream=None) -> None:
    _check("mla_prefill_chunk_mha", load().mla_prefill_chunk_mha(
        ctx, _ptr(q_latent), _ptr(residual), start_pos, T, _ptr(kv_cache), kv_stride_b,
        kv_stride_t, _ptr(pe_cache), pe_stride_b, pe_stride_t, B, _ptr(kv_scratch), scratch_bytes,
        _ptr(out), _ptr(lse), _ptr(wo), dim, _ptr(y), _stream(stream)))


def mla_set_wait_limit(ctx, ns: int) -> None:
    _check("mla_set_wait_limit", load().mla_set_wait_limit(ctx, int(ns)))
