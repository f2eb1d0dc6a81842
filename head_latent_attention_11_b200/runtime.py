"""PyTorch-side convenience around the C ABI: device memory and streams come from torch.

``MLARuntime`` allocates the workspace as a torch tensor, creates the context and forwards
decode / prefill calls with tensor arguments to the C entry points.  No computation happens here.
"""
from __future__ import annotations

import torch

from . import (MLAConfig, mla_attach_producer, mla_decode, mla_decode_sparse, mla_destroy,
               mla_init, mla_init_fp8, mla_mha_scratch_size, mla_prefill_chunk,
               mla_prefill_chunk_mha, mla_produce, mla_sync_status, mla_workspace_size)

C_LAT, D_ROPE, D_V = 512, 64, 128


def _stream_handle(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


class MLARuntime:
    """One MLA layer's weights bound to a workspace on the current CUDA device.

    ``gamma`` [1536] fp32, ``wq_b`` [H*192, 1536] bf16, ``wkv_b`` [H*256, 512] bf16 (CUDA tensors,
    kept alive by this object)."""

    def __init__(self, gamma: torch.Tensor, wq_b: torch.Tensor, wkv_b: torch.Tensor, *,
                 n_heads: int, max_rows: int, max_seq_len: int, rope_theta: float = 10000.0,
                 softmax_scale: float = 0.0, rms_eps: float = 1e-6, stream=None,
                 wq_b_scale: torch.Tensor | None = None, wkv_b_scale: torch.Tensor | None = None):
        """bf16 weights, or FP8 E4M3 codes (uint8 tensors) with their 128 x 128 block scales
        (fp32) passed as wq_b_scale / wkv_b_scale."""
        fp8 = wq_b_scale is not None
        wdt = torch.uint8 if fp8 else torch.bfloat16
        for t, dt in ((gamma, torch.float32), (wq_b, wdt), (wkv_b, wdt)):
            if not (t.is_cuda and t.dtype == dt and t.is_contiguous()):
                raise ValueError("weights must be contiguous CUDA tensors (gamma fp32, wq_b/wkv_b "
                                 "bf16, or uint8 FP8 codes with scales)")
        self.cfg = MLAConfig.make(n_heads, max_rows, max_seq_len, rope_theta=rope_theta,
                                  softmax_scale=softmax_scale, rms_eps=rms_eps)
        self.n_heads = n_heads
        self.max_seq_len = max_seq_len
        self.workspace_bytes = mla_workspace_size(self.cfg)
        if self.workspace_bytes == 0:
            raise ValueError("unsupported MLA configuration")
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=gamma.device)
        self._weights = (gamma, wq_b, wkv_b, wq_b_scale, wkv_b_scale)
        if fp8:
            self.ctx = mla_init_fp8(self.cfg, gamma, wq_b, wq_b_scale, wkv_b, wkv_b_scale,
                                    self.workspace, self.workspace_bytes, _stream_handle(stream))
        else:
            self.ctx = mla_init(self.cfg, gamma, wq_b, wkv_b, self.workspace,
                                self.workspace_bytes, _stream_handle(stream))

    # cache helpers -------------------------------------------------------------------------
    @staticmethod
    def cache_views(cache: torch.Tensor):
        """Packed cache [B, max_t, 576] → (kv pointer, strides, pe pointer, strides)."""
        if cache.dim() != 3 or cache.shape[-1] != C_LAT + D_ROPE or cache.stride(-1) != 1:
            raise ValueError("packed cache must be [B, max_t, 576] with unit last stride")
        sb, st = cache.stride(0), cache.stride(1)
        kv = cache.data_ptr()
        pe = kv + C_LAT * cache.element_size()
        return kv, sb, st, pe, sb, st

    def decode(self, q_latent: torch.Tensor, start_pos: torch.Tensor, cache: torch.Tensor, *,
               residual: torch.Tensor | None = None, out: torch.Tensor | None = None,
               lse: torch.Tensor | None = None, logits: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
        B = q_latent.shape[0]
        if out is None:
            out = torch.empty(B, self.n_heads, D_V, dtype=torch.bfloat16, device=q_latent.device)
        kv, ksb, kst, pe, psb, pst = self.cache_views(cache)
        mla_decode(self.ctx, q_latent, residual, start_pos, kv, ksb, kst, pe, psb, pst, B, out,
                   lse, logits, _stream_handle(stream))
        return out

    def decode_sparse(self, q_latent: torch.Tensor, start_pos: torch.Tensor, topk_idx: torch.Tensor,
                      topk_len: torch.Tensor, cache: torch.Tensor, *,
                      residual: torch.Tensor | None = None, out: torch.Tensor | None = None,
                      lse: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """Decode attending only each sequence's selected keys (topk_idx [B, k] int32, counts
        topk_len [B] int32, both on the device)."""
        B = q_latent.shape[0]
        if out is None:
            out = torch.empty(B, self.n_heads, D_V, dtype=torch.bfloat16, device=q_latent.device)
        kv, ksb, kst, pe, psb, pst = self.cache_views(cache)
        mla_decode_sparse(self.ctx, q_latent, residual, start_pos, topk_idx, topk_len,
                          topk_idx.shape[1], kv, ksb, kst, pe, psb, pst, B, out, lse,
                          _stream_handle(stream))
        return out

    def prefill(self, q_latent: torch.Tensor, start_pos: int, cache: torch.Tensor, *,
                residual: torch.Tensor | None = None, out: torch.Tensor | None = None,
                lse: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        B, T = q_latent.shape[0], q_latent.shape[1]
        if out is None:
            out = torch.empty(B, T, self.n_heads, D_V, dtype=torch.bfloat16,
                              device=q_latent.device)
        kv, ksb, kst, pe, psb, pst = self.cache_views(cache)
        mla_prefill_chunk(self.ctx, q_latent, residual, int(start_pos), T, kv, ksb, kst, pe, psb,
                          pst, B, out, lse, _stream_handle(stream))
        return out

    def attach_producer(self, wq_a: torch.Tensor, wkv_a: torch.Tensor,
                        kv_norm_gain: torch.Tensor) -> None:
        """Borrow the cache producer's weights: wq_a [1536, dim], wkv_a [576, dim] bf16,
        kv_norm_gain [512] fp32 (CUDA tensors, kept alive by this object)."""
        dim = wq_a.shape[1]
        self._producer = (wq_a, wkv_a, kv_norm_gain)
        mla_attach_producer(self.ctx, dim, wq_a, wkv_a, kv_norm_gain)

    def produce(self, x: torch.Tensor, cache: torch.Tensor, *, start_pos=None,
                start_pos_host: int = 0, q_latent: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
        """x [B, T, dim] → q_latent [B, T, 1536]; writes the tokens' rows of the packed cache
        (positions start_pos[b] + t, or start_pos_host + t)."""
        B, T = x.shape[0], x.shape[1]
        if q_latent is None:
            q_latent = torch.empty(B, T, 1536, dtype=torch.bfloat16, device=x.device)
        kv, ksb, kst, pe, psb, pst = self.cache_views(cache)
        mla_produce(self.ctx, x, start_pos, int(start_pos_host), T, B, kv, ksb, kst, pe, psb, pst,
                    q_latent, _stream_handle(stream))
        return q_latent

    def prefill_mha(self, q_latent: torch.Tensor, start_pos: int, cache: torch.Tensor, *,
                    residual: torch.Tensor | None = None, out: torch.Tensor | None = None,
                    lse: torch.Tensor | None = None, wo: torch.Tensor | None = None,
                    scratch: torch.Tensor | None = None, stream=None):
        """The chunk in the non-absorbed form (keys / values rebuilt per head); returns out
        [B, T, H, 128] and, with wo [dim, H*128], also y = wo(out) [B, T, dim]."""
        B, T = q_latent.shape[0], q_latent.shape[1]
        if out is None:
            out = torch.empty(B, T, self.n_heads, D_V, dtype=torch.bfloat16,
                              device=q_latent.device)
        need = mla_mha_scratch_size(self.ctx, B, T, int(start_pos))
        if scratch is None or scratch.numel() * scratch.element_size() < need:
            scratch = torch.empty(need, dtype=torch.uint8, device=q_latent.device)
        y = None
        dim = 0
        if wo is not None:
            dim = wo.shape[0]
            y = torch.empty(B, T, dim, dtype=torch.bfloat16, device=q_latent.device)
        kv, ksb, kst, pe, psb, pst = self.cache_views(cache)
        mla_prefill_chunk_mha(self.ctx, q_latent, residual, int(start_pos), T, kv, ksb, kst, pe,
                              psb, pst, B, scratch, need, out, lse, wo, dim, y,
                              _stream_handle(stream))
        return (out, y) if wo is not None else out

    def sync_status(self, stream=None) -> int:
        return mla_sync_status(self.ctx, _stream_handle(stream))

    def close(self) -> None:
        if getattr(self, "ctx", None) is not None:
            mla_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
