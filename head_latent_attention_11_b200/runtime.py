"""PyTorch-side convenience around the C ABI: device memory and streams come from torch.

``MLARuntime`` allocates the workspace as a torch tensor, creates the context and forwards
decode / prefill calls with tensor arguments to the C entry points.  No computation happens here.
"""
from __future__ import annotations

import torch

from . import (MLAConfig, mla_decode, mla_destroy, mla_init, mla_prefill_chunk,
               mla_sync_status, mla_workspace_size)

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
                 softmax_scale: float = 0.0, rms_eps: float = 1e-6, stream=None):
        for t, dt in ((gamma, torch.float32), (wq_b, torch.bfloat16), (wkv_b, torch.bfloat16)):
            if not (t.is_cuda and t.dtype == dt and t.is_contiguous()):
                raise ValueError("weights must be contiguous CUDA tensors (gamma fp32, wq_b/wkv_b bf16)")
        self.cfg = MLAConfig.make(n_heads, max_rows, max_seq_len, rope_theta=rope_theta,
                                  softmax_scale=softmax_scale, rms_eps=rms_eps)
        self.n_heads = n_heads
        self.max_seq_len = max_seq_len
        self.workspace_bytes = mla_workspace_size(self.cfg)
        if self.workspace_bytes == 0:
            raise ValueError("unsupported MLA configuration")
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=gamma.device)
        self._weights = (gamma, wq_b, wkv_b)
        self.ctx = mla_init(self.cfg, gamma, wq_b, wkv_b, self.workspace, self.workspace_bytes,
                            _stream_handle(stream))

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
