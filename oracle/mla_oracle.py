"""fp64 CPU oracle for absorbed multi-head latent attention (MLA).

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke entry and the CPU-baseline leg of the
benchmark may import this module.  The library's GPU path never calls it and shares no code
with it; this file imports nothing but numpy.

Every function follows one passage of the source pages and is written as the plain definition,
in float64.  By default nothing is rounded in between (the pages round to bf16 after each
Linear/einsum; the GPU path rounds at similar points and the parity tolerance absorbs it); see the
precision modes below.  Library primitives used as steps: numpy ``matmul``/``einsum``
(contractions), ``exp``/``log``/``sqrt``/``sin``/``cos``/``frexp``/``rint``.

Source pages (cited by title and section):
  [QRMS]  DeepSeek V4.1 · Query RMSNorm — formula block and the ``RMSNorm`` excerpt.
  [QH]    DeepSeek-V3.2-Exp · Query heads — the six-step formula block, the parameter table, the
          "Explanation" (one wq_b, split per head after the product), the ``mla-init`` and
          ``mla-queries`` excerpts.
  [AU]    DeepSeek-V3.2-Exp · Attention update — ``block``, ``rmsnorm`` (residual form) and the
          ``mla-decode`` (absorbed "MQA decode") excerpts.
  [VS]    Kimi-K2 · value_states — parameter table, ``mla-init`` and ``mla-prefill`` excerpts
          (the non-absorbed form: rebuilt per-head keys/values, additive causal mask).

Readings where the pages are silent or garbled (each also listed in the design notes):
  * RoPE is the interleaved kind (adjacent pairs (2i, 2i+1)); base theta = 10000;
    theta_i = theta^(-2i/rope_dim); positive rotation (x0 cos - x1 sin, x0 sin + x1 cos).
  * The pe cache holds keys that are already rotated (the cache producer is off the path).
  * The index mask of the V3.2 decode excerpt is taken with top-k >= end_pos, i.e. dense.
  * Decode query sits at position start_pos and sees keys 0..start_pos; a prefill query t sees
    keys 0..start_pos+t.
  * softmax_scale = qk_head_dim^-0.5 (the YaRN mscale branch of [QH] mla-init is off).

Precision modes of ``decode`` / ``prefill``:
  * ``query_precision="exact"`` (default): every step in float64, no rounding.
  * ``query_precision="bf16"``: the query side is rounded to bfloat16 where the pages' tensors are
    bfloat16 — the RMSNorm output (``.to(dtype)``, [AU] rmsnorm), the wq_b output (a bf16
    Linear, [QH] mla-queries), the rotated q_pe (``apply_rotary_emb`` returns the input dtype,
    [QH] mla-queries) and the absorbed q_nope (einsum of bf16 tensors, [AU] mla-decode).  Scores,
    softmax and everything after stay float64 (the fp32 softmax of the method).  This is the
    reference for the softmax probabilities, whose 1e-3 bound is tighter than the effect of those
    four roundings.  Pinned by a pure-Python scalar enumeration with its own bit-level bf16
    rounding, compared bit for bit on inputs whose sums are exact, and by mutations that drop
    each rounding in turn.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "round_bf16", "rmsnorm", "rope_frequencies", "apply_rope_interleaved", "query_heads", "absorb_w_uk",
    "latent_scores", "softmax_fp", "latent_weighted_sum", "expand_w_uv", "decode", "prefill",
    "nonabsorbed_attention", "split_wkv_b", "split_wq_b", "produce_latents", "write_cache_rows",
    "index_mask", "output_projection", "nonabsorbed_prefill", "fp8_e4m3_value",
    "dequant_block_fp8",
]


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 value (8 significant bits, ties to even),
    returned as float64.  Done directly from float64 (no detour through float32)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)


# ------------------------------------------------------------------------------------------
# a1: RMSNorm with optional residual  ([AU] rmsnorm; [QRMS] formula and excerpt)
# ------------------------------------------------------------------------------------------
def rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float = 1e-6,
            residual: np.ndarray | None = None):
    """y = gamma * u / sqrt(mean_j(u_j^2) + eps) over the last axis, u = x (+ residual).

    With a residual, the pages first add it (``x = residual = x + residual``) and return the
    sum as the new residual.  Returns ``(y, u_or_None)``.
    """
    u = np.asarray(x, dtype=np.float64)
    if residual is not None:
        u = u + np.asarray(residual, dtype=np.float64)
    m2 = np.mean(u * u, axis=-1, keepdims=True)
    y = np.asarray(gamma, dtype=np.float64) * (u / np.sqrt(m2 + eps))
    return y, (u if residual is not None else None)


# ------------------------------------------------------------------------------------------
# a3: interleaved rotary embedding  ([QH] step "Q^R_t = RoPE(Q^pe_t, R_t)", R [T, 32 pairs])
# ------------------------------------------------------------------------------------------
def rope_frequencies(rope_dim: int, theta: float = 10000.0) -> np.ndarray:
    """theta_i = theta^(-2i/rope_dim), i < rope_dim/2 (one angle rate per pair)."""
    i = np.arange(rope_dim // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * i / rope_dim)


def apply_rope_interleaved(x: np.ndarray, pos: np.ndarray, theta: float = 10000.0) -> np.ndarray:
    """Rotate each adjacent pair (x[2i], x[2i+1]) of the last axis by angle pos * theta_i.

    ``x`` is [..., rope_dim]; ``pos`` broadcasts against ``x.shape[:-1]``.
    """
    x = np.asarray(x, dtype=np.float64)
    rope_dim = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_frequencies(rope_dim, theta)
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty(np.broadcast_shapes(x.shape, ang.shape[:-1] + (rope_dim,)), dtype=np.float64)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


# ------------------------------------------------------------------------------------------
# a2-a3: query heads  ([QH] formula block, Explanation, mla-queries excerpt)
# ------------------------------------------------------------------------------------------
def split_wq_b(wq_b: np.ndarray, n_heads: int, nope: int, rope: int):
    """View wq_b [H*(nope+rope), q_lora] per head and return (W_UQ rows, W_QR rows):
    [H, nope, q_lora] and [H, rope, q_lora].  Each head's block is nope content rows followed by
    rope rows ([QH] Explanation: one matrix, split per head after the product)."""
    w = np.asarray(wq_b, dtype=np.float64).reshape(n_heads, nope + rope, -1)
    return w[:, :nope, :], w[:, nope:, :]


def query_heads(y: np.ndarray, wq_b: np.ndarray, n_heads: int, nope: int, rope: int,
                pos: np.ndarray, theta: float = 10000.0):
    """q = y @ wq_b^T viewed [M, H, nope+rope]; q_nope = first nope features of each head,
    q_pe = RoPE(last rope features).  ``y`` is [M, q_lora]; ``pos`` is [M]."""
    q = np.asarray(y, dtype=np.float64) @ np.asarray(wq_b, dtype=np.float64).T
    q = q.reshape(q.shape[0], n_heads, nope + rope)
    q_nope = q[..., :nope]
    q_pe = apply_rope_interleaved(q[..., nope:], np.asarray(pos)[:, None], theta)
    return q_nope, q_pe


# ------------------------------------------------------------------------------------------
# a4-a8: absorbed attention  ([AU] mla-decode excerpt)
# ------------------------------------------------------------------------------------------
def split_wkv_b(wkv_b: np.ndarray, n_heads: int, nope: int, v: int):
    """wkv_b [H*(nope+v), kv_lora] viewed [H, nope+v, kv_lora]: W_UK = the first nope rows of each
    head, W_UV = the last v rows ([AU] mla-decode: ``wkv_b[:, :nope]`` and ``wkv_b[:, -v:]``)."""
    w = np.asarray(wkv_b, dtype=np.float64).reshape(n_heads, nope + v, -1)
    return w[:, :nope, :], w[:, nope:, :]


def absorb_w_uk(q_nope: np.ndarray, w_uk: np.ndarray) -> np.ndarray:
    """q_lat[m, h, c] = sum_d q_nope[m, h, d] * W_UK[h, d, c]  ("bshd,hdc->bshc")."""
    return np.einsum("mhd,hdc->mhc", np.asarray(q_nope, np.float64), w_uk)


def latent_scores(q_lat: np.ndarray, q_pe: np.ndarray, kv: np.ndarray, pe: np.ndarray,
                  scale: float) -> np.ndarray:
    """s[h, t] = (q_lat[h]·kv[t] + q_pe[h]·pe[t]) * scale for one query row.

    ``q_lat`` [H, kv_lora], ``q_pe`` [H, rope], ``kv`` [keys, kv_lora], ``pe`` [keys, rope]."""
    return (q_lat @ kv.T + q_pe @ pe.T) * scale


def softmax_fp(s: np.ndarray):
    """Softmax along the last axis with max subtraction; also returns lse = log sum exp(s)."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    z = np.sum(e, axis=-1, keepdims=True)
    return e / z, (m + np.log(z))[..., 0]


def latent_weighted_sum(p: np.ndarray, kv: np.ndarray) -> np.ndarray:
    """o_lat[h, c] = sum_t p[h, t] * kv[t, c]  ("bsht,btc->bshc")."""
    return p @ kv


def expand_w_uv(o_lat: np.ndarray, w_uv: np.ndarray) -> np.ndarray:
    """out[..., h, d] = sum_c o_lat[..., h, c] * W_UV[h, d, c]  ("bshc,hdc->bshd")."""
    return np.einsum("...hc,hdc->...hd", o_lat, w_uv)


def index_mask(topk, end_pos: int) -> np.ndarray:
    """[AU] mla-decode: ``full((end_pos,), -inf).scatter_(-1, topk_indices, 0)`` — 0 at every
    selected key, -inf elsewhere.  Entries < 0 are unused slots of a padded index list (this
    build's convention for rows with fewer than K selected keys)."""
    m = np.full(end_pos, -np.inf)
    idx = np.asarray(topk, dtype=np.int64)
    m[idx[idx >= 0]] = 0.0
    return m


def _attend_row(q_lat_h, q_pe_h, kv, pe, scale, w_uv, want_logits=False, mask=None):
    s = latent_scores(q_lat_h, q_pe_h, kv, pe, scale)
    if mask is not None:
        s = s + mask[None, :]
    p, lse = softmax_fp(s)
    o_lat = latent_weighted_sum(p, kv)
    out = expand_w_uv(o_lat, w_uv)
    return out, lse, (s if want_logits else None), o_lat


def _front(q_latent_rows, residual_rows, gamma, wq_b, wkv_b, dims, pos, theta, eps,
           query_precision="exact"):
    H, nope, rope, v = dims["n_heads"], dims["nope"], dims["rope"], dims["v"]
    w_uk, w_uv = split_wkv_b(wkv_b, H, nope, v)
    y, res = rmsnorm(q_latent_rows, gamma, eps, residual_rows)
    if query_precision == "exact":
        q_nope, q_pe = query_heads(y, wq_b, H, nope, rope, pos, theta)
        q_lat = absorb_w_uk(q_nope, w_uk)
    elif query_precision == "bf16":
        y = round_bf16(y)
        q = round_bf16(y @ np.asarray(wq_b, dtype=np.float64).T).reshape(y.shape[0], H, nope + rope)
        q_nope = q[..., :nope]
        q_pe = round_bf16(apply_rope_interleaved(q[..., nope:], np.asarray(pos)[:, None], theta))
        q_lat = round_bf16(absorb_w_uk(q_nope, w_uk))
    else:
        raise ValueError(query_precision)
    return y, res, q_nope, q_pe, q_lat, w_uv


def _dims(n_heads, nope=128, rope=64, v=128):
    return {"n_heads": n_heads, "nope": nope, "rope": rope, "v": v}


def decode(q_latent, gamma, wq_b, wkv_b, cache, start_pos, n_heads, *, residual=None,
           kv_lora=512, nope=128, rope=64, v=128, theta=10000.0, eps=1e-6, scale=None,
           rows=None, want_logits=False, want_intermediates=False, query_precision="exact",
           topk=None):
    """Absorbed decode ([AU] mla-decode).  With ``topk`` [B, K] (selected key indices of each
    sequence) the index mask of the excerpt is added to the scores; without it every key is kept
    (the mask of a top-k that covers all end_pos keys is all zeros).

    ``q_latent`` [B, q_lora]; ``cache`` [B, max_t, kv_lora+rope] (packed latents ‖ pe key);
    ``start_pos`` [B]: sequence b's query is at position start_pos[b] and sees keys 0..start_pos[b].
    ``rows`` optionally restricts the computation to some sequences.  Returns a dict with
    ``out`` [R, H, v], ``lse`` [R, H] and, on request, ``logits`` (list of [H, keys]) and the
    intermediates y, residual_out, q_nope, q_pe, q_lat, o_lat."""
    rows = np.arange(len(start_pos)) if rows is None else np.asarray(rows)
    if scale is None:
        scale = float(nope + rope) ** -0.5
    dims = _dims(n_heads, nope, rope, v)
    q_latent = np.asarray(q_latent, np.float64)[rows]
    res_in = None if residual is None else np.asarray(residual, np.float64)[rows]
    pos = np.asarray(start_pos)[rows].astype(np.int64)
    y, res, q_nope, q_pe, q_lat, w_uv = _front(q_latent, res_in, gamma, wq_b, wkv_b, dims,
                                                pos, theta, eps, query_precision)
    outs, lses, logits, olats = [], [], [], []
    for i, b in enumerate(rows):
        n = int(pos[i]) + 1
        kv = np.asarray(cache[b, :n, :kv_lora], np.float64)
        pe = np.asarray(cache[b, :n, kv_lora:kv_lora + rope], np.float64)
        mask = None if topk is None else index_mask(np.asarray(topk)[b], n)
        o, lse, s, o_lat = _attend_row(q_lat[i], q_pe[i], kv, pe, scale, w_uv, want_logits, mask)
        outs.append(o)
        lses.append(lse)
        logits.append(s)
        olats.append(o_lat)
    r = {"out": np.stack(outs), "lse": np.stack(lses)}
    if want_logits:
        r["logits"] = logits
    if want_intermediates:
        r.update(y=y, residual_out=res, q_nope=q_nope, q_pe=q_pe, q_lat=q_lat,
                 o_lat=np.stack(olats))
    return r


def prefill(q_latent, gamma, wq_b, wkv_b, cache, start_pos, n_heads, *, residual=None,
            kv_lora=512, nope=128, rope=64, v=128, theta=10000.0, eps=1e-6, scale=None,
            batch_rows=None, tokens=None, want_intermediates=False, query_precision="exact"):
    """Absorbed attention for a chunk of T new tokens after ``start_pos`` (int) cached positions.

    Query t of sequence b is at position start_pos + t and sees keys 0..start_pos+t (causal;
    the additive mask of [VS] mla-prefill, -inf above the diagonal).  ``q_latent`` [B, T, q_lora];
    cache rows start_pos..start_pos+T-1 already hold the chunk's own latents.  ``tokens``
    optionally restricts the computation to some token indices.  Returns ``out`` [B', T', H, v]
    and ``lse`` [B', T', H]."""
    q_latent = np.asarray(q_latent, np.float64)
    B, T, _ = q_latent.shape
    batch_rows = np.arange(B) if batch_rows is None else np.asarray(batch_rows)
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    if scale is None:
        scale = float(nope + rope) ** -0.5
    dims = _dims(n_heads, nope, rope, v)
    out = np.empty((len(batch_rows), len(tokens), n_heads, v))
    lse = np.empty((len(batch_rows), len(tokens), n_heads))
    inter = []
    for bi, b in enumerate(batch_rows):
        xs = q_latent[b, tokens]
        rs = None if residual is None else np.asarray(residual, np.float64)[b, tokens]
        pos = int(start_pos) + tokens.astype(np.int64)
        y, res, q_nope, q_pe, q_lat, w_uv = _front(xs, rs, gamma, wq_b, wkv_b, dims, pos,
                                                    theta, eps, query_precision)
        for ti in range(len(tokens)):
            n = int(pos[ti]) + 1
            kv = np.asarray(cache[b, :n, :kv_lora], np.float64)
            pe = np.asarray(cache[b, :n, kv_lora:kv_lora + rope], np.float64)
            o, l, _, _ = _attend_row(q_lat[ti], q_pe[ti], kv, pe, scale, w_uv)
            out[bi, ti] = o
            lse[bi, ti] = l
        inter.append(dict(y=y, residual_out=res, q_nope=q_nope, q_pe=q_pe, q_lat=q_lat))
    r = {"out": out, "lse": lse}
    if want_intermediates:
        r["intermediates"] = inter
    return r


# ------------------------------------------------------------------------------------------
# Non-absorbed form  ([VS] mla-prefill: rebuilt per-head keys and values, additive mask)
# ------------------------------------------------------------------------------------------
def nonabsorbed_attention(q_nope, q_pe, kv, pe, wkv_b, n_heads, *, q_positions, nope=128,
                          v=128, scale=None):
    """Multi-head attention with keys and values rebuilt from the latent cache.

    ``q_nope`` [Tq, H, nope], ``q_pe`` [Tq, H, rope] (rotated); ``kv`` [keys, kv_lora];
    ``pe`` [keys, rope] is the shared rotary key of every head.  Per head h:
    k_nope[t] = W_UK[h] kv[t], key[t] = [k_nope[t] ‖ pe[t]], value[t] = W_UV[h] kv[t];
    weights = softmax(query·key^T·scale + mask) with mask[i, t] = 0 if t <= q_positions[i] else
    -inf; output = weights · value.  Returns ([Tq, H, v], lse [Tq, H])."""
    rope = q_pe.shape[-1]
    if scale is None:
        scale = float(nope + rope) ** -0.5
    w_uk, w_uv = split_wkv_b(wkv_b, n_heads, nope, v)
    kv = np.asarray(kv, np.float64)
    pe = np.asarray(pe, np.float64)
    keys_n = kv.shape[0]
    mask = np.where(np.arange(keys_n)[None, :] <= np.asarray(q_positions)[:, None], 0.0, -np.inf)
    out = np.empty((q_nope.shape[0], n_heads, v))
    lse = np.empty((q_nope.shape[0], n_heads))
    for h in range(n_heads):
        k_nope = kv @ w_uk[h].T                                   # [keys, nope]
        key = np.concatenate([k_nope, pe], axis=1)                # [keys, nope+rope]
        value = kv @ w_uv[h].T                                    # [keys, v]
        query = np.concatenate([q_nope[:, h], q_pe[:, h]], axis=1)  # [Tq, nope+rope]
        logits = query @ key.T * scale + mask
        p, l = softmax_fp(logits)
        out[:, h] = p @ value
        lse[:, h] = l
    return out, lse


# ------------------------------------------------------------------------------------------
# Cache producer  ([QH] mla-init: wq_a, wkv_a, kv_norm; [QH] mla-queries: qr = q_norm(wq_a(x));
# [VS] mla-init: the joint key-value down-projection kv_a_proj_with_mqa that also emits the shared
# rotary key, and its latent RMSNorm kv_a_layernorm)
# ------------------------------------------------------------------------------------------
def produce_latents(x, wq_a, wkv_a, kv_norm_gain, pos, *, kv_lora=512, rope=64, theta=10000.0,
                    eps=1e-6, precision="exact"):
    """The step upstream of the attention for new tokens ``x`` [M, dim] at positions ``pos`` [M].

    q_latent = x wq_a^T                      (the query latent, input of q_norm)
    c        = x wkv_a^T  [M, kv_lora + rope] (one Linear: the latent, then the shared rotary key)
    kv       = RMSNorm(c[:, :kv_lora]) with gain kv_norm_gain (eps 1e-6)
    k_pe     = RoPE(c[:, kv_lora:], pos)      (interleaved pairs, like q_pe)
    Returns (q_latent, kv, k_pe).  ``precision="bf16"`` rounds where the pages' tensors are bf16:
    both Linear outputs, the normalised latent (``.to(dtype)``) and the rotated key."""
    x = np.asarray(x, np.float64)
    r = round_bf16 if precision == "bf16" else (lambda a: a)
    if precision not in ("exact", "bf16"):
        raise ValueError(precision)
    q_latent = r(x @ np.asarray(wq_a, np.float64).T)
    c = r(x @ np.asarray(wkv_a, np.float64).T)
    kv, _ = rmsnorm(c[:, :kv_lora], kv_norm_gain, eps)
    k_pe = apply_rope_interleaved(c[:, kv_lora:kv_lora + rope], np.asarray(pos), theta)
    return q_latent, r(kv), r(k_pe)


def write_cache_rows(cache, kv, k_pe, batch_index, pos, kv_lora=512):
    """Store the new rows: cache[b, pos] = [kv ‖ k_pe] for each new token (the pages write
    ``kv_cache[:bsz, start_pos:end_pos]`` / ``pe_cache`` before attending over ``:end_pos``).
    Returns a float64 copy of ``cache`` [B, max_t, kv_lora + rope] with the rows replaced."""
    out = np.array(cache, dtype=np.float64, copy=True)
    for i, (b, t) in enumerate(zip(np.asarray(batch_index), np.asarray(pos))):
        out[b, t, :kv_lora] = kv[i]
        out[b, t, kv_lora:] = k_pe[i]
    return out


# ------------------------------------------------------------------------------------------
# Output projection and the non-absorbed prefill  ([AU] mla-output: x = wo(x.flatten(2));
# [VS] mla-prefill: per-head keys and values rebuilt from the latent, additive causal mask)
# ------------------------------------------------------------------------------------------
def output_projection(o, wo):
    """wo applied to the flattened head outputs: ``o`` [..., H, v] → [..., dim] with
    y[..., i] = sum_{h, d} wo[i, h*v + d] * o[..., h, d] (wo in nn.Linear layout [dim, H*v])."""
    o = np.asarray(o, np.float64)
    flat = o.reshape(o.shape[:-2] + (o.shape[-2] * o.shape[-1],))
    return flat @ np.asarray(wo, np.float64).T


def nonabsorbed_prefill(q_latent, gamma, wq_b, wkv_b, cache, start_pos, n_heads, wo=None, *,
                        residual=None, kv_lora=512, nope=128, rope=64, v=128, theta=10000.0,
                        eps=1e-6, scale=None, tokens=None):
    """A prefill chunk in the pages' other form: the query as in the absorbed path (q_norm, wq_b,
    RoPE), then for every head the keys [W_UK kv ‖ pe] and values W_UV kv rebuilt from the latent
    cache, causal softmax attention with the additive mask, and (with ``wo``) the output
    projection.  ``q_latent`` [B, T, q_lora]; returns ``out`` [B, T', H, v], ``lse`` [B, T', H]
    and ``y`` [B, T', dim] when ``wo`` is given."""
    q_latent = np.asarray(q_latent, np.float64)
    B, T, _ = q_latent.shape
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    dims = _dims(n_heads, nope, rope, v)
    out = np.empty((B, len(tokens), n_heads, v))
    lse = np.empty((B, len(tokens), n_heads))
    for b in range(B):
        rs = None if residual is None else np.asarray(residual, np.float64)[b, tokens]
        pos = int(start_pos) + tokens.astype(np.int64)
        _, _, q_nope, q_pe, _, _ = _front(q_latent[b, tokens], rs, gamma, wq_b, wkv_b, dims, pos,
                                          theta, eps)
        n = int(pos.max()) + 1
        kv = np.asarray(cache[b, :n, :kv_lora], np.float64)
        pe = np.asarray(cache[b, :n, kv_lora:kv_lora + rope], np.float64)
        o, l = nonabsorbed_attention(q_nope, q_pe, kv, pe, wkv_b, n_heads, q_positions=pos,
                                     nope=nope, v=v, scale=scale)
        out[b], lse[b] = o, l
    r = {"out": out, "lse": lse}
    if wo is not None:
        r["y"] = output_projection(out, wo)
    return r


# ------------------------------------------------------------------------------------------
# FP8 block-scaled weights  ([AU] mla-decode: ``weight_dequant(self.wkv_b.weight,
# self.wkv_b.scale)``; [QH] parameter table note: the checkpoint stores FP8 weights with block
# scales)
# ------------------------------------------------------------------------------------------
def fp8_e4m3_value(bits) -> np.ndarray:
    """Value of FP8 E4M3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent
    field 0 is subnormal: m/8 * 2^-6; no infinities; S.1111.111 is NaN) as float64."""
    b = np.asarray(bits, dtype=np.int64) & 0xFF
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    normal = (1.0 + m / 8.0) * np.power(2.0, e - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    v = sign * np.where(e == 0, sub, normal)
    return np.where((b & 0x7F) == 0x7F, np.nan, v)


def dequant_block_fp8(bits, scale, block: int = 128) -> np.ndarray:
    """weight_dequant: w[i, j] = value(bits[i, j]) * scale[i // block, j // block], returned in
    the default dtype (bf16) as the pages' decode uses it — rounded to bf16 here, as float64."""
    v = fp8_e4m3_value(bits)
    s = np.asarray(scale, np.float64)
    rows = np.arange(v.shape[0]) // block
    cols = np.arange(v.shape[1]) // block
    return round_bf16(v * s[rows][:, cols])
