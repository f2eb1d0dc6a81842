"""Pins of the oracle's cache producer (q_latent = wq_a x; c = wkv_a x split into the 512-wide
latent and the shared rotary key; kv_norm on the latent; RoPE on the key; rows written at their
positions before attending).  None of these needs a GPU.

Sources: "DeepSeek-V3.2-Exp · Query heads" (mla-init: wq_a, wkv_a = Linear(dim, kv_lora + rope),
kv_norm = RMSNorm(kv_lora); mla-queries: qr = q_norm(wq_a(x))), "Kimi-K2 · value_states" (mla-init:
kv_a_proj_with_mqa emits the latent and the rotary key, kv_a_layernorm normalises the latent),
"DeepSeek-V3.2-Exp · Attention update" (mla-decode attends over kv_cache[:, :end_pos])."""
import cmath
import math

import numpy as np
import pytest

import oracle
import oracle.mla_oracle as om
from test_oracle_pins import _bf16_bits


def _brute_produce_one(x, wq_a, wkv_a, gain, pos, C, Dr, theta, eps, rnd=None):
    """Scalar enumeration of one token: returns (q_latent, kv, k_pe) as lists."""
    keep = rnd if rnd is not None else (lambda v: v)
    dim = len(x)
    q_latent = [keep(sum(wq_a[i][k] * x[k] for k in range(dim))) for i in range(len(wq_a))]
    c = [keep(sum(wkv_a[i][k] * x[k] for k in range(dim))) for i in range(C + Dr)]
    lat, key = c[:C], c[C:]
    ms = sum(v * v for v in lat) / C
    kv = [keep(gain[j] * (lat[j] / math.sqrt(ms + eps))) for j in range(C)]
    k_pe = []
    for i in range(Dr // 2):
        z = complex(key[2 * i], key[2 * i + 1]) * cmath.exp(1j * pos * theta ** (-2 * i / Dr))
        k_pe += [keep(z.real), keep(z.imag)]
    return q_latent, kv, k_pe


def _tiny(seed, dyadic=False):
    rng = np.random.default_rng(500 + seed)
    dim, Rq, C, Dr, M = 6, 3, 4, 4, 3
    if dyadic:
        x = rng.integers(-3, 4, (M, dim)).astype(float)
        wq_a = rng.integers(-3, 4, (Rq, dim)) / 8.0
        wkv_a = rng.integers(-3, 4, (C + Dr, dim)) / 8.0
        gain = rng.integers(1, 4, C) / 2.0
    else:
        x = rng.standard_normal((M, dim))
        wq_a = rng.standard_normal((Rq, dim))
        wkv_a = rng.standard_normal((C + Dr, dim))
        gain = rng.uniform(0.5, 1.5, C)
    pos = np.array([0, 5, 1234])
    return dict(x=x, wq_a=wq_a, wkv_a=wkv_a, gain=gain, pos=pos, C=C, Dr=Dr)


def _max_err_vs_brute(S, precision="exact"):
    q, kv, pe = oracle.produce_latents(S["x"], S["wq_a"], S["wkv_a"], S["gain"], S["pos"],
                                       kv_lora=S["C"], rope=S["Dr"], precision=precision)
    err = 0.0
    for m in range(len(S["x"])):
        bq, bkv, bpe = _brute_produce_one(list(S["x"][m]), S["wq_a"].tolist(), S["wkv_a"].tolist(),
                                          list(S["gain"]), int(S["pos"][m]), S["C"], S["Dr"],
                                          10000.0, 1e-6,
                                          rnd=_bf16_bits if precision == "bf16" else None)
        err = max(err, float(np.max(np.abs(q[m] - bq))), float(np.max(np.abs(kv[m] - bkv))),
                  float(np.max(np.abs(pe[m] - bpe))))
    return err


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_producer_matches_enumeration(seed):
    assert _max_err_vs_brute(_tiny(seed)) < 1e-12


@pytest.mark.parametrize("seed", [0, 1])
def test_producer_bf16_mode_matches_rounded_enumeration_bit_for_bit(seed):
    """Dyadic inputs make every Linear output exact in float64, so the bf16 roundings (both
    Linear outputs, the normalised latent, the rotated key) compare bit for bit."""
    assert _max_err_vs_brute(_tiny(seed, dyadic=True), "bf16") == 0.0
    S = _tiny(seed, dyadic=True)
    a = oracle.produce_latents(S["x"], S["wq_a"], S["wkv_a"], S["gain"], S["pos"], kv_lora=4,
                               rope=4, precision="bf16")
    b = oracle.produce_latents(S["x"], S["wq_a"], S["wkv_a"], S["gain"], S["pos"], kv_lora=4,
                               rope=4)
    assert not np.array_equal(a[1], b[1])   # the roundings are active


def test_kv_norm_of_constant_latent_is_the_gain():
    """wkv_a rows that make every latent feature equal c: kv = gain * c / sqrt(c^2 + eps)."""
    dim, C, Dr = 8, 512, 64
    gain = np.random.default_rng(3).uniform(0.5, 1.5, C)
    x = np.zeros((1, dim))
    x[0, 0] = 1.0
    for c in (0.25, 3.0):
        wkv_a = np.zeros((C + Dr, dim))
        wkv_a[:C, 0] = c
        _, kv, _ = oracle.produce_latents(x, np.zeros((4, dim)), wkv_a, gain, np.array([7]))
        np.testing.assert_allclose(kv[0], gain * c / math.sqrt(c * c + 1e-6), rtol=1e-14)


def test_rotary_key_is_unrotated_at_position_zero_and_keeps_pair_norms():
    rng = np.random.default_rng(4)
    dim, C, Dr = 16, 512, 64
    x = rng.standard_normal((3, dim))
    wkv_a = rng.standard_normal((C + Dr, dim))
    _, _, pe0 = oracle.produce_latents(x, np.zeros((2, dim)), wkv_a, np.ones(C), np.zeros(3, int))
    np.testing.assert_array_equal(pe0, x @ wkv_a[C:].T)
    _, _, pe = oracle.produce_latents(x, np.zeros((2, dim)), wkv_a, np.ones(C),
                                      np.array([1, 100, 32768]))
    n_in = pe0[:, 0::2] ** 2 + pe0[:, 1::2] ** 2
    np.testing.assert_allclose(pe[:, 0::2] ** 2 + pe[:, 1::2] ** 2, n_in, rtol=1e-12)


def test_written_row_is_what_a_single_key_decode_returns():
    """Write-then-attend: a sequence whose only key is the produced row (start_pos = 0) decodes to
    W_UV · kv (one key: softmax weight 1), whatever the query."""
    rng = np.random.default_rng(5)
    H, R, C, Dn, Dr, Dv, dim = 2, 8, 4, 2, 2, 2, 6
    x = rng.standard_normal((1, dim))
    wq_a = rng.standard_normal((R, dim))
    wkv_a = rng.standard_normal((C + Dr, dim))
    q_lat, kv, pe = oracle.produce_latents(x, wq_a, wkv_a, np.ones(C), np.array([0]), kv_lora=C,
                                           rope=Dr)
    cache = oracle.write_cache_rows(np.full((1, 3, C + Dr), np.nan), kv, pe, [0], [0], kv_lora=C)
    assert np.all(np.isnan(cache[0, 1:])) and np.array_equal(cache[0, 0], np.r_[kv[0], pe[0]])
    wq_b = rng.standard_normal((H * (Dn + Dr), R))
    wkv_b = rng.standard_normal((H * (Dn + Dv), C))
    r = oracle.decode(q_lat, np.ones(R), wq_b, wkv_b, cache, np.array([0]), n_heads=H, kv_lora=C,
                      nope=Dn, rope=Dr, v=Dv)
    w_uv = wkv_b.reshape(H, Dn + Dv, C)[:, Dn:]
    np.testing.assert_allclose(r["out"][0], w_uv @ kv[0], rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------------------------------
# Planted mistakes in the producer (on the CPU): each must be caught by the enumeration
# ------------------------------------------------------------------------------------------
_REAL_RMS = om.rmsnorm
_REAL_ROPE = om.apply_rope_interleaved


def _rope_on_wrong_slice(x, pos, theta=10000.0):     # rotates the first pairs of the row
    return _REAL_ROPE(np.asarray(x)[..., ::-1], pos, theta)[..., ::-1]


def _rms_no_eps_sqrt_of_sum(x, gamma, eps=1e-6, residual=None):
    u = np.asarray(x, np.float64)
    return gamma * u / np.sqrt(np.sum(u * u, axis=-1, keepdims=True)), None


def _rope_inverse(x, pos, theta=10000.0):
    return _REAL_ROPE(x, -np.asarray(pos), theta)


@pytest.mark.parametrize("target,replacement", [
    ("apply_rope_interleaved", _rope_on_wrong_slice),
    ("apply_rope_interleaved", _rope_inverse),
    ("rmsnorm", _rms_no_eps_sqrt_of_sum),
])
def test_planted_producer_mistake_is_caught(monkeypatch, target, replacement):
    S = _tiny(0)
    assert _max_err_vs_brute(S) < 1e-12
    monkeypatch.setattr(om, target, replacement)
    assert _max_err_vs_brute(S) > 1e-6


def test_swapped_split_order_is_caught():
    """Reading the rotary key from the first 64 outputs instead of the last is caught."""
    S = _tiny(1)
    w = S["wkv_a"]
    swapped = np.concatenate([w[S["C"]:], w[:S["C"]]])   # rope rows first
    S2 = dict(S, wkv_a=swapped)
    q, kv, pe = oracle.produce_latents(S2["x"], S2["wq_a"], S2["wkv_a"], S2["gain"], S2["pos"],
                                       kv_lora=4, rope=4)
    bq, bkv, bpe = _brute_produce_one(list(S["x"][1]), S["wq_a"].tolist(), w.tolist(),
                                      list(S["gain"]), int(S["pos"][1]), 4, 4, 10000.0, 1e-6)
    assert np.max(np.abs(kv[1] - bkv)) > 1e-6
