"""Pins of the fp64 oracle against facts the source pages and the mathematics fix.

None of these tests needs a GPU.  Each pin is chosen so that a plausible slip in the oracle (a
dropped term, a wrong sign or index, a transposed operand, the wrong weight slice) fails at least
one of them: the brute-force enumeration, the absorbed/non-absorbed agreement, the closed forms
and the page figures are independent of the oracle's own loop structure.
"""
import cmath
import json
import math
import os
import struct

import numpy as np
import pytest
import scipy.special

import oracle
from mla_synth import bf16_bits_to_f64, f32_to_bf16_bits, make_inputs, workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")


@pytest.fixture(scope="module")
def figures():
    with open(GOLDEN) as f:
        return json.load(f)


def _rand_setup(rng, H=4, R=24, C=16, Dn=6, Dr=8, Dv=5, B=3, keys=9):
    return dict(
        x=rng.standard_normal((B, R)), gamma=rng.uniform(0.5, 1.5, R),
        wq_b=rng.standard_normal((H * (Dn + Dr), R)) / math.sqrt(R),
        wkv_b=rng.standard_normal((H * (Dn + Dv), C)) / math.sqrt(C),
        cache=rng.standard_normal((B, keys, C + Dr)),
        dims=dict(n_heads=H, kv_lora=C, nope=Dn, rope=Dr, v=Dv), R=R, B=B, keys=keys)


# ------------------------------------------------------------------------------------------
# Page figures
# ------------------------------------------------------------------------------------------
def test_wq_b_parameter_count(figures):
    """Query heads page, parameter table: 1,536x16,384 + 1,536x8,192 = 37,748,736 for H=128."""
    f = figures["wq_b_parameters"]
    H, R, Dn, Dr = f["n_heads"], f["q_lora_rank"], f["qk_nope_head_dim"], f["qk_rope_head_dim"]
    w = np.zeros((H * (Dn + Dr), R), dtype=np.float32)
    w_uq, w_qr = oracle.split_wq_b(w, H, Dn, Dr)
    assert w_uq.size == f["content_up_projection"]
    assert w_qr.size == f["rotary_up_projection"]
    assert w.size == f["per_instance_total"] == w_uq.size + w_qr.size
    assert f["per_instance_total"] * 58 == f["across_58_blocks"]


def test_w_uv_parameter_count(figures):
    """Kimi-K2 value_states page: value up-projection of 4,194,304 parameters (H=64)."""
    f = figures["w_uv_parameters"]
    H, C, Dv = f["n_heads"], f["kv_lora_rank"], f["v_head_dim"]
    wkv_b = np.zeros((H * (128 + Dv), C), dtype=np.float32)
    _, w_uv = oracle.split_wkv_b(wkv_b, H, 128, Dv)
    assert w_uv.size == f["per_instance_total"]
    assert f["per_instance_total"] * 60 == f["across_60_blocks"]


def test_page_shapes(figures):
    """In/out shapes printed on the Query heads and value_states pages."""
    rng = np.random.default_rng(1)
    B, T, H = 2, 3, 128
    f = figures["query_heads_shapes"]
    y = rng.standard_normal((B * T, f["in_q_latent"][2]))
    wq_b = rng.standard_normal((H * 192, 1536)) * 0.01
    q_nope, q_pe = oracle.query_heads(y, wq_b, H, 128, 64, np.arange(B * T) % T)
    Q = np.concatenate([q_nope, q_pe], -1).reshape(B, T, H, 192).transpose(0, 2, 1, 3)
    assert list(Q.shape) == [B, f["out_Q"][1], T, f["out_Q"][3]]
    assert len(oracle.rope_frequencies(64)) == f["in_R"][1]
    g = figures["value_states_shapes"]
    wkv_b = rng.standard_normal((64 * 256, 512))
    _, w_uv = oracle.split_wkv_b(wkv_b, 64, 128, 128)
    v = oracle.expand_w_uv(rng.standard_normal((B, 1, 64, g["in"][2])), w_uv)
    assert list(v.transpose(0, 2, 1, 3).shape) == [B, g["out"][1], 1, g["out"][3]]


# ------------------------------------------------------------------------------------------
# RMSNorm
# ------------------------------------------------------------------------------------------
def test_rmsnorm_constant_vector_gives_gain():
    gamma = np.random.default_rng(2).uniform(0.5, 1.5, 1536)
    for c in (0.5, 3.0, 100.0):
        y, _ = oracle.rmsnorm(np.full(1536, c), gamma, 1e-6)
        np.testing.assert_allclose(y, gamma * c / math.sqrt(c * c + 1e-6), rtol=1e-14)
        assert np.max(np.abs(y / gamma - 1)) <= 1e-6 / (2 * c * c) * 1.01
    y, _ = oracle.rmsnorm(np.full(1536, -2.0), gamma, 1e-6)
    np.testing.assert_allclose(y, -gamma, rtol=1e-6)


def test_rmsnorm_matches_l2_norm_form():
    """With eps = 0, y = gamma * x * sqrt(d) / ||x||_2 (textbook form via numpy's norm)."""
    rng = np.random.default_rng(3)
    x, g = rng.standard_normal((5, 64)), rng.uniform(0.5, 1.5, 64)
    y, _ = oracle.rmsnorm(x, g, 0.0)
    ref = g * x * math.sqrt(64) / np.linalg.norm(x, axis=-1, keepdims=True)
    np.testing.assert_allclose(y, ref, rtol=1e-13)
    y2, _ = oracle.rmsnorm(7.5 * x, g, 0.0)
    np.testing.assert_allclose(y2, y, rtol=1e-13)


def test_rmsnorm_residual_adds_first():
    rng = np.random.default_rng(4)
    x, r, g = rng.standard_normal((3, 32)), rng.standard_normal((3, 32)), rng.uniform(0.5, 1.5, 32)
    y, res = oracle.rmsnorm(x, g, 1e-6, r)
    y_ref, _ = oracle.rmsnorm(x + r, g, 1e-6)
    np.testing.assert_array_equal(res, x + r)
    np.testing.assert_allclose(y, y_ref, rtol=1e-15)
    m2 = np.mean((x + r) ** 2, axis=-1, keepdims=True)
    np.testing.assert_allclose(y, g * (x + r) / np.sqrt(m2 + 1e-6), rtol=1e-14)


# ------------------------------------------------------------------------------------------
# RoPE
# ------------------------------------------------------------------------------------------
def test_rope_frequencies_closed_form():
    f = oracle.rope_frequencies(64, 10000.0)
    assert f[0] == 1.0
    assert math.isclose(f[16], 0.01, rel_tol=1e-14)        # 10000^(-32/64)
    assert math.isclose(f[31], 10000.0 ** (-62 / 64), rel_tol=1e-14)


def test_rope_identity_at_zero_and_norm_preserving():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 64))
    np.testing.assert_array_equal(oracle.apply_rope_interleaved(x, np.zeros(7)), x)
    y = oracle.apply_rope_interleaved(x, np.arange(7) * 1000 + 3)
    n_in = x[:, 0::2] ** 2 + x[:, 1::2] ** 2
    n_out = y[:, 0::2] ** 2 + y[:, 1::2] ** 2
    np.testing.assert_allclose(n_out, n_in, rtol=1e-12)


def test_rope_is_complex_rotation_of_adjacent_pairs():
    """Interleaved RoPE == multiply the complex number x[2i] + i x[2i+1] by exp(i pos theta_i)."""
    rng = np.random.default_rng(6)
    x = rng.standard_normal(64)
    for pos in (1, 17, 4096, 32768):
        y = oracle.apply_rope_interleaved(x, np.array(pos))
        for i in range(32):
            z = complex(x[2 * i], x[2 * i + 1]) * cmath.exp(1j * pos * 10000.0 ** (-2 * i / 64))
            tol = 1e-13 * (1 + pos)    # the angle pos*theta_i carries ~1 ulp of pos
            assert abs(y[2 * i] - z.real) < tol and abs(y[2 * i + 1] - z.imag) < tol
    # pair 0 at position 1 rotates (1, 0) by exactly one radian, counter-clockwise
    e = np.zeros(64)
    e[0] = 1.0
    y = oracle.apply_rope_interleaved(e, np.array(1))
    assert math.isclose(y[0], math.cos(1.0)) and math.isclose(y[1], math.sin(1.0))


def test_rope_relative_position():
    """<R(p) a, R(q) b> = <a, R(q - p) b>: the score depends on positions only through q - p."""
    rng = np.random.default_rng(7)
    a, b = rng.standard_normal(64), rng.standard_normal(64)
    for p, q in ((3, 10), (100, 2000), (4096, 4097)):
        lhs = oracle.apply_rope_interleaved(a, np.array(p)) @ oracle.apply_rope_interleaved(b, np.array(q))
        rhs = a @ oracle.apply_rope_interleaved(b, np.array(q - p))
        assert abs(lhs - rhs) < 1e-10 * (1 + abs(lhs))


# ------------------------------------------------------------------------------------------
# Softmax
# ------------------------------------------------------------------------------------------
def test_softmax_against_scipy():
    rng = np.random.default_rng(8)
    s = rng.standard_normal((6, 300)) * 5
    p, lse = oracle.softmax_fp(s)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(p, scipy.special.softmax(s, axis=-1), rtol=1e-12)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(s, axis=-1), rtol=1e-13)
    p2, lse2 = oracle.softmax_fp(s + 1234.5)
    np.testing.assert_allclose(p2, p, rtol=1e-10)
    np.testing.assert_allclose(lse2 - lse, 1234.5, rtol=1e-12)


# ------------------------------------------------------------------------------------------
# Absorbed == non-absorbed (associativity of the two page forms)
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("seed", [0, 1])
def test_absorbed_equals_nonabsorbed_decode(seed):
    rng = np.random.default_rng(seed)
    S = _rand_setup(rng)
    d = S["dims"]
    pos = np.array([0, 4, 8])
    r = oracle.decode(S["x"], S["gamma"], S["wq_b"], S["wkv_b"], S["cache"], pos,
                      want_intermediates=True, **d)
    C, Dr = d["kv_lora"], d["rope"]
    for i, b in enumerate(range(S["B"])):
        n = pos[b] + 1
        o, lse = oracle.nonabsorbed_attention(
            r["q_nope"][i:i + 1], r["q_pe"][i:i + 1], S["cache"][b, :n, :C],
            S["cache"][b, :n, C:C + Dr], S["wkv_b"], d["n_heads"], q_positions=np.array([n - 1]),
            nope=d["nope"], v=d["v"])
        np.testing.assert_allclose(r["out"][i], o[0], rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(r["lse"][i], lse[0], rtol=1e-12)


def test_absorbed_equals_nonabsorbed_prefill_with_additive_mask():
    rng = np.random.default_rng(9)
    H, R, C, Dn, Dr, Dv = 3, 16, 12, 4, 6, 5
    T, sp = 5, 4
    x = rng.standard_normal((1, T, R))
    g = rng.uniform(0.5, 1.5, R)
    wq_b = rng.standard_normal((H * (Dn + Dr), R)) / 4
    wkv_b = rng.standard_normal((H * (Dn + Dv), C)) / 3.5
    cache = rng.standard_normal((1, sp + T, C + Dr))
    kw = dict(n_heads=H, kv_lora=C, nope=Dn, rope=Dr, v=Dv)
    r = oracle.prefill(x, g, wq_b, wkv_b, cache, sp, want_intermediates=True, **kw)
    it = r["intermediates"][0]
    o, lse = oracle.nonabsorbed_attention(it["q_nope"], it["q_pe"], cache[0, :, :C],
                                          cache[0, :, C:], wkv_b, H,
                                          q_positions=sp + np.arange(T), nope=Dn, v=Dv)
    np.testing.assert_allclose(r["out"][0], o, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(r["lse"][0], lse, rtol=1e-12)
    # a prefill token is the same as a decode step at position start_pos + t
    for t in range(T):
        dec = oracle.decode(x[:, t], g, wq_b, wkv_b, cache, np.array([sp + t]), **kw)
        np.testing.assert_allclose(r["out"][0, t], dec["out"][0], rtol=1e-12, atol=1e-14)


# ------------------------------------------------------------------------------------------
# Closed forms
# ------------------------------------------------------------------------------------------
def _w_uv_by_index(wkv_b, H, Dn, Dv, h):
    """The value rows of head h are rows h*(Dn+Dv)+Dn .. h*(Dn+Dv)+Dn+Dv-1 (last v rows)."""
    return np.array([wkv_b[h * (Dn + Dv) + Dn + d] for d in range(Dv)])


def test_single_key_output_is_w_uv_times_latent():
    rng = np.random.default_rng(10)
    S = _rand_setup(rng)
    d = S["dims"]
    r = oracle.decode(S["x"], S["gamma"], S["wq_b"], S["wkv_b"], S["cache"], np.zeros(3, int), **d)
    for b in range(3):
        for h in range(d["n_heads"]):
            ref = _w_uv_by_index(S["wkv_b"], d["n_heads"], d["nope"], d["v"], h) @ S["cache"][b, 0, :d["kv_lora"]]
            np.testing.assert_allclose(r["out"][b, h], ref, rtol=1e-12, atol=1e-14)


def test_identical_keys_make_output_query_independent():
    rng = np.random.default_rng(11)
    S = _rand_setup(rng)
    d = S["dims"]
    cache = np.repeat(S["cache"][:, :1], S["keys"], axis=1)
    pos = np.full(3, S["keys"] - 1)
    r1 = oracle.decode(S["x"], S["gamma"], S["wq_b"], S["wkv_b"], cache, pos, want_logits=True, **d)
    r2 = oracle.decode(-3 * S["x"] + 1, S["gamma"], S["wq_b"], S["wkv_b"], cache, pos, **d)
    np.testing.assert_allclose(r1["out"], r2["out"], rtol=1e-12, atol=1e-14)
    for b in range(3):
        s = r1["logits"][b]
        p = np.exp(s - r1["lse"][b][:, None])
        np.testing.assert_allclose(p, 1.0 / S["keys"], rtol=1e-12)


def test_zero_query_averages_latents():
    rng = np.random.default_rng(12)
    S = _rand_setup(rng)
    d = S["dims"]
    pos = np.array([2, 5, 8])
    r = oracle.decode(np.zeros_like(S["x"]), S["gamma"], S["wq_b"], S["wkv_b"], S["cache"], pos, **d)
    for b in range(3):
        mean = S["cache"][b, :pos[b] + 1, :d["kv_lora"]].mean(0)
        for h in range(d["n_heads"]):
            ref = _w_uv_by_index(S["wkv_b"], d["n_heads"], d["nope"], d["v"], h) @ mean
            np.testing.assert_allclose(r["out"][b, h], ref, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(r["lse"][b], math.log(pos[b] + 1) * np.ones(d["n_heads"]), rtol=1e-13)


# ------------------------------------------------------------------------------------------
# Brute force on tiny inputs (pure-Python scalar loops written from the pages' description)
# ------------------------------------------------------------------------------------------
def _bf16_bits(v: float) -> float:
    """Nearest bfloat16 value to the float64 ``v`` (ties to even), found by editing the IEEE-754
    bit pattern: keep the sign, the exponent and the top 7 of the 52 stored mantissa bits."""
    (u,) = struct.unpack("<Q", struct.pack("<d", v))
    drop = 52 - 7
    half = 1 << (drop - 1)
    keep_lsb = (u >> drop) & 1
    u = (u + half - 1 + keep_lsb) & ~((1 << drop) - 1)   # a carry may bump the exponent: correct
    (r,) = struct.unpack("<d", struct.pack("<Q", u))
    return r


def _brute_decode_one(x, gamma, wq_b, wkv_b, cache, pos, H, C, Dn, Dr, Dv, theta, eps,
                      rnd=None, trace=None):
    """Scalar enumeration of one decode row.  ``rnd`` (optional) rounds the query side where the
    pages' tensors are bf16: the RMSNorm output, the wq_b output, the rotated q_pe and the absorbed
    q_nope.  ``trace`` (a dict) receives those four query tensors."""
    keep = rnd if rnd is not None else (lambda v: v)
    R = len(x)
    ms = sum(v * v for v in x) / R
    y = [keep(gamma[j] * (x[j] / math.sqrt(ms + eps))) for j in range(R)]
    scale = (Dn + Dr) ** -0.5
    outs, lses = [], []
    if trace is not None:
        trace.update(y=y, q_nope=[], q_pe=[], q_lat=[])
    for h in range(H):
        qh = [keep(sum(y[k] * wq_b[h * (Dn + Dr) + j][k] for k in range(R))) for j in range(Dn + Dr)]
        q_nope, q_pe = qh[:Dn], qh[Dn:]
        q_rot = []
        for i in range(Dr // 2):
            z = complex(q_pe[2 * i], q_pe[2 * i + 1]) * cmath.exp(1j * pos * theta ** (-2 * i / Dr))
            q_rot += [keep(z.real), keep(z.imag)]
        q_lat = [keep(sum(q_nope[dd] * wkv_b[h * (Dn + Dv) + dd][c] for dd in range(Dn)))
                 for c in range(C)]
        if trace is not None:
            trace["q_nope"].append(q_nope)
            trace["q_pe"].append(q_rot)
            trace["q_lat"].append(q_lat)
        logits = []
        for t in range(pos + 1):
            acc = 0.0
            for c in range(C):
                acc += q_lat[c] * cache[t][c]
            acc += sum(q_rot[r] * cache[t][C + r] for r in range(Dr))
            logits.append(acc * scale)
        mx = max(logits)
        z = sum(math.exp(s - mx) for s in logits)
        p = [math.exp(s - mx) / z for s in logits]
        o_lat = [sum(p[t] * cache[t][c] for t in range(pos + 1)) for c in range(C)]
        outs.append([sum(o_lat[c] * wkv_b[h * (Dn + Dv) + Dn + dd][c] for c in range(C))
                     for dd in range(Dv)])
        lses.append(mx + math.log(z))
    return outs, lses


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(100 + seed)
    H, R, C, Dn, Dr, Dv, L = 2, 8, 4, 2, 2, 2, 4
    x = rng.integers(-3, 4, (2, R)).astype(float)
    x[x.sum(1) == 0, 0] = 1.0
    gamma = rng.integers(1, 4, R).astype(float) / 2
    wq_b = rng.integers(-2, 3, (H * (Dn + Dr), R)).astype(float) / 4
    wkv_b = rng.integers(-2, 3, (H * (Dn + Dv), C)).astype(float) / 2
    cache = rng.integers(-3, 4, (2, L, C + Dr)).astype(float)
    pos = np.array([L - 1, 1])
    r = oracle.decode(x, gamma, wq_b, wkv_b, cache, pos, n_heads=H, kv_lora=C, nope=Dn, rope=Dr,
                      v=Dv, theta=10000.0, eps=1e-6)
    for b in range(2):
        o, l = _brute_decode_one(list(x[b]), list(gamma), wq_b.tolist(), wkv_b.tolist(),
                                 cache[b].tolist(), int(pos[b]), H, C, Dn, Dr, Dv, 10000.0, 1e-6)
        np.testing.assert_allclose(r["out"][b], np.array(o), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(r["lse"][b], np.array(l), rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------------------------------------
# bf16 rounding of the oracle's "bf16" precision mode
# ------------------------------------------------------------------------------------------
def test_round_bf16_matches_torch_and_ties_to_even():
    import torch
    rng = np.random.default_rng(14)
    a = (rng.standard_normal(200000) * np.exp(rng.uniform(-20, 20, 200000))).astype(np.float32)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(oracle.round_bf16(a.astype(np.float64)), ref)
    # halfway cases: 1 + 2^-8 lies between 1 and 1 + 2^-7 -> even (1.0); 1 + 3*2^-8 -> 1 + 2^-6
    assert oracle.round_bf16(np.array(1 + 2.0 ** -8)) == 1.0
    assert oracle.round_bf16(np.array(1 + 3 * 2.0 ** -8)) == 1 + 2.0 ** -6
    # just above a tie (not representable in fp32) must round up, directly from float64
    assert oracle.round_bf16(np.array(1 + 2.0 ** -8 + 2.0 ** -40)) == 1 + 2.0 ** -7
    x = rng.standard_normal(1000)
    np.testing.assert_array_equal(oracle.round_bf16(oracle.round_bf16(x)), oracle.round_bf16(x))


def test_bf16_rounding_by_bits_matches_torch():
    """The enumeration's own bf16 rounding (bit editing) against torch's float32 -> bfloat16."""
    import torch
    rng = np.random.default_rng(15)
    a = (rng.standard_normal(20000) * np.exp(rng.uniform(-30, 30, 20000))).astype(np.float32)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(np.array([_bf16_bits(float(v)) for v in a]), ref)
    assert _bf16_bits(1 + 2.0 ** -8) == 1.0                 # tie, even neighbour below
    assert _bf16_bits(1 + 3 * 2.0 ** -8) == 1 + 2.0 ** -6   # tie, even neighbour above
    assert _bf16_bits(-(1 + 2.0 ** -8 + 2.0 ** -40)) == -(1 + 2.0 ** -7)
    assert _bf16_bits(2 - 2.0 ** -9) == 2.0                 # carry into the exponent


def _dyadic_setup(seed, L=5):
    """Small-integer / dyadic inputs: every sum of products the query side forms is exact in
    float64, so the only inexact steps are the RMSNorm square root and the RoPE angles, and the
    bf16 roundings can be compared bit for bit."""
    rng = np.random.default_rng(300 + seed)
    H, R, C, Dn, Dr, Dv = 2, 8, 4, 2, 4, 2
    x = rng.integers(-3, 4, (2, R)).astype(float)
    x[np.all(x == 0, axis=1), 0] = 1.0
    return dict(
        x=x, gamma=rng.integers(1, 4, R) / 2.0,
        wq_b=rng.integers(-3, 4, (H * (Dn + Dr), R)) / 8.0,
        wkv_b=rng.integers(-3, 4, (H * (Dn + Dv), C)) / 4.0,
        cache=rng.integers(-3, 4, (2, L, C + Dr)).astype(float),
        pos=np.array([L - 1, 2]), dims=dict(H=H, C=C, Dn=Dn, Dr=Dr, Dv=Dv))


def bf16_mode_mismatches(seed):
    """Oracle decode in query_precision="bf16" against the rounded scalar enumeration: the number
    of query elements (y, q_nope, q_pe, q_lat) that differ bit for bit, and the largest output /
    lse difference."""
    S = _dyadic_setup(seed)
    d = S["dims"]
    r = oracle.decode(S["x"], S["gamma"], S["wq_b"], S["wkv_b"], S["cache"], S["pos"],
                      n_heads=d["H"], kv_lora=d["C"], nope=d["Dn"], rope=d["Dr"], v=d["Dv"],
                      want_intermediates=True, query_precision="bf16")
    bad, err = 0, 0.0
    for b in range(2):
        tr = {}
        o, l = _brute_decode_one(list(S["x"][b]), list(S["gamma"]), S["wq_b"].tolist(),
                                 S["wkv_b"].tolist(), S["cache"][b].tolist(), int(S["pos"][b]),
                                 d["H"], d["C"], d["Dn"], d["Dr"], d["Dv"], 10000.0, 1e-6,
                                 rnd=_bf16_bits, trace=tr)
        for k in ("y", "q_nope", "q_pe", "q_lat"):
            bad += int(np.sum(np.asarray(r[k][b]) != np.asarray(tr[k])))
        err = max(err, float(np.max(np.abs(r["out"][b] - np.array(o)))),
                  float(np.max(np.abs(r["lse"][b] - np.array(l)))))
    return bad, err


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_bf16_query_mode_matches_rounded_enumeration(seed):
    """query_precision="bf16" rounds exactly where the pages' tensors are bf16: RMSNorm output
    ("Attention update" rmsnorm: ``.to(dtype)``), the wq_b Linear output and the rotated q_pe
    ("Query heads" mla-queries), the absorbed q_nope ("Attention update" mla-decode einsum)."""
    bad, err = bf16_mode_mismatches(seed)
    assert bad == 0
    assert err < 1e-12
    # the roundings are active on these inputs: the exact mode differs
    S = _dyadic_setup(seed)
    d = S["dims"]
    kw = dict(n_heads=d["H"], kv_lora=d["C"], nope=d["Dn"], rope=d["Dr"], v=d["Dv"],
              want_intermediates=True)
    ex = oracle.decode(S["x"], S["gamma"], S["wq_b"], S["wkv_b"], S["cache"], S["pos"], **kw)
    bq = oracle.decode(S["x"], S["gamma"], S["wq_b"], S["wkv_b"], S["cache"], S["pos"],
                       query_precision="bf16", **kw)
    for k in ("y", "q_nope", "q_pe", "q_lat"):
        assert not np.array_equal(ex[k], bq[k]), k


def test_bf16_query_mode_stays_close_to_exact():
    """The pages' bf16 query roundings move the output by far less than the parity bound."""
    w = workload("tiny_decode")
    inp = make_inputs(w, seed=2)
    args = (bf16_bits_to_f64(inp["q_latent"][:, 0]), inp["gamma"].astype(np.float64),
            bf16_bits_to_f64(inp["wq_b"]), bf16_bits_to_f64(inp["wkv_b"]),
            bf16_bits_to_f64(inp["cache"]), inp["start_pos"], 16)
    ex = oracle.decode(*args, want_intermediates=True)
    bq = oracle.decode(*args, want_intermediates=True, query_precision="bf16")
    assert np.max(np.abs(bq["out"] - ex["out"])) < 5e-3 * np.max(np.abs(ex["out"]))
    np.testing.assert_array_equal(bq["q_lat"], oracle.round_bf16(bq["q_lat"]))
    assert not np.array_equal(bq["q_lat"], ex["q_lat"])


# ------------------------------------------------------------------------------------------
# Input generator
# ------------------------------------------------------------------------------------------
def test_bf16_rounding_matches_torch():
    import torch
    rng = np.random.default_rng(13)
    a = np.concatenate([rng.standard_normal(100000).astype(np.float32),
                        np.array([1.00390625, 1.01171875, -3.0e38, 1e-40, 0.0], np.float32)])
    ours = f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


def test_generator_is_seeded_and_shaped():
    w = workload("tiny_decode")
    a, b = make_inputs(w, seed=0), make_inputs(w, seed=0)
    c = make_inputs(w, seed=1)
    for k in ("q_latent", "wq_b", "wkv_b", "cache"):
        np.testing.assert_array_equal(a[k], b[k])
    assert not np.array_equal(a["cache"], c["cache"])
    assert a["q_latent"].shape == (2, 1, 1536)
    assert a["wq_b"].shape == (16 * 192, 1536) and a["wkv_b"].shape == (16 * 256, 512)
    assert a["cache"].shape == (2, 129, 576)  # max_t = L + 1 and list(a["start_pos"]) == [128, 128]
    wq = bf16_bits_to_f64(a["wq_b"])
    assert abs(wq.std() * math.sqrt(1536) - 1) < 0.01
    wr = workload("ragged_decode", batch=8)
    r = make_inputs(wr, seed=0, tail="nan", max_t=40000)
    assert r["residual"] is not None
    assert np.all((r["start_pos"] >= 1024) & (r["start_pos"] <= 32768))
    b0 = int(r["n_keys"][0])
    assert np.all(r["cache"][0, b0:] == 0x7FC0) and not np.any(r["cache"][0, :b0] == 0x7FC0)
