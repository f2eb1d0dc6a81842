"""Plant plausible mistakes in the oracle (on the CPU) and check that the pins catch them.

Each mutation replaces one oracle step with a wrong variant for the duration of one test; the
brute-force enumeration or the closed-form pins must then disagree with the oracle.
"""
import numpy as np
import pytest

import oracle
import oracle.mla_oracle as om
from test_oracle_pins import _brute_decode_one, bf16_mode_mismatches


def _max_err_vs_brute(seed=0):
    rng = np.random.default_rng(200 + seed)
    H, R, C, Dn, Dr, Dv, L = 2, 8, 4, 2, 2, 2, 4
    x = rng.standard_normal((2, R))
    gamma = rng.uniform(0.5, 1.5, R)
    wq_b = rng.standard_normal((H * (Dn + Dr), R))
    wkv_b = rng.standard_normal((H * (Dn + Dv), C))
    cache = rng.standard_normal((2, L, C + Dr))
    pos = np.array([L - 1, 2])
    r = om.decode(x, gamma, wq_b, wkv_b, cache, pos, n_heads=H, kv_lora=C, nope=Dn, rope=Dr, v=Dv)
    err = 0.0
    for b in range(2):
        o, l = _brute_decode_one(list(x[b]), list(gamma), wq_b.tolist(), wkv_b.tolist(),
                                 cache[b].tolist(), int(pos[b]), H, C, Dn, Dr, Dv, 10000.0, 1e-6)
        err = max(err, float(np.max(np.abs(r["out"][b] - np.array(o)))),
                  float(np.max(np.abs(r["lse"][b] - np.array(l)))))
    return err


def _no_pe_scores(q_lat, q_pe, kv, pe, scale):
    return (q_lat @ kv.T) * scale


def _swapped_wkv(wkv_b, n_heads, nope, v):
    w = np.asarray(wkv_b, dtype=np.float64).reshape(n_heads, nope + v, -1)
    return w[:, v:, :], w[:, :v, :]


def _rope_negative_angle(x, pos, theta=10000.0):
    return _ORIG_ROPE(x, -np.asarray(pos), theta)


def _rms_no_mean(x, gamma, eps=1e-6, residual=None):
    u = np.asarray(x, np.float64) + (0 if residual is None else residual)
    y = gamma * u / np.sqrt(np.sum(u * u, axis=-1, keepdims=True) + eps)
    return y, (u if residual is not None else None)


def _absorb_wrong_head(q_nope, w_uk):
    return np.einsum("mhd,hdc->mhc", q_nope, w_uk[::-1])


def _pv_transposed_keys(p, kv):
    return p[:, ::-1] @ kv


_ORIG_ROPE = om.apply_rope_interleaved


@pytest.mark.parametrize("name,target,replacement", [
    ("dropped rope term", "latent_scores", _no_pe_scores),
    ("rope sign", "apply_rope_interleaved", _rope_negative_angle),
    ("W_UK/W_UV slices swapped", "split_wkv_b", _swapped_wkv),
    ("rmsnorm sum instead of mean", "rmsnorm", _rms_no_mean),
    ("absorb uses another head", "absorb_w_uk", _absorb_wrong_head),
    ("weighted sum over reversed keys", "latent_weighted_sum", _pv_transposed_keys),
])
def test_planted_mistake_is_caught(monkeypatch, name, target, replacement):
    assert _max_err_vs_brute() < 1e-12
    monkeypatch.setattr(om, target, replacement)
    assert _max_err_vs_brute() > 1e-6, name


# ------------------------------------------------------------------------------------------
# Placement of the bf16 roundings in query_precision="bf16"
# ------------------------------------------------------------------------------------------
_ROUNDING_POINTS = ["RMSNorm output", "wq_b output (before RoPE)", "q_pe after RoPE",
                    "absorbed q_nope"]


@pytest.mark.parametrize("skip", range(4), ids=_ROUNDING_POINTS)
def test_dropped_bf16_rounding_is_caught(monkeypatch, skip):
    """Drop one of the four roundings (the oracle rounds in that order on every call); dropping
    the one after RoPE is the "round q_pe before RoPE instead of after" slip."""
    assert bf16_mode_mismatches(0)[0] == 0
    real = om.round_bf16
    calls = {"n": 0}

    def dropped(a):
        k = calls["n"]
        calls["n"] += 1
        return np.asarray(a, np.float64) if k % 4 == skip else real(a)

    monkeypatch.setattr(om, "round_bf16", dropped)
    bad = sum(bf16_mode_mismatches(s)[0] for s in range(3))
    assert bad > 0, _ROUNDING_POINTS[skip]


def test_wrong_rounding_format_is_caught(monkeypatch):
    monkeypatch.setattr(om, "round_bf16",
                        lambda a: np.asarray(a, np.float64).astype(np.float16).astype(np.float64))
    assert bf16_mode_mismatches(0)[0] > 0
