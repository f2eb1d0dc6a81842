"""Pins of the oracle's non-absorbed prefill and output projection ("Kimi-K2 · value_states"
mla-prefill: per-head keys [k_nope ‖ k_pe] and values rebuilt from the latent, additive causal
mask, fp32 softmax; "DeepSeek-V3.2-Exp · Attention update" mla-output: wo on the flattened heads).
No GPU needed."""
import numpy as np
import pytest

import oracle
import oracle.mla_oracle as om


def _setup(seed):
    rng = np.random.default_rng(700 + seed)
    H, R, C, Dn, Dr, Dv, dim = 3, 16, 12, 4, 6, 5, 7
    T, sp = 5, 4
    return dict(x=rng.standard_normal((2, T, R)), g=rng.uniform(0.5, 1.5, R),
                wq_b=rng.standard_normal((H * (Dn + Dr), R)) / 4,
                wkv_b=rng.standard_normal((H * (Dn + Dv), C)) / 3.5,
                cache=rng.standard_normal((2, sp + T, C + Dr)),
                wo=rng.standard_normal((dim, H * Dv)),
                kw=dict(n_heads=H, kv_lora=C, nope=Dn, rope=Dr, v=Dv), T=T, sp=sp, H=H, Dv=Dv,
                dim=dim)


@pytest.mark.parametrize("seed", [0, 1])
def test_nonabsorbed_prefill_equals_absorbed_prefill(seed):
    """Associativity of the two page forms (the absorbed chunk is pinned by brute force)."""
    S = _setup(seed)
    a = oracle.prefill(S["x"], S["g"], S["wq_b"], S["wkv_b"], S["cache"], S["sp"], **S["kw"])
    n = oracle.nonabsorbed_prefill(S["x"], S["g"], S["wq_b"], S["wkv_b"], S["cache"], S["sp"],
                                   **S["kw"])
    np.testing.assert_allclose(n["out"], a["out"], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(n["lse"], a["lse"], rtol=1e-12)


def test_output_projection_is_the_flattened_sum():
    """y[i] = sum over heads h and value features d of wo[i, h*v + d] * o[h, d] — enumerated."""
    S = _setup(2)
    o = np.random.default_rng(3).standard_normal((2, 3, S["H"], S["Dv"]))
    y = oracle.output_projection(o, S["wo"])
    for b in range(2):
        for t in range(3):
            for i in range(S["dim"]):
                ref = sum(S["wo"][i][h * S["Dv"] + d] * o[b, t, h, d]
                          for h in range(S["H"]) for d in range(S["Dv"]))
                assert abs(y[b, t, i] - ref) < 1e-12


def test_output_projection_with_head_selecting_weight():
    """A wo that copies head h's feature d to output i returns exactly that feature."""
    H, Dv = 4, 3
    o = np.random.default_rng(5).standard_normal((H, Dv))
    wo = np.zeros((2, H * Dv))
    wo[0, 2 * Dv + 1] = 1.0   # head 2, feature 1
    wo[1, 3 * Dv + 0] = 1.0   # head 3, feature 0
    y = oracle.output_projection(o, wo)
    assert y[0] == o[2, 1] and y[1] == o[3, 0]


def test_prefill_with_wo_applies_it_to_every_token():
    S = _setup(4)
    r = oracle.nonabsorbed_prefill(S["x"], S["g"], S["wq_b"], S["wkv_b"], S["cache"], S["sp"],
                                   wo=S["wo"], **S["kw"])
    flat = r["out"].reshape(2, S["T"], -1)
    np.testing.assert_allclose(r["y"], flat @ S["wo"].T, rtol=1e-13)


def _flatten_head_major_wrong(o, wo):   # d-major instead of h-major flattening
    o = np.asarray(o, np.float64)
    flat = np.swapaxes(o, -1, -2).reshape(o.shape[:-2] + (o.shape[-2] * o.shape[-1],))
    return flat @ np.asarray(wo, np.float64).T


def test_planted_flatten_order_mistake_is_caught(monkeypatch):
    S = _setup(2)
    o = np.random.default_rng(3).standard_normal((S["H"], S["Dv"]))
    ref = np.array([sum(S["wo"][i][h * S["Dv"] + d] * o[h, d] for h in range(S["H"])
                        for d in range(S["Dv"])) for i in range(S["dim"])])
    np.testing.assert_allclose(om.output_projection(o, S["wo"]), ref, rtol=1e-12)
    monkeypatch.setattr(om, "output_projection", _flatten_head_major_wrong)
    assert np.max(np.abs(om.output_projection(o, S["wo"]) - ref)) > 1e-6
