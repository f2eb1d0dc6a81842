"""Pins of the oracle's index-mask (sparse) decode: the V3.2 mla-decode excerpt adds
``full(-inf).scatter_(-1, topk_indices, 0)`` to the scores ("DeepSeek-V3.2-Exp · Attention
update"), with ``topk = min(index_topk, end_pos)`` keys selected ("DeepSeek-V3.2-Exp · Indexer"
forward).  No GPU needed."""
import math

import numpy as np
import pytest

import oracle
import oracle.mla_oracle as om
from test_oracle_pins import _brute_decode_one, _rand_setup


def _decode(S, topk, pos, **kw):
    d = S["dims"]
    return oracle.decode(S["x"], S["gamma"], S["wq_b"], S["wkv_b"], S["cache"], pos, topk=topk,
                         **d, **kw)


def test_topk_covering_every_key_is_the_dense_decode():
    """min(index_topk, end_pos) = end_pos keeps every key: the mask is all zeros."""
    S = _rand_setup(np.random.default_rng(40))
    pos = np.array([3, 8, 0])
    full = np.full((3, 9), -1)
    for b in range(3):
        full[b, :pos[b] + 1] = np.random.default_rng(b).permutation(pos[b] + 1)
    a = _decode(S, full, pos)
    b = _decode(S, None, pos)
    np.testing.assert_array_equal(a["out"], b["out"])
    np.testing.assert_array_equal(a["lse"], b["lse"])


def test_topk_equals_dense_attention_over_the_selected_rows():
    """Attending to a selected subset = the dense decode over a cache that holds only those rows
    (in any order: the softmax and the weighted sum do not depend on key order).  The rotary rows
    of wq_b are zeroed so that the query does not depend on its position (the compact cache puts
    the query at another position)."""
    rng = np.random.default_rng(41)
    S = _rand_setup(rng, keys=12)
    d = S["dims"]
    wq_b = S["wq_b"].reshape(d["n_heads"], d["nope"] + d["rope"], -1).copy()
    wq_b[:, d["nope"]:] = 0.0
    S = dict(S, wq_b=wq_b.reshape(S["wq_b"].shape))
    pos = np.array([11, 7, 9])
    sel = [np.array([3, 0, 11, 5]), np.array([7]), np.array([2, 9, 4, 6, 1, 8])]
    K = max(len(s) for s in sel)
    topk = np.full((3, K), -1)
    for b, s in enumerate(sel):
        topk[b, :len(s)] = s
    r = _decode(S, topk, pos)
    for b, s in enumerate(sel):
        compact = S["cache"][b, s][None]
        ref = oracle.decode(S["x"][b:b + 1], S["gamma"], S["wq_b"], S["wkv_b"], compact,
                            np.array([len(s) - 1]), **d)
        np.testing.assert_allclose(r["out"][b], ref["out"][0], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(r["lse"][b], ref["lse"][0], rtol=1e-13)


def test_single_selected_key_returns_its_value():
    S = _rand_setup(np.random.default_rng(42))
    d = S["dims"]
    pos = np.array([8, 8, 8])
    topk = np.array([[5, -1], [0, -1], [8, -1]])
    r = _decode(S, topk, pos)
    w_uv = S["wkv_b"].reshape(d["n_heads"], d["nope"] + d["v"], -1)[:, d["nope"]:]
    for b, t in enumerate([5, 0, 8]):
        np.testing.assert_allclose(r["out"][b], w_uv @ S["cache"][b, t, :d["kv_lora"]],
                                   rtol=1e-12, atol=1e-14)


def _brute_sparse(S, b, pos, sel):
    """Scalar enumeration over the selected keys only (the mask written as a key set)."""
    d = S["dims"]
    sub = [S["cache"][b][t].tolist() for t in sorted(sel)]
    # enumerate with the RoPE position of the query = pos, keys = the selected rows
    H, C, Dn, Dr, Dv = d["n_heads"], d["kv_lora"], d["nope"], d["rope"], d["v"]
    x = list(S["x"][b])
    R = len(x)
    ms = sum(v * v for v in x) / R
    y = [S["gamma"][j] * (x[j] / math.sqrt(ms + 1e-6)) for j in range(R)]
    outs, lses = [], []
    import cmath
    for h in range(H):
        qh = [sum(y[k] * S["wq_b"][h * (Dn + Dr) + j][k] for k in range(R)) for j in range(Dn + Dr)]
        qn, qp = qh[:Dn], qh[Dn:]
        qr = []
        for i in range(Dr // 2):
            z = complex(qp[2 * i], qp[2 * i + 1]) * cmath.exp(1j * pos * 10000.0 ** (-2 * i / Dr))
            qr += [z.real, z.imag]
        ql = [sum(qn[dd] * S["wkv_b"][h * (Dn + Dv) + dd][c] for dd in range(Dn)) for c in range(C)]
        lg = [(sum(ql[c] * row[c] for c in range(C)) + sum(qr[r] * row[C + r] for r in range(Dr)))
              * (Dn + Dr) ** -0.5 for row in sub]
        mx = max(lg)
        z = sum(math.exp(v - mx) for v in lg)
        p = [math.exp(v - mx) / z for v in lg]
        ol = [sum(p[t] * sub[t][c] for t in range(len(sub))) for c in range(C)]
        outs.append([sum(ol[c] * S["wkv_b"][h * (Dn + Dv) + Dn + dd][c] for c in range(C))
                     for dd in range(Dv)])
        lses.append(mx + math.log(z))
    return np.array(outs), np.array(lses)


@pytest.mark.parametrize("seed", [0, 1])
def test_sparse_decode_matches_enumeration(seed):
    S = _rand_setup(np.random.default_rng(60 + seed), keys=10)
    pos = np.array([9, 6, 9])
    sel = [[1, 4, 9], [6, 0], [2, 3, 5, 7, 8]]
    topk = np.full((3, 5), -1)
    for b, s in enumerate(sel):
        topk[b, :len(s)] = s
    r = _decode(S, topk, pos)
    for b, s in enumerate(sel):
        o, l = _brute_sparse(S, b, int(pos[b]), s)
        np.testing.assert_allclose(r["out"][b], o, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(r["lse"][b], l, rtol=1e-13, atol=1e-13)


def _mask_complement(topk, end_pos):
    m = np.zeros(end_pos)
    idx = np.asarray(topk)
    m[idx[idx >= 0]] = -np.inf
    return m


def _mask_off_by_one(topk, end_pos):
    idx = np.asarray(topk)
    return _REAL_MASK(np.where(idx >= 0, np.minimum(idx + 1, end_pos - 1), idx), end_pos)


_REAL_MASK = om.index_mask


@pytest.mark.parametrize("replacement", [_mask_complement, _mask_off_by_one])
def test_planted_mask_mistake_is_caught(monkeypatch, replacement):
    S = _rand_setup(np.random.default_rng(61), keys=10)
    pos = np.array([9, 6, 9])
    topk = np.array([[1, 4, 9, -1, -1], [6, 0, -1, -1, -1], [2, 3, 5, 7, -1]])

    def err():
        r = _decode(S, topk, pos)
        e = 0.0
        for b in range(3):
            o, _ = _brute_sparse(S, b, int(pos[b]), [t for t in topk[b] if t >= 0])
            e = max(e, float(np.max(np.abs(r["out"][b] - o))))
        return e

    assert err() < 1e-12
    monkeypatch.setattr(om, "index_mask", replacement)
    assert err() > 1e-6
