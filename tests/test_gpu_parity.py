"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same seeded bf16
inputs.  Bounds: bf16 outputs |err| <= 1e-2 * max|ref| + 1e-3; probabilities within 1e-3."""
import math

import numpy as np
import pytest

from mla_cases import (LSE_ATOL, LSE_RTOL, PROB_TOL, assert_close_bf16, bf16_to_np, f64,
                       make_inputs, oracle_decode, oracle_parallel, to_device, workload)
from mla_synth import bf16_bits_to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_11_b200 import build
    build.build()


def _runtime(dev, w, max_rows, max_t):
    from head_latent_attention_11_b200.runtime import MLARuntime
    return MLARuntime(dev["gamma"], dev["wq_b"], dev["wkv_b"], n_heads=w.dims.n_heads,
                      max_rows=max_rows, max_seq_len=max_t, rope_theta=w.rope_theta,
                      rms_eps=w.rms_eps)


def _debug(rt, which, shape, dtype=torch.bfloat16):
    from head_latent_attention_11_b200 import mla_debug_copy
    t = torch.empty(shape, dtype=dtype, device="cuda")
    mla_debug_copy(rt.ctx, which, t, t.numel() * t.element_size(),
                   torch.cuda.current_stream().cuda_stream)
    return t


# ------------------------------------------------------------------------------------------
# a1 alone
# ------------------------------------------------------------------------------------------
@pytest.mark.parametrize("rows,dim,with_res", [(1, 1536, False), (37, 1536, True), (5, 512, True),
                                               (3, 4096, False)])
def test_rmsnorm_parity(rows, dim, with_res):
    import oracle
    from head_latent_attention_11_b200 import mla_rmsnorm
    from mla_synth import f32_to_bf16_bits
    rng = np.random.default_rng(rows * 7 + dim)
    x = f32_to_bf16_bits(rng.standard_normal((rows, dim)).astype(np.float32) * 3)
    r = f32_to_bf16_bits(rng.standard_normal((rows, dim)).astype(np.float32))
    g = rng.uniform(0.5, 1.5, dim).astype(np.float32)
    tx = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    tr = torch.from_numpy(r.view(np.int16)).view(torch.bfloat16).cuda() if with_res else None
    tg = torch.from_numpy(g).cuda()
    ty = torch.empty_like(tx)
    mla_rmsnorm(tx, tr, tg, rows, dim, 1e-6, ty, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    y_ref, u_ref = oracle.rmsnorm(bf16_bits_to_f64(x), g.astype(np.float64), 1e-6,
                                  bf16_bits_to_f64(r) if with_res else None)
    assert_close_bf16(f64(ty), y_ref, "rmsnorm y", rel=8e-3, abs_=0)
    if with_res:
        assert_close_bf16(f64(tr), u_ref, "residual out", rel=8e-3, abs_=0)


# ------------------------------------------------------------------------------------------
# decode
# ------------------------------------------------------------------------------------------
def _decode_case(w, seed=0, tail="zero", rows=None, check_intermediates=True, check_probs=True):
    """Decode through the C ABI against the oracle on every row (or ``rows``):
    * out, o_lat and the query intermediates against the exact oracle within the stated bound;
    * out within half that bound, probabilities within 1e-3 and lse within LSE_ATOL of the oracle
      that rounds the query where the pages' tensors are bf16 (the GPU rounds at those points)."""
    inp = make_inputs(w, seed=seed, tail=tail)
    dev = to_device(inp)
    B, H = w.batch, w.dims.n_heads
    max_t = inp["max_t"]
    rt = _runtime(dev, w, B, max_t)
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    logits = (torch.full((B, H, max_t), float("nan"), dtype=torch.float32, device="cuda")
              if check_probs else None)
    res = dev["residual"].reshape(B, -1).clone() if dev["residual"] is not None else None
    out = rt.decode(dev["q_latent"].reshape(B, -1), dev["start_pos"], dev["cache"], residual=res,
                    lse=lse, logits=logits)
    torch.cuda.synchronize()
    assert rt.sync_status() == 0
    ref = oracle_parallel("decode", inp, w, rows,
                          want_intermediates=check_intermediates or res is not None)
    refq = oracle_parallel("decode", inp, w, rows, want_logits=check_probs,
                           query_precision="bf16")
    sel = np.arange(B) if rows is None else np.asarray(rows)
    got = f64(out)[sel]
    assert_close_bf16(got, ref["out"], f"{w.name} out")
    assert_close_bf16(got, refq["out"], f"{w.name} out (bf16-query oracle)", rel=5e-3)
    np.testing.assert_allclose(lse.cpu().numpy()[sel], refq["lse"], atol=LSE_ATOL, rtol=LSE_RTOL)
    if res is not None:
        assert_close_bf16(f64(res)[sel], ref["residual_out"], "residual out", rel=8e-3, abs_=0)
    if check_intermediates:
        y = f64(_debug(rt, 0, (B, 1536)))[sel]
        assert_close_bf16(y, ref["y"], "y")
        qn = f64(_debug(rt, 1, (B, H, 128)))[sel]
        assert_close_bf16(qn, ref["q_nope"], "q_nope")
        qabs = f64(_debug(rt, 2, (B, 128, 576)))[sel]
        assert_close_bf16(qabs[:, :H, 512:], ref["q_pe"], "q_pe")
        assert np.all(qabs[:, H:] == 0), "padding heads must stay zero"
        assert_close_bf16(qabs[:, :H, :512], ref["q_lat"], "q_lat")
        olat = f64(_debug(rt, 3, (B, H, 512)))[sel]
        assert_close_bf16(olat, ref["o_lat"], "o_lat")
    if check_probs:
        lg = logits.cpu().numpy()
        lse_np = lse.cpu().numpy()
        for i, b in enumerate(sel):
            n = int(inp["start_pos"][b]) + 1
            s_ref = refq["logits"][i]
            s_got = lg[b, :, :n].astype(np.float64)
            assert np.all(np.isnan(lg[b, :, n:])), "logits written past the last key"
            p_got = np.exp(s_got - lse_np[b][:, None])
            p_ref = np.exp(s_ref - refq["lse"][i][:, None])
            assert float(np.max(np.abs(p_got - p_ref))) <= PROB_TOL, f"probabilities row {b}"
            np.testing.assert_allclose(p_got.sum(-1), 1.0, atol=PROB_TOL)
    rt.close()


def test_decode_tiny():
    _decode_case(workload("tiny_decode"))


def test_decode_tiny_nan_tail():
    _decode_case(workload("tiny_decode"), seed=3, tail="nan")


@pytest.mark.parametrize("H,B,L", [(16, 1, 0), (16, 3, 63), (64, 5, 64), (128, 4, 65),
                                   (128, 7, 300), (64, 9, 1000), (128, 3, 127), (16, 2, 128)])
def test_decode_edges(H, B, L):
    """One key (L=0), ragged tile tails, batches cut across SM pairs."""
    from mla_synth import MLADims
    w = workload("tiny_decode", dims=MLADims(H), batch=B, cache_len=L)
    _decode_case(w, seed=H + B + L, tail="nan")


def test_decode_repeat_is_bitwise_stable():
    """Rows cut across SM pairs, debug logits on (which skews the two CTAs of a pair): repeated
    calls must give bit-identical results within the bound (guards the score exchange)."""
    from mla_synth import MLADims
    w = workload("tiny_decode", dims=MLADims(128), batch=7, cache_len=300)
    inp = make_inputs(w, seed=435, tail="nan")
    dev = to_device(inp)
    rt = _runtime(dev, w, w.batch, inp["max_t"])
    ref = oracle_decode(inp, w)
    logits = torch.full((w.batch, 128, inp["max_t"]), float("nan"), device="cuda")
    first = None
    for _ in range(12):
        out = rt.decode(dev["q_latent"].reshape(w.batch, -1), dev["start_pos"], dev["cache"],
                        logits=logits)
        torch.cuda.synchronize()
        got = bf16_to_np(out)
        if first is None:
            first = got
            assert_close_bf16(f64(out), ref["out"], "repeat out")
        else:
            assert np.array_equal(got, first), "results differ between identical calls"
    assert rt.sync_status() == 0
    rt.close()


def test_decode_ragged_small():
    from mla_synth import MLADims
    w = workload("ragged_decode", dims=MLADims(128), batch=6, ragged=(1, 3000))
    _decode_case(w, seed=11, tail="nan")


def test_decode_v32_full():
    """DeepSeek-V3.2-shaped decode at full size (B=32, H=128, L=4096), every row."""
    _decode_case(workload("v32_decode"))


def test_decode_kimi_full():
    """Kimi-K2-shaped decode at full size (B=128, H=64, L=2048), every row."""
    _decode_case(workload("kimi_decode"))


def test_decode_ragged_full():
    """Ragged long-context decode at full size (B=64, L_b ~ U{1024..32768}, residual), every
    row, probabilities included; cache rows past each sequence's end hold NaN."""
    _decode_case(workload("ragged_decode"), tail="nan")


# ------------------------------------------------------------------------------------------
# prefill
# ------------------------------------------------------------------------------------------
def _prefill_case(w, seed=0, tokens=None, tail="zero"):
    inp = make_inputs(w, seed=seed, tail=tail)
    dev = to_device(inp)
    B, T, H = w.batch, w.tokens, w.dims.n_heads
    rt = _runtime(dev, w, B * T, inp["max_t"])
    lse = torch.empty(B, T, H, dtype=torch.float32, device="cuda")
    res = dev["residual"].clone() if dev["residual"] is not None else None
    out = rt.prefill(dev["q_latent"], w.prefill_start, dev["cache"], residual=res, lse=lse)
    torch.cuda.synchronize()
    assert rt.sync_status() == 0
    sel = np.arange(T) if tokens is None else np.asarray(tokens)
    ref = oracle_parallel("prefill", inp, w, sel)
    # the bf16-query oracle (tighter bound, lse) on every token of small chunks, and on every
    # 8th token plus the last of large ones
    selq = sel if len(sel) <= 256 else np.unique(np.concatenate([sel[::8], sel[-1:]]))
    refq = oracle_parallel("prefill", inp, w, selq, query_precision="bf16")
    got = f64(out)
    assert_close_bf16(got[:, sel], ref["out"], f"{w.name} out")
    assert_close_bf16(got[:, selq], refq["out"], f"{w.name} out (bf16-query oracle)", rel=5e-3)
    np.testing.assert_allclose(lse.cpu().numpy()[:, selq], refq["lse"], atol=LSE_ATOL,
                               rtol=LSE_RTOL)
    rt.close()


@pytest.mark.parametrize("B,T,sp,H", [(1, 1, 0, 128), (1, 5, 0, 16), (2, 70, 100, 64),
                                      (1, 200, 200, 128), (3, 33, 1, 16), (1, 130, 63, 128)])
def test_prefill_small(B, T, sp, H):
    from mla_synth import MLADims
    w = workload("prefill_chunk", dims=MLADims(H), batch=B, tokens=T, prefill_start=sp)
    _prefill_case(w, seed=B * 1000 + T + sp, tail="nan")


def test_prefill_with_residual():
    from mla_synth import MLADims
    w = workload("prefill_chunk", dims=MLADims(64), batch=2, tokens=40, prefill_start=30,
                 residual=True)
    _prefill_case(w, seed=5)


def test_prefill_chunk_full():
    """Prefill chunk at full size (T=2048 after 2048, H=128), every token."""
    _prefill_case(workload("prefill_chunk"))


# ------------------------------------------------------------------------------------------
# device-side argument check
# ------------------------------------------------------------------------------------------
def test_decode_bad_start_pos_reports_status():
    from head_latent_attention_11_b200 import STATUS
    w = workload("tiny_decode")
    inp = make_inputs(w, seed=1)
    dev = to_device(inp)
    rt = _runtime(dev, w, w.batch, inp["max_t"])
    sp = dev["start_pos"].clone()
    sp[1] = inp["max_t"] + 5          # beyond the cache: recorded, clamped, no fault
    rt.decode(dev["q_latent"].reshape(w.batch, -1), sp, dev["cache"])
    assert STATUS[rt.sync_status()] == "MLA_ERR_DEVICE_ARG"
    assert rt.sync_status() == 0      # the status word is cleared by reading it
    rt.close()
