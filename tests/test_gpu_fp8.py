"""GPU parity of the path with FP8 block-scaled weights (mla_init_fp8): the GEMMs dequantise
wq_b / wkv_b block by block; the reference is the oracle on the weights the pages' weight_dequant
returns (oracle.dequant_block_fp8: code × block scale, rounded to bf16).  Same bounds as the bf16
path."""
import numpy as np
import pytest

import oracle
from mla_cases import (LSE_ATOL, LSE_RTOL, assert_close_bf16, f64, make_inputs, oracle_parallel,
                       to_device, workload)
from mla_synth import MLADims, f32_to_bf16_bits, make_fp8_weights

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_11_b200 import build
    build.build()


def _fp8_setup(w, seed):
    from head_latent_attention_11_b200.runtime import MLARuntime
    inp = make_inputs(w, seed=seed, tail="nan")
    f8 = make_fp8_weights(w, seed=seed)
    # the oracle's weights: what weight_dequant returns (bf16 values), as bf16 bit patterns
    deq = {k: f32_to_bf16_bits(oracle.dequant_block_fp8(f8[k], f8[k + "_scale"]).astype(np.float32))
           for k in ("wq_b", "wkv_b")}
    ref_inp = dict(inp, **deq)
    dev = to_device(inp)
    B, T = w.batch, w.tokens
    rt = MLARuntime(dev["gamma"], torch.from_numpy(f8["wq_b"]).cuda(),
                    torch.from_numpy(f8["wkv_b"]).cuda(), n_heads=w.dims.n_heads,
                    max_rows=B * T, max_seq_len=inp["max_t"], rope_theta=w.rope_theta,
                    rms_eps=w.rms_eps, wq_b_scale=torch.from_numpy(f8["wq_b_scale"]).cuda(),
                    wkv_b_scale=torch.from_numpy(f8["wkv_b_scale"]).cuda())
    return rt, inp, ref_inp, dev


@pytest.mark.parametrize("name,kw", [
    ("tiny_decode", {}),
    ("v32_decode", {}),
    ("kimi_decode", {}),                       # 128 rows: the separate combine path
    ("tiny_decode", dict(dims=MLADims(128), batch=7, cache_len=300)),
])
def test_fp8_decode(name, kw):
    w = workload(name, **kw)
    rt, inp, ref_inp, dev = _fp8_setup(w, seed=31)
    B, H = w.batch, w.dims.n_heads
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    out = rt.decode(dev["q_latent"].reshape(B, -1), dev["start_pos"], dev["cache"], lse=lse)
    torch.cuda.synchronize()
    assert rt.sync_status() == 0
    ref = oracle_parallel("decode", ref_inp, w, None)
    refq = oracle_parallel("decode", ref_inp, w, None, query_precision="bf16")
    got = f64(out)
    assert_close_bf16(got, ref["out"], f"{w.name} fp8 out")
    assert_close_bf16(got, refq["out"], f"{w.name} fp8 out (bf16-query oracle)", rel=5e-3)
    np.testing.assert_allclose(lse.cpu().numpy(), refq["lse"], atol=LSE_ATOL, rtol=LSE_RTOL)
    rt.close()


@pytest.mark.parametrize("B,T,sp,H", [(1, 200, 100, 128), (2, 70, 30, 64)])
def test_fp8_prefill_chunk(B, T, sp, H):
    """Wider token tiles (128 / 256) of the FP8 GEMMs."""
    w = workload("prefill_chunk", dims=MLADims(H), batch=B, tokens=T, prefill_start=sp)
    rt, inp, ref_inp, dev = _fp8_setup(w, seed=32)
    out = rt.prefill(dev["q_latent"], sp, dev["cache"])
    torch.cuda.synchronize()
    assert rt.sync_status() == 0
    ref = oracle_parallel("prefill", ref_inp, w, None)
    assert_close_bf16(f64(out), ref["out"], "fp8 prefill out")
    rt.close()
