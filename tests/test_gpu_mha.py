"""GPU parity of the non-absorbed prefill chunk (mla_prefill_chunk_mha: keys and values rebuilt per
head from the latent, causal multi-head attention, then wo) against the oracle's
nonabsorbed_prefill / output_projection on the same seeded inputs.
Bounds: bf16 outputs |err| <= 1e-2 * max|ref| + 1e-3.  lse: the GPU rounds the query (as the
absorbed path) and the rebuilt keys to bf16 (the pages' key_states are bf16), which moves a score
by at most 2^-8 * sum|q_d k_d| * scale (about 0.05 for these inputs): lse within 5e-2."""
import numpy as np
import pytest

import oracle
from mla_cases import assert_close_bf16, f64, make_inputs, to_device, workload
from mla_synth import MLADims, bf16_bits_to_f64, make_wo

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_11_b200 import build
    build.build()


def _oracle_mha(inp, w, wo, tokens=None):
    d = w.dims
    n = int(inp["start_pos"][0]) + w.tokens
    cache = bf16_bits_to_f64(inp["cache"][:, :n])
    return oracle.nonabsorbed_prefill(
        bf16_bits_to_f64(inp["q_latent"]), inp["gamma"].astype(np.float64),
        bf16_bits_to_f64(inp["wq_b"]), bf16_bits_to_f64(inp["wkv_b"]), cache,
        int(inp["start_pos"][0]), d.n_heads, wo=None if wo is None else bf16_bits_to_f64(wo),
        residual=None if inp["residual"] is None else bf16_bits_to_f64(inp["residual"]),
        theta=w.rope_theta, eps=w.rms_eps, tokens=tokens)


def _mha_case(w, seed, dim=512, tokens=None):
    from head_latent_attention_11_b200.runtime import MLARuntime
    inp = make_inputs(w, seed=seed, tail="nan")
    wo = make_wo(w, seed=seed, dim=dim)
    dev = to_device(inp)
    B, T, H = w.batch, w.tokens, w.dims.n_heads
    rt = MLARuntime(dev["gamma"], dev["wq_b"], dev["wkv_b"], n_heads=H, max_rows=B * T,
                    max_seq_len=inp["max_t"], rope_theta=w.rope_theta, rms_eps=w.rms_eps)
    lse = torch.empty(B, T, H, dtype=torch.float32, device="cuda")
    two = torch.from_numpy(wo.view(np.int16)).view(torch.bfloat16).cuda()
    res = dev["residual"].clone() if dev["residual"] is not None else None
    out, y = rt.prefill_mha(dev["q_latent"], w.prefill_start, dev["cache"], residual=res, lse=lse,
                            wo=two)
    torch.cuda.synchronize()
    assert rt.sync_status() == 0
    ref = _oracle_mha(inp, w, wo, tokens)
    sel = np.arange(T) if tokens is None else np.asarray(tokens)
    assert_close_bf16(f64(out)[:, sel], ref["out"], f"{w.name} mha out")
    np.testing.assert_allclose(lse.cpu().numpy()[:, sel], ref["lse"], atol=5e-2, rtol=0)
    assert_close_bf16(f64(y)[:, sel], ref["y"], f"{w.name} wo(out)")
    rt.close()


@pytest.mark.parametrize("B,T,sp,H", [(1, 5, 0, 16), (2, 70, 100, 64), (1, 200, 200, 128),
                                      (1, 130, 63, 128), (3, 33, 1, 16)])
def test_mha_prefill_small(B, T, sp, H):
    """Query tiles cut by the chunk end, key tiles cut by the causal diagonal, several
    sequences."""
    w = workload("prefill_chunk", dims=MLADims(H), batch=B, tokens=T, prefill_start=sp)
    _mha_case(w, seed=B * 100 + T + sp)


def test_mha_prefill_with_residual():
    w = workload("prefill_chunk", dims=MLADims(64), batch=2, tokens=40, prefill_start=30,
                 residual=True)
    _mha_case(w, seed=6)


def test_mha_prefill_chunk_full_size():
    """The 2048-token chunk after 2048 cached positions, H=128, wo to the 7168-wide model, on
    every 16th token (and the last) — the oracle rebuilds 128 heads' keys and values per token."""
    w = workload("prefill_chunk")
    toks = np.unique(np.concatenate([np.arange(0, 2048, 16), [2047]]))
    _mha_case(w, seed=7, dim=7168, tokens=toks)
