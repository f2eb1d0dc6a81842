"""GPU parity of the index-mask decode (mla_decode_sparse) against the oracle's decode with the
same top-k (the "Attention update" mla-decode index mask), through the C ABI, on seeded inputs
and seeded key selections.  Bound: bf16 outputs |err| <= 1e-2 * max|ref| + 1e-3; lse within the
derived bound of the bf16-query oracle."""
import numpy as np
import pytest

from mla_cases import (LSE_ATOL, LSE_RTOL, assert_close_bf16, f64, make_inputs, oracle_parallel,
                       to_device, workload)
from mla_synth import MLADims, make_topk

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_11_b200 import build
    build.build()


def _sparse_case(w, k, seed=0, tail="nan"):
    from head_latent_attention_11_b200.runtime import MLARuntime
    inp = make_inputs(w, seed=seed, tail=tail)
    idx, lens = make_topk(inp["start_pos"], k, seed=seed)
    dev = to_device(inp)
    B, H = w.batch, w.dims.n_heads
    rt = MLARuntime(dev["gamma"], dev["wq_b"], dev["wkv_b"], n_heads=H, max_rows=B,
                    max_seq_len=inp["max_t"], rope_theta=w.rope_theta, rms_eps=w.rms_eps)
    lse = torch.empty(B, H, dtype=torch.float32, device="cuda")
    res = dev["residual"].reshape(B, -1).clone() if dev["residual"] is not None else None
    t_idx = torch.from_numpy(idx).cuda()
    t_len = torch.from_numpy(lens).cuda()
    out = rt.decode_sparse(dev["q_latent"].reshape(B, -1), dev["start_pos"], t_idx, t_len,
                           dev["cache"], residual=res, lse=lse)
    torch.cuda.synchronize()
    assert rt.sync_status() == 0
    ref = oracle_parallel("decode", inp, w, None, topk=idx)
    refq = oracle_parallel("decode", inp, w, None, topk=idx, query_precision="bf16")
    got = f64(out)
    assert_close_bf16(got, ref["out"], f"{w.name} sparse out")
    assert_close_bf16(got, refq["out"], f"{w.name} sparse out (bf16-query oracle)", rel=5e-3)
    np.testing.assert_allclose(lse.cpu().numpy(), refq["lse"], atol=LSE_ATOL, rtol=LSE_RTOL)
    rt.close()


def test_sparse_topk_covering_all_keys_tiny():
    """k >= end_pos: every key is selected (in shuffled order) — the dense result."""
    _sparse_case(workload("tiny_decode"), k=200)


@pytest.mark.parametrize("H,B,L,k", [(16, 3, 300, 1), (64, 5, 1000, 65), (128, 4, 700, 100),
                                     (128, 7, 3000, 257)])
def test_sparse_edges(H, B, L, k):
    """One selected key, tiles cut by the selection length, rows split between SM pairs."""
    w = workload("tiny_decode", dims=MLADims(H), batch=B, cache_len=L)
    _sparse_case(w, k=k, seed=H + B + L + k)


def test_sparse_v32_top2048():
    """V3.2-shaped decode (B=32, H=128, L=4096) with 2048 selected keys per sequence."""
    _sparse_case(workload("v32_decode"), k=2048, seed=1)


def test_sparse_ragged_top2048():
    """Ragged long-context decode (B=64, L_b ~ U{1024..32768}, residual) with 2048 selected
    keys per sequence, every row."""
    _sparse_case(workload("ragged_decode"), k=2048, seed=2)


def test_sparse_bad_length_is_reported():
    from head_latent_attention_11_b200 import STATUS
    from head_latent_attention_11_b200.runtime import MLARuntime
    w = workload("tiny_decode")
    inp = make_inputs(w, seed=3)
    idx, lens = make_topk(inp["start_pos"], 16, seed=3)
    dev = to_device(inp)
    rt = MLARuntime(dev["gamma"], dev["wq_b"], dev["wkv_b"], n_heads=16, max_rows=2,
                    max_seq_len=inp["max_t"])
    lens[1] = 0                      # no key selected: clamped to one, reported
    rt.decode_sparse(dev["q_latent"].reshape(2, -1), dev["start_pos"],
                     torch.from_numpy(idx).cuda(), torch.from_numpy(lens).cuda(), dev["cache"])
    assert STATUS[rt.sync_status()] == "MLA_ERR_DEVICE_ARG"
    rt.close()
