"""The allocation-free attention entry point matches the oracle on the queries it is given.

Callers that cannot allocate device memory where they run (code confined to a fixed pool, a
plug-in given a device budget by its host) use mla_latent_attention_noalloc.  This file is named so pytest collects it last; it runs the same
whether started alone in a fresh process or after the other tests.
"""
import numpy as np
import pytest

from mla_cases import LSE_ATOL, LSE_RTOL, assert_close_bf16, f64, make_inputs, to_device, workload

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_11_b200 import build
    build.build()


@pytest.mark.parametrize("H,B,L", [(128, 32, 4096), (64, 5, 300)])
def test_noalloc_attention_matches_oracle(H, B, L):
    """Absorbed queries come from the context path (they are an input of this entry point); its
    o_lat and lse are compared with the fp64 oracle's scores, softmax and weighted sum on the same
    queries, element by element, on two calls in a row that share the scratch array."""
    from head_latent_attention_11_b200 import mla_debug_copy, mla_latent_attention_noalloc
    from head_latent_attention_11_b200.runtime import MLARuntime
    from mla_synth import MLADims
    w = workload("v32_decode", dims=MLADims(H), batch=B, cache_len=L)
    inp = make_inputs(w, seed=7 + H + B, tail="nan")
    dev = to_device(inp)
    max_t = inp["max_t"]
    stream = torch.cuda.current_stream().cuda_stream
    rt = MLARuntime(dev["gamma"], dev["wq_b"], dev["wkv_b"], n_heads=H, max_rows=B,
                    max_seq_len=max_t)
    rt.decode(dev["q_latent"].reshape(B, -1), dev["start_pos"], dev["cache"])
    q_abs = torch.empty(B, 128, 576, dtype=torch.bfloat16, device="cuda")
    mla_debug_copy(rt.ctx, 2, q_abs, q_abs.numel() * 2, stream)
    torch.cuda.synchronize()
    assert rt.sync_status() == 0
    # the oracle's scores, softmax and weighted sum (a5-a7) on exactly these absorbed queries
    import oracle
    from mla_synth import bf16_bits_to_f64
    qa = f64(q_abs)
    ref_olat = np.empty((B, H, 512))
    ref_lse = np.empty((B, H))
    for b in range(B):
        n = int(inp["start_pos"][b]) + 1
        rows = bf16_bits_to_f64(inp["cache"][b, :n])
        s = oracle.latent_scores(qa[b, :H, :512], qa[b, :H, 512:], rows[:, :512], rows[:, 512:],
                                 192 ** -0.5)
        p, ref_lse[b] = oracle.softmax_fp(s)
        ref_olat[b] = oracle.latent_weighted_sum(p, rows[:, :512])
    kv, ksb, kst, pe, psb, pst = rt.cache_views(dev["cache"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):   # two calls in a row share the scratch array
        o_lat = torch.full((B, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
        mla_latent_attention_noalloc(q_abs, dev["start_pos"], B, H, 192 ** -0.5, kv, ksb, kst, pe,
                                     psb, pst, max_t, o_lat, lse, status, stream)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_close_bf16(f64(o_lat), ref_olat, f"o_lat call {call}")
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, atol=LSE_ATOL, rtol=LSE_RTOL)
    rt.close()


def test_noalloc_rejects_rows_beyond_scratch():
    from head_latent_attention_11_b200 import MLAError, STATUS, mla_latent_attention_noalloc
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(MLAError) as e:
        mla_latent_attention_noalloc(16, 16, 4097, 128, 0.07, 16, 576 * 64, 576, 16, 576 * 64, 576,
                                     64, 16, None, status)
    assert STATUS[e.value.status] == "MLA_ERR_INVALID_ARG"
