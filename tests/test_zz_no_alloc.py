"""The allocation-free attention entry point gives the same result as the context path.

Callers that cannot allocate device memory (a fixed pool, a host-imposed budget) use
mla_latent_attention_noalloc.  This file is named so pytest collects it last; it runs the same
whether started alone in a fresh process or after the other tests.
"""
import numpy as np
import pytest

from mla_cases import assert_close_bf16, f64, make_inputs, to_device, workload

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_11_b200 import build
    build.build()


@pytest.mark.parametrize("H,B,L", [(128, 32, 4096), (64, 5, 300)])
def test_noalloc_attention_matches_context_path(H, B, L):
    from head_latent_attention_11_b200 import mla_debug_copy, mla_latent_attention_noalloc
    from head_latent_attention_11_b200.runtime import MLARuntime
    from mla_synth import MLADims
    w = workload("v32_decode", dims=MLADims(H), batch=B, cache_len=L)
    inp = make_inputs(w, seed=7 + H + B, tail="nan")
    dev = to_device(inp)
    max_t = inp["max_t"]
    stream = torch.cuda.current_stream().cuda_stream
    # reference: the existing decode entry point, with its absorbed queries and o_lat
    rt = MLARuntime(dev["gamma"], dev["wq_b"], dev["wkv_b"], n_heads=H, max_rows=B,
                    max_seq_len=max_t)
    lse_ref = torch.empty(B, H, dtype=torch.float32, device="cuda")
    rt.decode(dev["q_latent"].reshape(B, -1), dev["start_pos"], dev["cache"], lse=lse_ref)
    q_abs = torch.empty(B, 128, 576, dtype=torch.bfloat16, device="cuda")
    o_ref = torch.empty(B, H, 512, dtype=torch.bfloat16, device="cuda")
    mla_debug_copy(rt.ctx, 2, q_abs, q_abs.numel() * 2, stream)
    mla_debug_copy(rt.ctx, 3, o_ref, o_ref.numel() * 2, stream)
    torch.cuda.synchronize()
    assert rt.sync_status() == 0
    kv, ksb, kst, pe, psb, pst = rt.cache_views(dev["cache"])
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):   # two calls in a row share the scratch array
        o_lat = torch.full((B, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
        mla_latent_attention_noalloc(q_abs, dev["start_pos"], B, H, 192 ** -0.5, kv, ksb, kst, pe,
                                     psb, pst, max_t, o_lat, lse, status, stream)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert_close_bf16(f64(o_lat), f64(o_ref), f"o_lat call {call}")
        np.testing.assert_allclose(lse.cpu().numpy(), lse_ref.cpu().numpy(), atol=2e-3, rtol=1e-4)
    rt.close()


def test_noalloc_rejects_rows_beyond_scratch():
    from head_latent_attention_11_b200 import MLAError, STATUS, mla_latent_attention_noalloc
    with pytest.raises(MLAError) as e:
        mla_latent_attention_noalloc(16, 16, 4097, 128, 0.07, 16, 576 * 64, 576, 16, 576 * 64, 576,
                                     64, 16)
    assert STATUS[e.value.status] == "MLA_ERR_INVALID_ARG"
