"""The failure path of the bounded waits, made to happen without faulting anything: with the GEMM
kernels' wait bound set to 1 ns, their first wait that is not already satisfied gives up; the call
must report MLA_ERR_DEVICE_TIMEOUT through mla_sync_status, and the next call with the normal bound
must match the oracle (the kernels drained their copies and MMAs and released their tensor
memory, so the device stays usable)."""
import pytest

from mla_cases import assert_close_bf16, f64, make_inputs, oracle_decode, to_device, workload

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_11_b200 import build
    build.build()


def test_gemm_wait_timeout_is_reported_and_the_next_call_is_correct():
    from head_latent_attention_11_b200 import STATUS, mla_set_wait_limit
    from head_latent_attention_11_b200.runtime import MLARuntime
    w = workload("tiny_decode")
    inp = make_inputs(w, seed=41)
    dev = to_device(inp)
    rt = MLARuntime(dev["gamma"], dev["wq_b"], dev["wkv_b"], n_heads=16, max_rows=2,
                    max_seq_len=inp["max_t"])
    q = dev["q_latent"].reshape(2, -1)
    mla_set_wait_limit(rt.ctx, 1)
    for _ in range(3):
        rt.decode(q, dev["start_pos"], dev["cache"])
        torch.cuda.synchronize()
        assert STATUS[rt.sync_status()] == "MLA_ERR_DEVICE_TIMEOUT"
    mla_set_wait_limit(rt.ctx, 0)
    out = rt.decode(q, dev["start_pos"], dev["cache"])
    torch.cuda.synchronize()
    assert rt.sync_status() == 0
    assert_close_bf16(f64(out), oracle_decode(inp, w)["out"], "decode after the timeouts")
    rt.close()
