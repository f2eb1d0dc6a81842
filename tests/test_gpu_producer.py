"""GPU parity of the cache producer (mla_produce) and of produce → decode / prefill end to end,
through the C ABI, against the oracle's produce_latents / write_cache_rows / decode / prefill on
the same seeded bf16 inputs.  Bound: bf16 outputs |err| <= 1e-2 * max|ref| + 1e-3."""
import numpy as np
import pytest

import oracle
from mla_cases import assert_close_bf16, f64, make_inputs, oracle_parallel, to_device, workload
from mla_synth import MLADims, bf16_bits_to_f64, make_producer_inputs

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from head_latent_attention_11_b200 import build
    build.build()


class _PatchedCache:
    """The bf16 cache widened lazily, with some rows replaced by float64 values (the rows the
    oracle's producer wrote)."""

    def __init__(self, bits, rows):
        self.bits, self.rows = bits, rows     # rows: {(b, t): float64 [576]}

    def __getitem__(self, idx):
        b, ts, cols = idx
        out = bf16_bits_to_f64(self.bits[b, ts])
        start = ts.start or 0
        for (bb, t), v in self.rows.items():
            if bb == b and start <= t < start + out.shape[0]:
                out[t - start] = v
        return out[:, cols]


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def _produce(w, seed, dim=7168):
    from head_latent_attention_11_b200.runtime import MLARuntime
    inp = make_inputs(w, seed=seed, tail="nan")
    pin = make_producer_inputs(w, seed=seed, dim=dim)
    dev = to_device(inp)
    B, T = w.batch, w.tokens
    rt = MLARuntime(dev["gamma"], dev["wq_b"], dev["wkv_b"], n_heads=w.dims.n_heads,
                    max_rows=B * T, max_seq_len=inp["max_t"], rope_theta=w.rope_theta,
                    rms_eps=w.rms_eps)
    wq_a, wkv_a = _bf16(pin["wq_a"]), _bf16(pin["wkv_a"])
    gain = torch.from_numpy(pin["kv_gain"]).cuda()
    rt.attach_producer(wq_a, wkv_a, gain)
    cache = dev["cache"].clone()
    x = _bf16(pin["x"])
    if w.mode == "decode":
        q_lat = rt.produce(x, cache, start_pos=dev["start_pos"])
        pos = np.asarray(inp["start_pos"], np.int64)[:, None] + np.arange(T)[None, :]
    else:
        q_lat = rt.produce(x, cache, start_pos_host=w.prefill_start)
        pos = np.full((B, 1), w.prefill_start, np.int64) + np.arange(T)[None, :]
    torch.cuda.synchronize()
    assert rt.sync_status() == 0
    # oracle producer on the same bf16 inputs
    xr = bf16_bits_to_f64(pin["x"]).reshape(B * T, dim)
    q_ref, kv_ref, pe_ref = oracle.produce_latents(
        xr, bf16_bits_to_f64(pin["wq_a"]), bf16_bits_to_f64(pin["wkv_a"]),
        pin["kv_gain"].astype(np.float64), pos.reshape(-1), theta=w.rope_theta, eps=w.rms_eps)
    assert_close_bf16(f64(q_lat).reshape(B * T, -1), q_ref, "q_latent")
    got = cache.cpu().view(torch.int16).numpy().view(np.uint16)
    b_idx = np.repeat(np.arange(B), T)
    rows = got[b_idx, pos.reshape(-1)]
    assert_close_bf16(bf16_bits_to_f64(rows[:, :512]), kv_ref, "kv rows")
    assert_close_bf16(bf16_bits_to_f64(rows[:, 512:]), pe_ref, "pe rows")
    # every other cache row is untouched, bit for bit
    mask = np.ones(got.shape[:2], bool)
    mask[b_idx, pos.reshape(-1)] = False
    assert np.array_equal(got[mask], inp["cache"][mask])
    patched = {(int(b), int(t)): np.r_[kv_ref[i], pe_ref[i]]
               for i, (b, t) in enumerate(zip(b_idx, pos.reshape(-1)))}
    return rt, inp, dev, cache, q_lat, q_ref, _PatchedCache(inp["cache"], patched)


@pytest.mark.parametrize("name,kw", [
    ("tiny_decode", {}),
    ("v32_decode", {}),
    ("tiny_decode", dict(dims=MLADims(64), batch=5, cache_len=300)),
])
def test_produce_then_decode(name, kw):
    """The producer writes row start_pos of every sequence, then the decode attends over it: the
    whole chain equals the oracle's produce → write → decode."""
    w = workload(name, **kw)
    rt, inp, dev, cache, q_lat, q_ref, cache_ref = _produce(w, seed=21)
    B = w.batch
    out = rt.decode(q_lat.reshape(B, -1), dev["start_pos"], cache)
    torch.cuda.synchronize()
    assert rt.sync_status() == 0
    d = w.dims
    ref = oracle.decode(q_ref, inp["gamma"].astype(np.float64), bf16_bits_to_f64(inp["wq_b"]),
                        bf16_bits_to_f64(inp["wkv_b"]), cache_ref, inp["start_pos"], d.n_heads,
                        theta=w.rope_theta, eps=w.rms_eps)
    assert_close_bf16(f64(out), ref["out"], f"{w.name} produce->decode out")
    rt.close()


def test_produce_then_prefill_chunk():
    """A chunk of 70 new tokens per sequence after 100 cached ones: producer rows 100..169, then
    the causal chunk attention over them."""
    w = workload("prefill_chunk", dims=MLADims(64), batch=2, tokens=70, prefill_start=100)
    rt, inp, dev, cache, q_lat, q_ref, cache_ref = _produce(w, seed=22)
    out = rt.prefill(q_lat, w.prefill_start, cache)
    torch.cuda.synchronize()
    assert rt.sync_status() == 0
    d = w.dims
    ref = oracle.prefill(q_ref.reshape(w.batch, w.tokens, -1), inp["gamma"].astype(np.float64),
                         bf16_bits_to_f64(inp["wq_b"]), bf16_bits_to_f64(inp["wkv_b"]), cache_ref,
                         w.prefill_start, d.n_heads, theta=w.rope_theta, eps=w.rms_eps)
    assert_close_bf16(f64(out), ref["out"], "produce->prefill out")
    rt.close()


def test_produce_prefill_chunk_full_size():
    """The producer for the 2048-token chunk (B=1, after 2048 cached rows): every written row and
    every query latent against the oracle."""
    rt, *_ = _produce(workload("prefill_chunk"), seed=23)
    rt.close()


def test_produce_bad_position_writes_nothing():
    from head_latent_attention_11_b200 import STATUS
    w = workload("tiny_decode")
    inp = make_inputs(w, seed=24)
    pin = make_producer_inputs(w, seed=24, dim=512)
    dev = to_device(inp)
    from head_latent_attention_11_b200.runtime import MLARuntime
    rt = MLARuntime(dev["gamma"], dev["wq_b"], dev["wkv_b"], n_heads=16, max_rows=2,
                    max_seq_len=inp["max_t"])
    rt.attach_producer(_bf16(pin["wq_a"]), _bf16(pin["wkv_a"]),
                       torch.from_numpy(pin["kv_gain"]).cuda())
    cache = dev["cache"].clone()
    sp = dev["start_pos"].clone()
    sp[1] = inp["max_t"] + 3
    rt.produce(_bf16(pin["x"]), cache, start_pos=sp)
    assert STATUS[rt.sync_status()] == "MLA_ERR_DEVICE_ARG"
    got = cache.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got[1], inp["cache"][1]), "nothing written for the bad row"
    assert not np.array_equal(got[0], inp["cache"][0])
    rt.close()
