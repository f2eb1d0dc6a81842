"""The reference arm of bench.py (the fp64 oracle timed on the host cores) on CPU: one JSON line
with the keys the benchmark contract asks for, and silence on ranks other than 0."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CMD = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
       "--warmup", "3", "--ref-step-seconds", "0.5", "--workload", "tiny_decode"]


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    return subprocess.run(CMD, capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)


def test_reference_arm_prints_one_contract_line():
    r = _run({"RANK": "0", "WORLD_SIZE": "1"})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference"
    assert d["value"] > 0 and d["unit"] == "queries/s" and d["higher_is_better"] is True
    assert d["steps"] == 1 and d["warmup"] == 3
    assert d["config"]["workload"] == "tiny_decode"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"]
    assert cb["value"] == d["value"] and cb["unit"] == d["unit"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_is_silent_off_rank_zero():
    r = _run({"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_warmup_below_three_is_refused():
    r = subprocess.run(CMD[:6] + ["--warmup", "2"], capture_output=True, text=True, timeout=300,
                       cwd=ROOT)
    assert r.returncode != 0 and "--warmup must be >= 3" in r.stderr


def test_algorithmic_work_matches_the_hand_count():
    """The roofline's numerator: for the V3.2 decode batch (B=32, H=128, L=4096, each row sees
    its 4097 keys) the attention must move every cached key once (512 latent + 64 rotary bf16 =
    1152 B); the flops are 2 per multiply-add of the score (576 wide) and P·V (512 wide)
    products."""
    sys.path.insert(0, ROOT)
    import numpy as np
    import bench
    from mla_synth import make_inputs, workload
    w = workload("v32_decode")
    inp = make_inputs(w, seed=0)
    work = bench.algorithmic_work(w, inp["start_pos"])
    B, H, keys = 32, 128, 4097
    assert work["keys"] == B * keys == 131104
    assert work["cache_bytes"] == B * keys * 1152
    assert work["attn_bytes"] == B * keys * 1152 == 151031808   # cache rows attended only
    assert work["attn_flops"] == 2 * B * keys * H * (576 + 512)
    # whole step: weights (wq_b, wkv_b, fp32 gain), activations in/out, cache, output
    weights = H * 192 * 1536 * 2 + H * 256 * 512 * 2 + 1536 * 4
    assert work["weight_bytes"] == weights
    assert work["bytes"] == 2 * B * 1536 * 2 + weights + B * keys * 1152 + B * H * 128 * 2
    # a prefill chunk reads its sequence's cache prefix once, whatever the number of tokens
    wp = workload("prefill_chunk")
    inpp = make_inputs(wp, seed=0)
    wk = bench.algorithmic_work(wp, inpp["start_pos"])
    assert wk["cache_bytes"] == (2048 + 2048) * 1152
    t = np.arange(2048)
    assert wk["keys"] == int((2048 + t + 1).sum())


def test_recorded_traffic_follows_the_attention_source_only(tmp_path, monkeypatch):
    """The DRAM bytes of a committed ncu record are reported only while the attention kernel's
    source region (k_attn.cu before the combine kernel's section) is the one recorded: an edit to
    the combine kernel keeps the record, an edit to the attention kernel voids it."""
    sys.path.insert(0, ROOT)
    import bench
    src = os.path.join(ROOT, "head_latent_attention_11_b200", "csrc", "k_attn.cu")
    text = open(src, "rb").read()
    cut = text.find(bench.ATTN_SOURCE_END)
    assert cut > 0, "the combine section marker is missing from k_attn.cu"
    (tmp_path / "head_latent_attention_11_b200" / "csrc").mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    kattn = tmp_path / "head_latent_attention_11_b200" / "csrc" / "k_attn.cu"
    kattn.write_bytes(text)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    rec = {"source_sha256_prefix": bench.attention_source_sha256()[:16],
           "dram_bytes_read": 1000, "dram_bytes_write": 24}
    (tmp_path / "profiles" / "latent_attention_x.json").write_text(json.dumps(rec))
    assert bench.profiled_traffic("x") == 1024
    kattn.write_bytes(text + b"\n// a later change to the combine kernel\n")
    assert bench.profiled_traffic("x") == 1024
    kattn.write_bytes(text[:cut] + b"// a change to the attention kernel\n" + text[cut:])
    assert bench.profiled_traffic("x") is None
    assert bench.profiled_traffic("missing") is None
