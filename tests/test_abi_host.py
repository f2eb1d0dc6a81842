"""Host-side checks of the C ABI that need no GPU: the library builds for sm_100a, loads, exports
every entry point include/mla.h declares, and rejects bad arguments before launching anything."""
import ctypes
import os
import re
import subprocess

import pytest

import head_latent_attention_11_b200 as mla
from head_latent_attention_11_b200 import build

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "mla.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return mla.load()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(mla_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_header_declares_the_binding_symbols():
    assert _declared_functions() == sorted(mla.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", mla.lib_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(\w+)", out))
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, f"not exported: {missing}"
    for n in _declared_functions():
        assert getattr(lib, n) is not None


def test_library_is_built_for_sm100a(lib):
    out = subprocess.run(["/usr/local/cuda/bin/cuobjdump", "--list-elf", mla.lib_path()],
                         capture_output=True, text=True)
    if out.returncode != 0:
        pytest.skip("cuobjdump unavailable")
    assert "sm_100a" in out.stdout


def test_status_strings(lib):
    for code, name in mla.STATUS.items():
        assert mla.mla_status_string(code) == name


def test_unsupported_config_rejected(lib):
    bad = mla.MLAConfig.make(n_heads=24, max_rows=4, max_seq_len=128)
    assert mla.mla_workspace_size(bad) == 0
    with pytest.raises(mla.MLAError) as e:
        mla.mla_init(bad, 16, 16, 16, 256, 1 << 30)
    assert mla.STATUS[e.value.status] == "MLA_ERR_UNSUPPORTED"
    bad_dims = mla.MLAConfig.make(n_heads=128, max_rows=4, max_seq_len=128, kv_lora_rank=256)
    assert mla.mla_workspace_size(bad_dims) == 0


def test_invalid_config_values_rejected(lib):
    for kw in (dict(max_rows=0), dict(max_seq_len=32)):
        cfg = mla.MLAConfig.make(n_heads=128, **{"max_rows": 4, "max_seq_len": 128, **kw})
        with pytest.raises(mla.MLAError) as e:
            mla.mla_init(cfg, 16, 16, 16, 256, 1 << 30)
        assert mla.STATUS[e.value.status] == "MLA_ERR_INVALID_ARG"


def test_workspace_size_scales_with_rows(lib):
    a = mla.mla_workspace_size(mla.MLAConfig.make(n_heads=128, max_rows=32, max_seq_len=4097))
    b = mla.mla_workspace_size(mla.MLAConfig.make(n_heads=128, max_rows=64, max_seq_len=4097))
    assert 0 < a < b
    # 32 rows of the absorbed query alone are 32*128*576*2 bytes
    assert b - a >= 32 * 128 * 576 * 2


def test_init_rejects_null_and_misaligned(lib):
    cfg = mla.MLAConfig.make(n_heads=16, max_rows=2, max_seq_len=129)
    with pytest.raises(mla.MLAError) as e:
        mla.mla_init(cfg, None, 16, 16, 256, 1 << 30)
    assert mla.STATUS[e.value.status] == "MLA_ERR_INVALID_ARG"
    with pytest.raises(mla.MLAError) as e:
        mla.mla_init(cfg, 16, 18, 16, 256, 1 << 30)
    assert mla.STATUS[e.value.status] == "MLA_ERR_INVALID_ARG"
    with pytest.raises(mla.MLAError) as e:
        mla.mla_init(cfg, 16, 16, 16, 256 + 16, 1 << 30)
    assert mla.STATUS[e.value.status] == "MLA_ERR_WORKSPACE"
    with pytest.raises(mla.MLAError) as e:
        mla.mla_init(cfg, 16, 16, 16, 256, 16)
    assert mla.STATUS[e.value.status] == "MLA_ERR_WORKSPACE"


def test_rmsnorm_rejects_bad_shapes(lib):
    for rows, dim in ((0, 1536), (4, 1000), (4, 8192)):
        with pytest.raises(mla.MLAError) as e:
            mla.mla_rmsnorm(16, None, 16, rows, dim, 1e-6, 32)
        assert mla.STATUS[e.value.status] == "MLA_ERR_INVALID_ARG"
    with pytest.raises(mla.MLAError):
        mla.mla_rmsnorm(16, None, 16, 4, 1536, 1e-6, 16)       # y aliases x
    with pytest.raises(mla.MLAError):
        mla.mla_rmsnorm(18, None, 16, 4, 1536, 1e-6, 32)       # misaligned


def test_calls_without_context_rejected(lib):
    with pytest.raises(mla.MLAError):
        mla.mla_decode(None, 16, None, 16, 16, 576 * 64, 576, 16 + 1024, 576 * 64, 576, 1, 16)
    with pytest.raises(mla.MLAError):
        mla.mla_prefill_chunk(None, 16, None, 0, 1, 16, 576 * 64, 576, 16, 576 * 64, 576, 1, 16)
    assert mla.mla_sync_status(None) == 1
    assert mla.mla_last_launch_count(None) == 0


def test_noalloc_rejects_bad_arguments_before_launching(lib):
    """The allocation-free entry point checks its arguments on the host like mla_decode: a missing
    status word, rows beyond its scratch array, unsupported heads, bad strides or sequence lengths
    return an error before any CUDA call."""
    ok = dict(q_abs=16, start_pos=16, rows=4, n_heads=128, softmax_scale=0.07, kv_cache=16,
              kv_stride_b=576 * 64, kv_stride_t=576, pe_cache=16 + 1024, pe_stride_b=576 * 64,
              pe_stride_t=576, max_seq_len=64, o_lat=16, lse=None, status=16)
    cases = [
        (dict(status=None), "MLA_ERR_INVALID_ARG"),
        (dict(rows=4097), "MLA_ERR_INVALID_ARG"),
        (dict(rows=0), "MLA_ERR_INVALID_ARG"),
        (dict(n_heads=24), "MLA_ERR_UNSUPPORTED"),
        (dict(max_seq_len=32), "MLA_ERR_INVALID_ARG"),
        (dict(max_seq_len=(1 << 24) + 1), "MLA_ERR_INVALID_ARG"),
        (dict(kv_stride_t=500), "MLA_ERR_INVALID_ARG"),
        (dict(kv_stride_b=(1 << 40)), "MLA_ERR_INVALID_ARG"),
        (dict(pe_cache=18), "MLA_ERR_INVALID_ARG"),
        (dict(softmax_scale=float("nan")), "MLA_ERR_INVALID_ARG"),
    ]
    for change, want in cases:
        args = {**ok, **change}
        with pytest.raises(mla.MLAError) as e:
            mla.mla_latent_attention_noalloc(**args)
        assert mla.STATUS[e.value.status] == want, change
