"""The C-ABI library builds, loads, and exports what include/*.h declares.

CPU-only: no compute call reaches a device. Host-side argument checks run
before any CUDA call, so their error codes are testable without a GPU.
"""
import ctypes
import glob
import json
import os
import re
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = sorted(glob.glob(os.path.join(ROOT, "include", "*.h")))
SPEC = {k: v["value"] for k, v in json.load(open(os.path.join(ROOT, "tests", "golden", "qwen3_0_6b_spec.json"))).items()
        if not k.startswith("_")}


@pytest.fixture(scope="module")
def lib():
    from decode_attention_qk_b200 import binding, build
    build.build_library()
    return binding.load_library()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names.update(re.findall(r"\b(qwen3_decode_attn_\w+)\s*\(", text))
    return sorted(names)


def test_headers_declare_the_entry_points():
    names = declared_functions()
    for required in ("qwen3_decode_attn_create", "qwen3_decode_attn_append_and_attend",
                     "qwen3_decode_attn_destroy", "qwen3_decode_attn_check"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    from decode_attention_qk_b200 import binding
    out = subprocess.run(["nm", "-D", "--defined-only", binding.LIBRARY_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s+(\w+)$", out, flags=re.M))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_compiled_constants_match_the_pages():
    text = open(os.path.join(ROOT, "include", "qwen3_decode_attn.h")).read()
    consts = {k: int(v) for k, v in re.findall(r"#define\s+(QDA_\w+)\s+(\d+)\s*$", text, flags=re.M)}
    assert consts["QDA_NUM_Q_HEADS"] == SPEC["num_attention_heads"]
    assert consts["QDA_NUM_KV_HEADS"] == SPEC["num_key_value_heads"]
    assert consts["QDA_HEAD_DIM"] == SPEC["head_dim"]
    assert consts["QDA_PAGE_SIZE"] == SPEC["page_size"]
    assert consts["QDA_MAX_BATCH"] == SPEC["max_batch"]
    assert consts["QDA_MAX_SEQ_LEN"] == SPEC["max_cached_positions"]
    assert consts["QDA_QKV_WIDTH"] == SPEC["qkv_proj_out"]


def test_default_config_is_qwen3_0_6b(lib):
    from decode_attention_qk_b200 import binding
    cfg = binding.qwen3_decode_attn_default_config()
    assert ctypes.sizeof(binding.qda_config) == 64
    assert (cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim, cfg.page_size) == (16, 8, 128, 16)
    assert cfg.max_batch == 256 and cfg.max_seq_len == 40960 and cfg.max_pages_per_seq == 2560
    assert cfg.rope_theta == SPEC["rope_theta"] and cfg.rms_eps == SPEC["rms_norm_eps"]
    assert cfg.grid_ctas == 0 and cfg.flags == 0 and cfg.wait_timeout_ns == 0


def test_strerror_covers_every_code(lib):
    from decode_attention_qk_b200 import binding
    for code in (0, -1, -2, -3, -4, -5):
        assert binding.qwen3_decode_attn_strerror(code) != binding.qwen3_decode_attn_strerror(99)


def test_create_rejects_bad_configs_on_the_host(lib):
    from decode_attention_qk_b200 import binding
    h = ctypes.c_void_p(1234)
    cases = [({"num_q_heads": 24}, binding.QDA_ERR_UNSUPPORTED),
             ({"num_q_heads": 128}, binding.QDA_ERR_UNSUPPORTED),
             ({"num_kv_heads": 4}, binding.QDA_ERR_UNSUPPORTED),
             ({"head_dim": 64}, binding.QDA_ERR_UNSUPPORTED),
             ({"page_size": 32}, binding.QDA_ERR_UNSUPPORTED),
             ({"max_batch": 0}, binding.QDA_ERR_INVALID_ARG),
             ({"max_batch": 257}, binding.QDA_ERR_INVALID_ARG),
             ({"max_seq_len": 40961}, binding.QDA_ERR_INVALID_ARG),
             ({"max_pages_per_seq": 100}, binding.QDA_ERR_INVALID_ARG),
             ({"rope_theta": 0.0}, binding.QDA_ERR_INVALID_ARG),
             ({"rms_eps": -1.0}, binding.QDA_ERR_INVALID_ARG),
             ({"grid_ctas": -1}, binding.QDA_ERR_INVALID_ARG),
             ({"grid_ctas": 5000}, binding.QDA_ERR_INVALID_ARG),
             ({"flags": 0x80}, binding.QDA_ERR_INVALID_ARG)]
    for over, code in cases:
        cfg = binding.qwen3_decode_attn_default_config(**over)
        assert lib.qwen3_decode_attn_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == code, over
        assert h.value is None
    cfg = binding.qwen3_decode_attn_default_config()
    assert lib.qwen3_decode_attn_create(ctypes.byref(cfg), -1, ctypes.byref(h)) == binding.QDA_ERR_INVALID_ARG
    assert lib.qwen3_decode_attn_create(None, 0, ctypes.byref(h)) == binding.QDA_ERR_INVALID_ARG


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device error path")
def test_create_without_a_device_reports_cuda_error(lib):
    from decode_attention_qk_b200 import binding
    cfg = binding.qwen3_decode_attn_default_config()
    h = ctypes.c_void_p()
    assert lib.qwen3_decode_attn_create(ctypes.byref(cfg), 0, ctypes.byref(h)) == binding.QDA_ERR_CUDA
    assert h.value is None


def test_calls_on_a_null_handle_are_rejected(lib):
    from decode_attention_qk_b200 import binding
    p = ctypes.c_void_p(4096)
    i32 = ctypes.cast(p, ctypes.POINTER(ctypes.c_int32))
    for fn in (lib.qwen3_decode_attn_append_and_attend, lib.qwen3_decode_attn_append_and_attend_host):
        assert fn(None, p, p, p, i32, None, i32, 1, p, p, 1, p, 1, None) == binding.QDA_ERR_INVALID_ARG
    assert lib.qwen3_decode_attn_append_and_attend_tokens(None, p, p, p, i32, None, i32, 1, p, p, 1, p, 1, 2,
                                                          None) == binding.QDA_ERR_INVALID_ARG
    assert lib.qwen3_decode_attn_qkv_proj(None, p, p, p, 1024, p, 1, None) == binding.QDA_ERR_INVALID_ARG
    assert lib.qwen3_decode_attn_o_proj(None, p, p, 1024, p, 1, None) == binding.QDA_ERR_INVALID_ARG
    assert lib.qwen3_decode_attn_check(None, None) == binding.QDA_ERR_INVALID_ARG
    assert lib.qwen3_decode_attn_grid_ctas(None) == 0
    lib.qwen3_decode_attn_destroy(None)


def test_binding_fails_loudly_without_the_library(monkeypatch, tmp_path):
    from decode_attention_qk_b200 import binding
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIBRARY_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        binding.load_library()


def test_product_path_does_not_import_the_oracle():
    """The CUDA library's Python side never imports oracle/ (test infrastructure)."""
    pkg = os.path.join(ROOT, "decode_attention_qk_b200")
    for path in glob.glob(os.path.join(pkg, "**", "*.py"), recursive=True) + \
            glob.glob(os.path.join(pkg, "csrc", "*")):
        text = open(path).read()
        assert not re.search(r"^\s*(import|from)\s+oracle\b", text, flags=re.M), path
        assert "qwen3_decode_oracle" not in text and "liboracle" not in text, path
