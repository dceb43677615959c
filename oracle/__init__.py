"""Float64 CPU oracle of the Qwen3-0.6B decode-attention step (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg use this package; the CUDA library and its Python binding never
import it. The arithmetic lives in ``qwen3_decode_oracle.c`` (plain C, double
precision, written from the Qwen3-0.6B Model Spec's "Compute-graph nodes"
table); this module only marshals numpy arrays into it. bf16 tensors travel as
``numpy.uint16`` arrays of their bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "qwen3_decode_oracle.c")
LIBRARY = os.path.join(_HERE, "liboracle.so")

NUM_Q_HEADS = 16
NUM_KV_HEADS = 8
HEAD_DIM = 128
PAGE = 16
QKV_WIDTH = 4096

_ERRORS = {-1: "invalid argument", -4: "seq_len or block-table entry out of range"}


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (IEEE double, no contraction into FMA)."""
    if force or not os.path.exists(LIBRARY) or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE):
        cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
               "-shared", "-fPIC", "-o", LIBRARY, SOURCE, "-lm"]
        subprocess.run(cmd, check=True)
    return LIBRARY


_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIBRARY)
        dp = ctypes.POINTER(ctypes.c_double)
        u16p = ctypes.POINTER(ctypes.c_uint16)
        i32p = ctypes.POINTER(ctypes.c_int32)
        lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.oracle_bf16_to_f64.restype = ctypes.c_double
        lib.oracle_f64_to_bf16_rne.argtypes = [ctypes.c_double]
        lib.oracle_f64_to_bf16_rne.restype = ctypes.c_uint16
        lib.oracle_bf16_to_f64_array.argtypes = [u16p, dp, ctypes.c_size_t]
        lib.oracle_f64_to_bf16_rne_array.argtypes = [dp, u16p, ctypes.c_size_t]
        lib.oracle_rmsnorm.argtypes = [dp, dp, ctypes.c_int, ctypes.c_double, dp]
        lib.oracle_rope.argtypes = [dp, ctypes.c_int, ctypes.c_double, ctypes.c_double]
        lib.oracle_decode_head.argtypes = [dp, ctypes.c_int, i32p, u16p, u16p, ctypes.c_int, dp, dp]
        lib.oracle_append_and_attend.argtypes = [
            u16p, u16p, u16p, i32p, i32p, i32p, ctypes.c_int, u16p, u16p, ctypes.c_int,
            dp, ctypes.c_int, ctypes.c_double, ctypes.c_double, dp, dp]
        lib.oracle_append_and_attend.restype = ctypes.c_int
        lib.oracle_append_and_attend_gqa.argtypes = [
            u16p, u16p, u16p, i32p, i32p, i32p, ctypes.c_int, u16p, u16p, ctypes.c_int,
            dp, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double, dp, dp]
        lib.oracle_append_and_attend_gqa.restype = ctypes.c_int
        lib.oracle_input_norm_qkv_proj.argtypes = [u16p, u16p, u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_double, dp, u16p]
        lib.oracle_input_norm_qkv_proj.restype = ctypes.c_int
        lib.oracle_o_proj.argtypes = [u16p, u16p, ctypes.c_int, ctypes.c_int, ctypes.c_int, dp, u16p]
        lib.oracle_o_proj.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        lib.oracle_set_threads.restype = None
        lib.oracle_get_threads.argtypes = []
        lib.oracle_get_threads.restype = ctypes.c_int
        lib.oracle_append_and_attend_tokens.argtypes = [
            u16p, u16p, u16p, i32p, i32p, i32p, ctypes.c_int, u16p, u16p, ctypes.c_int,
            dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_double, dp, dp]
        lib.oracle_append_and_attend_tokens.restype = ctypes.c_int
        _lib = lib
    return _lib


def input_norm_qkv_proj(x, norm_w, w, rms_eps: float = 1e-6) -> dict:
    """input_norm then attn.qkv_proj (Model Spec, "Compute-graph nodes"): x bf16 bits
    [B, K], norm_w [K], w [N, K] (row n = output n). Returns ``y`` float64 [B, N]
    (exact) and ``bits`` uint16 [B, N] (y rounded once to bf16, nearest-even)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    norm_w = np.ascontiguousarray(norm_w, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.uint16)
    assert x.ndim == 2 and w.ndim == 2 and w.shape[1] == x.shape[1] and norm_w.shape == (x.shape[1],)
    B, K = x.shape
    N = w.shape[0]
    y = np.empty((B, N), dtype=np.float64)
    bits = np.empty((B, N), dtype=np.uint16)
    rc = _load().oracle_input_norm_qkv_proj(_ptr(x, ctypes.c_uint16), _ptr(norm_w, ctypes.c_uint16),
                                            _ptr(w, ctypes.c_uint16), B, K, N, rms_eps,
                                            _ptr(y, ctypes.c_double), _ptr(bits, ctypes.c_uint16))
    if rc != 0:
        raise ValueError(f"oracle_input_norm_qkv_proj: {_ERRORS.get(rc, rc)}")
    return {"y": y, "bits": bits}


def o_proj(x, w) -> dict:
    """attn.o_proj (Model Spec, "Compute-graph nodes": linear, K = 2048, N = 1024
    for Qwen3-0.6B): x bf16 bits [B, K] (the attention output o [B, Hq, 128] as
    rows of Hq * 128), w [N, K] (row n = output n). Returns ``y`` float64 [B, N]
    (exact) and ``bits`` uint16 [B, N] (y rounded once to bf16, nearest-even)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.uint16)
    x = x.reshape(x.shape[0], -1)
    assert w.ndim == 2 and w.shape[1] == x.shape[1]
    B, K = x.shape
    N = w.shape[0]
    y = np.empty((B, N), dtype=np.float64)
    bits = np.empty((B, N), dtype=np.uint16)
    rc = _load().oracle_o_proj(_ptr(x, ctypes.c_uint16), _ptr(w, ctypes.c_uint16), B, K, N,
                               _ptr(y, ctypes.c_double), _ptr(bits, ctypes.c_uint16))
    if rc != 0:
        raise ValueError(f"oracle_o_proj: {_ERRORS.get(rc, rc)}")
    return {"y": y, "bits": bits}


def set_threads(n: int) -> None:
    """Threads the step's attention loop uses (default 1); results do not depend on it."""
    _load().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_load().oracle_get_threads())


def _ptr(a: np.ndarray | None, ctype):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.POINTER(ctype))


def bf16_to_f64(bits) -> np.ndarray:
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    out = np.empty(bits.shape, dtype=np.float64)
    _load().oracle_bf16_to_f64_array(_ptr(bits, ctypes.c_uint16), _ptr(out, ctypes.c_double), bits.size)
    return out


def f64_to_bf16_rne(x) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    _load().oracle_f64_to_bf16_rne_array(_ptr(x, ctypes.c_double), _ptr(out, ctypes.c_uint16), x.size)
    return out


def rmsnorm(x, w, eps: float = 1e-6) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float64)
    w = np.ascontiguousarray(w, dtype=np.float64)
    assert x.ndim == 1 and w.shape == x.shape
    y = np.empty_like(x)
    _load().oracle_rmsnorm(_ptr(x, ctypes.c_double), _ptr(w, ctypes.c_double), x.size, eps,
                           _ptr(y, ctypes.c_double))
    return y


def rope(x, pos: float, theta: float = 1e6) -> np.ndarray:
    y = np.array(x, dtype=np.float64, copy=True)
    assert y.ndim == 1 and y.size % 2 == 0
    _load().oracle_rope(_ptr(y, ctypes.c_double), y.size, float(pos), float(theta))
    return y


def decode_head(q, seq_len: int, bt_row, k_cache, v_cache, kv_head: int) -> np.ndarray:
    """One query head of decodeGQA over the paged cache (bf16 bit arrays)."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    bt_row = np.ascontiguousarray(bt_row, dtype=np.int32)
    k_cache = np.ascontiguousarray(k_cache, dtype=np.uint16)
    v_cache = np.ascontiguousarray(v_cache, dtype=np.uint16)
    scores = np.empty(seq_len, dtype=np.float64)
    o = np.empty(HEAD_DIM, dtype=np.float64)
    _load().oracle_decode_head(_ptr(q, ctypes.c_double), seq_len, _ptr(bt_row, ctypes.c_int32),
                               _ptr(k_cache, ctypes.c_uint16), _ptr(v_cache, ctypes.c_uint16),
                               kv_head, _ptr(scores, ctypes.c_double), _ptr(o, ctypes.c_double))
    return o


def append_and_attend(qkv, q_norm_w, k_norm_w, seq_lens, block_table, k_cache, v_cache,
                      positions=None, rope_theta: float = 1e6, rms_eps: float = 1e-6,
                      inplace: bool = False, want_qk: bool = False) -> dict:
    """Run the whole step with one new token per sequence. bf16 inputs are
    uint16 bit arrays.

    The number of query heads follows from the qkv row width,
    (num_q_heads + 16) * 128: 16 for Qwen3-0.6B, 32, 40 or 64 for larger sizes.
    Returns a dict with ``o`` (float64 [B,Hq,128]), ``k_cache`` and ``v_cache``
    (uint16, after the append; the inputs themselves when ``inplace``), and,
    when ``want_qk``, ``q`` (float64 [B,Hq,128]) and ``k`` (float64 [B,8,128],
    the new k before its rounding to bf16).
    """
    qkv = np.ascontiguousarray(qkv, dtype=np.uint16)
    out = append_and_attend_tokens(qkv[:, None, :], q_norm_w, k_norm_w, seq_lens, block_table, k_cache,
                                   v_cache, positions=positions, rope_theta=rope_theta, rms_eps=rms_eps,
                                   inplace=inplace, want_qk=want_qk)
    out["o"] = out["o"][:, 0]
    if want_qk:
        out["q"], out["k"] = out["q"][:, 0], out["k"][:, 0]
    return out


def append_and_attend_tokens(qkv, q_norm_w, k_norm_w, seq_lens, block_table, k_cache, v_cache,
                             positions=None, rope_theta: float = 1e6, rms_eps: float = 1e-6,
                             inplace: bool = False, want_qk: bool = False) -> dict:
    """The step with T new tokens per sequence: qkv is [B, T, (Hq + 16) * 128];
    token t goes to slot L - T + t and attends causally over slots <= L - T + t.
    ``positions`` (if given) are the first new token's RoPE positions.
    Returns ``o`` float64 [B, T, Hq, 128], the caches, and with ``want_qk``
    ``q`` [B, T, Hq, 128] and ``k`` [B, T, 8, 128]."""
    qkv = np.ascontiguousarray(qkv, dtype=np.uint16)
    assert qkv.ndim == 3 and qkv.shape[2] % HEAD_DIM == 0
    B, T = qkv.shape[0], qkv.shape[1]
    Hq = qkv.shape[2] // HEAD_DIM - 2 * NUM_KV_HEADS
    q_norm_w = np.ascontiguousarray(q_norm_w, dtype=np.uint16)
    k_norm_w = np.ascontiguousarray(k_norm_w, dtype=np.uint16)
    seq_lens = np.ascontiguousarray(seq_lens, dtype=np.int32)
    block_table = np.ascontiguousarray(block_table, dtype=np.int32)
    assert block_table.ndim == 2 and block_table.shape[0] == B
    if positions is not None:
        positions = np.ascontiguousarray(positions, dtype=np.int32)
    if not inplace:
        k_cache = np.array(k_cache, dtype=np.uint16, copy=True)
        v_cache = np.array(v_cache, dtype=np.uint16, copy=True)
    assert k_cache.dtype == np.uint16 and k_cache.flags["C_CONTIGUOUS"]
    assert v_cache.dtype == np.uint16 and v_cache.flags["C_CONTIGUOUS"]
    num_pages = k_cache.shape[0]
    assert k_cache.shape == (num_pages, PAGE, NUM_KV_HEADS, HEAD_DIM) == v_cache.shape
    o = np.empty((B, T, Hq, HEAD_DIM), dtype=np.float64)
    q = np.empty((B, T, Hq, HEAD_DIM), dtype=np.float64) if want_qk else None
    k = np.empty((B, T, NUM_KV_HEADS, HEAD_DIM), dtype=np.float64) if want_qk else None
    rc = _load().oracle_append_and_attend_tokens(
        _ptr(qkv, ctypes.c_uint16), _ptr(q_norm_w, ctypes.c_uint16), _ptr(k_norm_w, ctypes.c_uint16),
        _ptr(seq_lens, ctypes.c_int32), _ptr(positions, ctypes.c_int32),
        _ptr(block_table, ctypes.c_int32), block_table.shape[1],
        _ptr(k_cache, ctypes.c_uint16), _ptr(v_cache, ctypes.c_uint16), num_pages,
        _ptr(o, ctypes.c_double), B, T, Hq, rope_theta, rms_eps,
        _ptr(q, ctypes.c_double), _ptr(k, ctypes.c_double))
    if rc != 0:
        raise ValueError(f"oracle_append_and_attend: {_ERRORS.get(rc, rc)}")
    out = {"o": o, "k_cache": k_cache, "v_cache": v_cache}
    if want_qk:
        out["q"], out["k"] = q, k
    return out
