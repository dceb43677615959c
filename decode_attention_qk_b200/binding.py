"""Python binding of the decode-attention C ABI (include/qwen3_decode_attn.h).

Argument marshalling only: every step of the computation runs in the CUDA
library. The functions carry the C names; tensors are torch tensors whose
device pointers are passed through, and the stream is torch's current stream
unless one is given. Loading fails loudly when the library has not been built;
there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

LIBRARY_PATH = _build.LIBRARY

QDA_OK = 0
QDA_ERR_INVALID_ARG = -1
QDA_ERR_CUDA = -2
QDA_ERR_UNSUPPORTED = -3
QDA_ERR_BOUNDS = -4
QDA_ERR_TIMEOUT = -5
QDA_FLAG_INJECT_WAIT_TIMEOUT = 0x1

NUM_Q_HEADS, NUM_KV_HEADS, HEAD_DIM, PAGE_SIZE, QKV_WIDTH = 16, 8, 128, 16, 4096
SUPPORTED_Q_HEADS = (16, 32, 40, 64)   # Qwen3 0.6B/1.7B, 4B/8B, 14B, 32B
MAX_NEW_TOKENS = 40960
# (query heads, new tokens) pairs with a kernel for more than one new token
# (query heads, new tokens) pairs that one launch of the multi-token step
# takes: T >= 2 with at most 16 query rows (T * Hq / 8) per kv head; longer
# blocks run as several launches
SUPPORTED_MULTI_TOKEN = tuple((hq, t) for hq in (16, 32, 40, 64) for t in range(2, 9) if t * hq // 8 <= 16)


class qda_config(ctypes.Structure):
    _fields_ = [
        ("num_q_heads", ctypes.c_int),
        ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("page_size", ctypes.c_int),
        ("max_batch", ctypes.c_int),
        ("max_seq_len", ctypes.c_int),
        ("max_pages_per_seq", ctypes.c_int),
        ("rope_theta", ctypes.c_double),
        ("rms_eps", ctypes.c_double),
        ("grid_ctas", ctypes.c_int),
        ("flags", ctypes.c_uint),
        ("wait_timeout_ns", ctypes.c_int64),
    ]


class QdaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {qwen3_decode_attn_strerror(code)} (code {code})")


_lib = None


def load_library():
    """Load libqwen3_decode_attn.so (built by decode_attention_qk_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIBRARY_PATH):
            raise RuntimeError(
                f"CUDA library {LIBRARY_PATH} is missing; build it with "
                "`python -m decode_attention_qk_b200.build` (there is no CPU fallback)")
        lib = ctypes.CDLL(LIBRARY_PATH)
        vp, i32p = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)
        lib.qwen3_decode_attn_default_config.argtypes = [ctypes.POINTER(qda_config)]
        lib.qwen3_decode_attn_default_config.restype = None
        lib.qwen3_decode_attn_create.argtypes = [ctypes.POINTER(qda_config), ctypes.c_int, ctypes.POINTER(vp)]
        lib.qwen3_decode_attn_create.restype = ctypes.c_int
        call = [vp, vp, vp, vp, i32p, i32p, i32p, ctypes.c_int, vp, vp, ctypes.c_int, vp, ctypes.c_int, vp]
        lib.qwen3_decode_attn_append_and_attend.argtypes = call
        lib.qwen3_decode_attn_append_and_attend.restype = ctypes.c_int
        lib.qwen3_decode_attn_append_and_attend_host.argtypes = call
        lib.qwen3_decode_attn_append_and_attend_host.restype = ctypes.c_int
        lib.qwen3_decode_attn_append_and_attend_tokens.argtypes = call[:-1] + [ctypes.c_int, vp]
        lib.qwen3_decode_attn_append_and_attend_tokens.restype = ctypes.c_int
        lib.qwen3_decode_attn_qkv_proj.argtypes = [vp, vp, vp, vp, ctypes.c_int, vp, ctypes.c_int, vp]
        lib.qwen3_decode_attn_qkv_proj.restype = ctypes.c_int
        lib.qwen3_decode_attn_o_proj.argtypes = [vp, vp, vp, ctypes.c_int, vp, ctypes.c_int, vp]
        lib.qwen3_decode_attn_o_proj.restype = ctypes.c_int
        lib.qwen3_decode_attn_from_hidden.argtypes = [vp, vp, vp, vp, ctypes.c_int, vp, vp, vp, i32p, i32p, i32p,
                                                      ctypes.c_int, vp, vp, ctypes.c_int, vp, ctypes.c_int, vp]
        lib.qwen3_decode_attn_from_hidden.restype = ctypes.c_int
        lib.qwen3_decode_attn_check.argtypes = [vp, vp]
        lib.qwen3_decode_attn_check.restype = ctypes.c_int
        lib.qwen3_decode_attn_grid_ctas.argtypes = [vp]
        lib.qwen3_decode_attn_grid_ctas.restype = ctypes.c_int
        lib.qwen3_decode_attn_destroy.argtypes = [vp]
        lib.qwen3_decode_attn_destroy.restype = None
        lib.qwen3_decode_attn_strerror.argtypes = [ctypes.c_int]
        lib.qwen3_decode_attn_strerror.restype = ctypes.c_char_p
        _lib = lib
    return _lib


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _i32p(t: torch.Tensor | None):
    return None if t is None else ctypes.cast(ctypes.c_void_p(t.data_ptr()), ctypes.POINTER(ctypes.c_int32))


def _stream(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _expect(t: torch.Tensor, name: str, dtype, shape, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def qwen3_decode_attn_strerror(code: int) -> str:
    return load_library().qwen3_decode_attn_strerror(int(code)).decode()


def qwen3_decode_attn_default_config(**overrides) -> qda_config:
    cfg = qda_config()
    load_library().qwen3_decode_attn_default_config(ctypes.byref(cfg))
    for k, v in overrides.items():
        setattr(cfg, k, v)
    return cfg


def qwen3_decode_attn_create(cfg: qda_config | None = None, device: int = 0) -> ctypes.c_void_p:
    cfg = cfg if cfg is not None else qwen3_decode_attn_default_config()
    h = ctypes.c_void_p()
    rc = load_library().qwen3_decode_attn_create(ctypes.byref(cfg), int(device), ctypes.byref(h))
    if rc != QDA_OK:
        raise QdaError(rc, "qwen3_decode_attn_create")
    return h


def num_q_heads_of(qkv: torch.Tensor) -> int:
    """Query heads of a fused qkv row of (Hq + 16) * 128 values (qkv [B, W] or [B, T, W])."""
    if qkv.dim() not in (2, 3) or qkv.shape[-1] % HEAD_DIM != 0:
        raise ValueError("qkv must be [B, (num_q_heads + 16) * 128] or [B, T, (num_q_heads + 16) * 128]")
    return int(qkv.shape[-1]) // HEAD_DIM - 2 * NUM_KV_HEADS


def _step_args(qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table, k_cache, v_cache, o,
               dev_of_step, dev_of_state):
    Hq = num_q_heads_of(qkv)
    B = qkv.shape[0]
    tokens = tuple(qkv.shape[1:-1])   # () for one new token, (T,) for several
    _expect(qkv, "qkv", torch.bfloat16, (B, *tokens, (Hq + 2 * NUM_KV_HEADS) * HEAD_DIM), dev_of_step)
    _expect(q_norm_w, "q_norm_w", torch.bfloat16, (HEAD_DIM,), dev_of_state)
    _expect(k_norm_w, "k_norm_w", torch.bfloat16, (HEAD_DIM,), dev_of_state)
    _expect(seq_lens, "seq_lens", torch.int32, (B,), dev_of_step)
    if positions is not None:
        _expect(positions, "positions", torch.int32, (B,), dev_of_step)
    if block_table.dim() != 2:
        raise ValueError("block_table must be [B, stride]")
    _expect(block_table, "block_table", torch.int32, (B, block_table.shape[1]), dev_of_step)
    P = k_cache.shape[0]
    _expect(k_cache, "k_cache", torch.bfloat16, (P, PAGE_SIZE, NUM_KV_HEADS, HEAD_DIM), dev_of_state)
    _expect(v_cache, "v_cache", torch.bfloat16, (P, PAGE_SIZE, NUM_KV_HEADS, HEAD_DIM), dev_of_state)
    _expect(o, "o", torch.bfloat16, (B, *tokens, Hq, HEAD_DIM), dev_of_step)
    return (_ptr(qkv), _ptr(q_norm_w), _ptr(k_norm_w), _i32p(seq_lens), _i32p(positions),
            _i32p(block_table), int(block_table.shape[1]), _ptr(k_cache), _ptr(v_cache), int(P),
            _ptr(o), int(B))


def qwen3_decode_attn_append_and_attend(handle, qkv, q_norm_w, k_norm_w, seq_lens, positions,
                                        block_table, k_cache, v_cache, o, stream=None) -> None:
    """The step on device tensors; asynchronous on `stream`. Raises QdaError on a host-side error."""
    dev = qkv.device
    if dev.type != "cuda":
        raise ValueError("qkv must be a CUDA tensor")
    if qkv.dim() != 2:
        raise ValueError("qkv must be [B, (num_q_heads + 16) * 128]; several new tokens go through "
                         "qwen3_decode_attn_append_and_attend_tokens")
    args = _step_args(qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table, k_cache, v_cache, o, dev, dev)
    rc = load_library().qwen3_decode_attn_append_and_attend(handle, *args, _stream(stream, dev))
    if rc != QDA_OK:
        raise QdaError(rc, "qwen3_decode_attn_append_and_attend")


def qwen3_decode_attn_append_and_attend_tokens(handle, qkv, q_norm_w, k_norm_w, seq_lens, positions,
                                               block_table, k_cache, v_cache, o, stream=None) -> None:
    """The step with T new tokens per sequence: qkv [B, T, W], o [B, T, Hq, 128];
    token t goes to cache slot seq_lens[b] - T + t and attends causally up to it.
    Asynchronous on `stream`; raises QdaError on a host-side error."""
    dev = qkv.device
    if dev.type != "cuda":
        raise ValueError("qkv must be a CUDA tensor")
    if qkv.dim() != 3:
        raise ValueError("qkv must be [B, T, (num_q_heads + 16) * 128]")
    args = _step_args(qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table, k_cache, v_cache, o, dev, dev)
    rc = load_library().qwen3_decode_attn_append_and_attend_tokens(handle, *args, int(qkv.shape[1]),
                                                                   _stream(stream, dev))
    if rc != QDA_OK:
        raise QdaError(rc, "qwen3_decode_attn_append_and_attend_tokens")


def _proj_args(qkv_width, x, input_norm_w, w_qkv, qkv, dev):
    if x.dim() != 2:
        raise ValueError("x must be [B, hidden]")
    B, hidden = int(x.shape[0]), int(x.shape[1])
    _expect(x, "x", torch.bfloat16, (B, hidden), dev)
    _expect(input_norm_w, "input_norm_w", torch.bfloat16, (hidden,), dev)
    _expect(w_qkv, "w_qkv", torch.bfloat16, (qkv_width, hidden), dev)
    _expect(qkv, "qkv", torch.bfloat16, (B, qkv_width), dev)
    return B, hidden


def qwen3_decode_attn_qkv_proj(handle, num_q_heads, x, input_norm_w, w_qkv, qkv, stream=None) -> None:
    """input_norm + attn.qkv_proj on device tensors: x [B, hidden], input_norm_w [hidden],
    w_qkv [(Hq + 16) * 128, hidden] (rows q | k | v), qkv [B, (Hq + 16) * 128] (output)."""
    dev = x.device
    B, hidden = _proj_args((num_q_heads + 2 * NUM_KV_HEADS) * HEAD_DIM, x, input_norm_w, w_qkv, qkv, dev)
    rc = load_library().qwen3_decode_attn_qkv_proj(handle, _ptr(x), _ptr(input_norm_w), _ptr(w_qkv), hidden,
                                                   _ptr(qkv), B, _stream(stream, dev))
    if rc != QDA_OK:
        raise QdaError(rc, "qwen3_decode_attn_qkv_proj")


def qwen3_decode_attn_o_proj(handle, num_q_heads, x, w_o, y, stream=None) -> None:
    """attn.o_proj on device tensors: x [B, Hq, 128] or [B, Hq * 128] (the attention
    output), w_o [hidden, Hq * 128], y [B, hidden] (output)."""
    dev = x.device
    K = num_q_heads * HEAD_DIM
    B = int(x.shape[0])
    if x.dim() == 3:
        _expect(x, "x", torch.bfloat16, (B, num_q_heads, HEAD_DIM), dev)
    else:
        _expect(x, "x", torch.bfloat16, (B, K), dev)
    if w_o.dim() != 2:
        raise ValueError("w_o must be [hidden, Hq * 128]")
    hidden = int(w_o.shape[0])
    _expect(w_o, "w_o", torch.bfloat16, (hidden, K), dev)
    _expect(y, "y", torch.bfloat16, (B, hidden), dev)
    rc = load_library().qwen3_decode_attn_o_proj(handle, _ptr(x), _ptr(w_o), hidden, _ptr(y), B, _stream(stream, dev))
    if rc != QDA_OK:
        raise QdaError(rc, "qwen3_decode_attn_o_proj")


def qwen3_decode_attn_from_hidden(handle, num_q_heads, x, input_norm_w, w_qkv, qkv, q_norm_w, k_norm_w, seq_lens,
                                  positions, block_table, k_cache, v_cache, o, stream=None) -> None:
    """qkv_proj into `qkv`, then the attention step on it (one new token per sequence)."""
    dev = x.device
    B, hidden = _proj_args((num_q_heads + 2 * NUM_KV_HEADS) * HEAD_DIM, x, input_norm_w, w_qkv, qkv, dev)
    args = _step_args(qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table, k_cache, v_cache, o, dev, dev)
    rc = load_library().qwen3_decode_attn_from_hidden(handle, _ptr(x), _ptr(input_norm_w), _ptr(w_qkv), hidden,
                                                      *args, _stream(stream, dev))
    if rc != QDA_OK:
        raise QdaError(rc, "qwen3_decode_attn_from_hidden")


def qwen3_decode_attn_append_and_attend_host(handle, qkv, q_norm_w, k_norm_w, seq_lens, positions,
                                             block_table, k_cache, v_cache, o, stream=None) -> None:
    """The step with per-step tensors (qkv, seq_lens, positions, block_table, o) in host
    memory and weights/cache on the device; o is valid after the stream synchronizes."""
    dev = k_cache.device
    cpu = torch.device("cpu")
    args = _step_args(qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table, k_cache, v_cache, o, cpu, dev)
    if qkv.dim() != 2:
        raise ValueError("the host-buffer entry point takes one new token per sequence: qkv [B, W]")
    rc = load_library().qwen3_decode_attn_append_and_attend_host(handle, *args, _stream(stream, dev))
    if rc != QDA_OK:
        raise QdaError(rc, "qwen3_decode_attn_append_and_attend_host")


def qwen3_decode_attn_append_and_attend_noalloc(qkv, q_norm_w, k_norm_w, seq_lens, positions,
                                                block_table, k_cache, v_cache, o, stream=None) -> None:
    """The step without a handle, for callers that cannot allocate device memory:
    its scratch is a fixed array inside the library (see the C header). Runs on
    the current device, asynchronously on `stream`; raises QdaError on a
    host-side error."""
    dev = qkv.device
    if dev.type != "cuda":
        raise ValueError("qkv must be a CUDA tensor")
    if qkv.dim() != 2:
        raise ValueError("the no-allocation entry point takes one new token per sequence: qkv [B, W]")
    args = _step_args(qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table, k_cache, v_cache, o, dev, dev)
    f = load_library().qwen3_decode_attn_append_and_attend_noalloc
    vp, i32p = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)
    f.argtypes = [vp, vp, vp, i32p, i32p, i32p, ctypes.c_int, vp, vp, ctypes.c_int, vp, ctypes.c_int, vp]
    f.restype = ctypes.c_int
    rc = f(*args, _stream(stream, dev))
    if rc != QDA_OK:
        raise QdaError(rc, "qwen3_decode_attn_append_and_attend_noalloc")


def qwen3_decode_attn_check(handle, stream=None, device=None) -> int:
    """Synchronize the stream and return (and clear) the device status code."""
    return int(load_library().qwen3_decode_attn_check(handle, _stream(stream, device)))


def qwen3_decode_attn_grid_ctas(handle) -> int:
    return int(load_library().qwen3_decode_attn_grid_ctas(handle))


def qwen3_decode_attn_destroy(handle) -> None:
    load_library().qwen3_decode_attn_destroy(handle)


class DecodeAttention:
    """A handle with its lifetime: DecodeAttention(device=0, **config fields).

    `num_q_heads` (16, 32, 40 or 64) selects the Qwen3 size; calls must pass qkv
    rows of (num_q_heads + 16) * 128 values: qkv [B, W] for one new token per
    sequence (o [B, Hq, 128]), or [B, T, W] for T new tokens (o [B, T, Hq, 128])."""

    def __init__(self, device: int = 0, **config):
        self.device = torch.device("cuda", device)
        self.config = qwen3_decode_attn_default_config(**config)
        self.handle = qwen3_decode_attn_create(self.config, device)

    @property
    def grid_ctas(self) -> int:
        return qwen3_decode_attn_grid_ctas(self.handle)

    def __call__(self, qkv, q_norm_w, k_norm_w, seq_lens, block_table, k_cache, v_cache, o=None,
                 positions=None, stream=None) -> torch.Tensor:
        if num_q_heads_of(qkv) != self.config.num_q_heads:
            raise ValueError(f"qkv rows hold {num_q_heads_of(qkv)} query heads; the handle was made for "
                             f"{self.config.num_q_heads}")
        if o is None:
            o = torch.empty((*qkv.shape[:-1], self.config.num_q_heads, HEAD_DIM), dtype=torch.bfloat16,
                            device=qkv.device)
        step = qwen3_decode_attn_append_and_attend_tokens if qkv.dim() == 3 else qwen3_decode_attn_append_and_attend
        step(self.handle, qkv, q_norm_w, k_norm_w, seq_lens, positions, block_table, k_cache, v_cache, o, stream)
        return o

    def qkv_proj(self, x, input_norm_w, w_qkv, qkv=None, stream=None) -> torch.Tensor:
        """input_norm + attn.qkv_proj: the step's qkv [B, (Hq + 16) * 128] from x [B, hidden]."""
        if qkv is None:
            qkv = torch.empty((x.shape[0], (self.config.num_q_heads + 16) * HEAD_DIM), dtype=torch.bfloat16,
                              device=x.device)
        qwen3_decode_attn_qkv_proj(self.handle, self.config.num_q_heads, x, input_norm_w, w_qkv, qkv, stream)
        return qkv

    def o_proj(self, x, w_o, y=None, stream=None) -> torch.Tensor:
        """attn.o_proj: y [B, hidden] from the attention output x [B, Hq, 128] (or [B, Hq * 128])."""
        if y is None:
            y = torch.empty((x.shape[0], w_o.shape[0]), dtype=torch.bfloat16, device=x.device)
        qwen3_decode_attn_o_proj(self.handle, self.config.num_q_heads, x, w_o, y, stream)
        return y

    def from_hidden(self, x, input_norm_w, w_qkv, q_norm_w, k_norm_w, seq_lens, block_table, k_cache, v_cache,
                    qkv=None, o=None, positions=None, stream=None):
        """The attention from the hidden state: returns (o, qkv)."""
        B = x.shape[0]
        if qkv is None:
            qkv = torch.empty((B, (self.config.num_q_heads + 16) * HEAD_DIM), dtype=torch.bfloat16, device=x.device)
        if o is None:
            o = torch.empty((B, self.config.num_q_heads, HEAD_DIM), dtype=torch.bfloat16, device=x.device)
        qwen3_decode_attn_from_hidden(self.handle, self.config.num_q_heads, x, input_norm_w, w_qkv, qkv, q_norm_w,
                                      k_norm_w, seq_lens, positions, block_table, k_cache, v_cache, o, stream)
        return o, qkv

    def check(self, stream=None) -> int:
        return qwen3_decode_attn_check(self.handle, stream, self.device)

    def close(self) -> None:
        if getattr(self, "handle", None) is not None:
            qwen3_decode_attn_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
