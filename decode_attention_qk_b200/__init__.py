"""B200-native (sm_100a) Qwen3-0.6B decode-attention step.

The compute lives in ``libqwen3_decode_attn.so`` (CUDA kernels behind a C ABI,
declared in ``include/qwen3_decode_attn.h``); :mod:`.binding` marshals Python
arguments into it. Importing this package loads nothing: the binding is
imported on first use of one of its names, and it raises if the CUDA library
is missing. :mod:`.inputs` holds the seeded synthetic workloads.
"""
_BINDING_NAMES = {
    "DecodeAttention", "QdaError", "qda_config", "load_library", "LIBRARY_PATH",
    "qwen3_decode_attn_default_config", "qwen3_decode_attn_create",
    "qwen3_decode_attn_append_and_attend", "qwen3_decode_attn_append_and_attend_host",
    "qwen3_decode_attn_append_and_attend_noalloc",
    "qwen3_decode_attn_check", "qwen3_decode_attn_destroy", "qwen3_decode_attn_strerror",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
