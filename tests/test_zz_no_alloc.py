"""The handle-free entry point for callers that cannot allocate device memory.

Some users of this library cannot call cudaMalloc: code running inside a
framework or server that owns all device memory through its own pool, plugins
that are only handed pre-allocated buffers, and latency-critical loops where an
allocation (which can synchronize the device or fail at call time) is not
acceptable. For them qwen3_decode_attn_append_and_attend_noalloc keeps the
kernel's scratch in a fixed array inside the library.

This test calls it through the C ABI twice in a row, on workloads whose
sequences are split across CTAs (so the scratch partials and merge counters are
used, and the second call starts from the first call's leftovers), and checks
each result against qwen3_decode_attn_append_and_attend on the same inputs: o
within the parity tests' tolerance, the cache bit for bit. The first call is
also checked against the float64 oracle itself, and one more call passes
explicit RoPE positions. Further calls must leave the device's free memory
where it was (the entry point allocates nothing), and a batch larger than the
scratch's maximum is refused. This file is collected last so that a run
stopping at the first failure has run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from decode_attention_qk_b200 import binding, inputs
import parity_helpers as ph

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


def _noalloc_fn():
    from decode_attention_qk_b200 import build
    build.build_library()
    f = binding.load_library().qwen3_decode_attn_append_and_attend_noalloc
    vp, i32p = ctypes.c_void_p, ctypes.POINTER(ctypes.c_int32)
    f.argtypes = [vp, vp, vp, i32p, i32p, i32p, ctypes.c_int, vp, vp, ctypes.c_int, vp, ctypes.c_int, vp]
    f.restype = ctypes.c_int
    return f


def _args(w, k_cache, v_cache, o, batch=None, positions=None):
    a = ph.device_args(w, DEV, positions)
    i32 = lambda t: ctypes.cast(ctypes.c_void_p(t.data_ptr()), ctypes.POINTER(ctypes.c_int32))
    keep = (a, k_cache, v_cache, o)   # the tensors must outlive the call
    pos = None if a["positions"] is None else i32(a["positions"])
    return keep, (ctypes.c_void_p(a["qkv"].data_ptr()), ctypes.c_void_p(a["q_norm_w"].data_ptr()),
                  ctypes.c_void_p(a["k_norm_w"].data_ptr()), i32(a["seq_lens"]), pos, i32(a["block_table"]),
                  int(w.block_table.shape[1]), ctypes.c_void_p(k_cache.data_ptr()),
                  ctypes.c_void_p(v_cache.data_ptr()), int(w.num_pages), ctypes.c_void_p(o.data_ptr()),
                  int(batch if batch is not None else w.batch),
                  ctypes.c_void_p(torch.cuda.current_stream(DEV).cuda_stream))


def test_noalloc_entry_point_matches_the_handle_entry_point_twice_in_a_row():
    f = _noalloc_fn()
    attn = binding.DecodeAttention(device=0)
    g = torch.Generator().manual_seed(40)
    workloads = [
        inputs.custom([5000, 3000, 17, 1, 40960, 777], seed=41, device="cuda", stride=2560, gap_fraction=0.1),
        inputs.custom(torch.randint(1, 4097, (32,), generator=g).tolist(), seed=42, device="cuda"),
    ]
    for n, w in enumerate(workloads):
        k_ref, v_ref = w.k_cache.clone(), w.v_cache.clone()
        o_ref = ph.run(attn, w, DEV, k_ref, v_ref)
        assert attn.check() == 0
        k, v = w.k_cache.clone(), w.v_cache.clone()
        o = torch.empty_like(o_ref)
        keep, args = _args(w, k, v, o)
        assert f(*args) == binding.QDA_OK
        torch.cuda.synchronize(DEV)
        ph.assert_o_close(o, o_ref.double().cpu().numpy(), f"no-alloc call {n + 1} vs handle call")
        assert torch.equal(k.view(torch.int16), k_ref.view(torch.int16))
        assert torch.equal(v.view(torch.int16), v_ref.view(torch.int16))
        if n == 0:   # and against the float64 oracle: cache bit for bit, o within the parity tolerance
            ref = ph.oracle_full(w, w.k_cache, w.v_cache)
            assert np.array_equal(inputs.bf16_bits(k), ref["k_cache"])
            assert np.array_equal(inputs.bf16_bits(v), ref["v_cache"])
            ph.assert_o_close(o, ref["o"], "no-alloc call vs the oracle")
    attn.close()


def test_noalloc_entry_point_with_explicit_positions_matches_the_oracle():
    f = _noalloc_fn()
    lens = [1, 16, 17, 2500, 40960, 300]
    w = inputs.custom(lens, seed=44, device="cuda", gap_fraction=0.1)
    positions = torch.tensor([7000, 3, 40000, 2499, 40959, 12345], dtype=torch.int32)
    k, v = w.k_cache.clone(), w.v_cache.clone()
    o = torch.empty((w.batch, 16, 128), dtype=torch.bfloat16, device=DEV)
    keep, args = _args(w, k, v, o, positions=positions)
    assert f(*args) == binding.QDA_OK
    torch.cuda.synchronize(DEV)
    ref = ph.oracle_full(w, w.k_cache, w.v_cache, positions=positions)
    assert np.array_equal(inputs.bf16_bits(k), ref["k_cache"])
    assert np.array_equal(inputs.bf16_bits(v), ref["v_cache"])
    ph.assert_o_close(o, ref["o"], "no-alloc call with positions vs the oracle")


def test_noalloc_calls_leave_device_memory_unchanged():
    """After the first call on the device (its one-time set-up), further calls
    take no device memory: the free memory the driver reports does not drop."""
    f = _noalloc_fn()
    w = inputs.custom([4000, 33, 1, 9000], seed=45, device="cuda")
    o = torch.empty((w.batch, 16, 128), dtype=torch.bfloat16, device=DEV)
    keep, args = _args(w, w.k_cache, w.v_cache, o)
    assert f(*args) == binding.QDA_OK
    torch.cuda.synchronize(DEV)
    free_before, _ = torch.cuda.mem_get_info(DEV)
    for _ in range(8):
        assert f(*args) == binding.QDA_OK
    torch.cuda.synchronize(DEV)
    free_after, _ = torch.cuda.mem_get_info(DEV)
    assert free_after >= free_before, f"free device memory dropped by {free_before - free_after} bytes"


def test_noalloc_entry_point_refuses_a_batch_beyond_its_maximum():
    f = _noalloc_fn()
    w = inputs.custom([3] * 4, seed=43, device="cuda")
    o = torch.empty((4, 16, 128), dtype=torch.bfloat16, device=DEV)
    keep, args = _args(w, w.k_cache, w.v_cache, o, batch=257)
    assert f(*args) == binding.QDA_ERR_INVALID_ARG
