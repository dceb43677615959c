"""Parity of the CUDA library (through its C ABI) with the float64 oracle.

Small cases compare everything: the whole cache bit for bit and every o value.
Full-size workloads (the shapes the benchmark times, in its launch
configuration) compare the whole cache bit for bit against the pre-call cache
plus the oracle's appended rows, and o on sampled sequences the oracle
recomputes one by one.
"""
import dataclasses

import numpy as np
import pytest
import torch

from decode_attention_qk_b200 import binding, inputs
import parity_helpers as ph

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module")
def attn():
    from decode_attention_qk_b200 import build
    build.build_library()
    a = binding.DecodeAttention(device=0)
    yield a
    a.close()


def full_check(attn, w, label, positions=None):
    """Run on the device and compare the whole cache and all of o with the oracle."""
    k, v = w.k_cache.to(DEV), w.v_cache.to(DEV)
    ref = ph.oracle_full(w, k, v, positions=positions)
    o = ph.run(attn, w, DEV, k, v, positions=positions)
    assert attn.check() == 0
    got_k, got_v = inputs.bf16_bits(k), inputs.bf16_bits(v)
    if not np.array_equal(got_k, ref["k_cache"]):
        bad = np.argwhere(got_k != ref["k_cache"])[:8].tolist()
        raise AssertionError(f"{label}: k cache differs at {bad}")
    assert np.array_equal(got_v, ref["v_cache"]), f"{label}: v cache differs"
    ph.assert_o_close(o, ref["o"], label)
    return o, ref


def test_config1(attn):
    full_check(attn, inputs.config1("cuda"), "cfg1")


@pytest.mark.parametrize("grid", [1, 2, 3, 5, 64, 148, 1024, 4096])
def test_split_count_does_not_change_the_result(grid):
    """The key range of a sequence may be cut into any number of pieces
    (online softmax + log-sum-exp combine equals the plain softmax)."""
    a = binding.DecodeAttention(device=0, grid_ctas=grid)
    assert a.grid_ctas == grid
    w = inputs.custom([1, 16, 17, 300, 1000, 33, 2], seed=11, device="cuda", gap_fraction=0.2)
    full_check(a, w, f"grid {grid}")
    a.close()


def test_gains_at_a_4_byte_aligned_address(attn):
    """The norm gains need only be 4-byte aligned (the ABI's requirement)."""
    w = inputs.custom([1, 17, 300, 33], seed=19, device="cuda")
    full_check(attn, ph.gains_at_a_4_byte_offset(w), "gains at +4 bytes")


def test_page_edge_lengths(attn):
    lens = [1, 2, 15, 16, 17, 18, 31, 32, 33, 47, 48, 49, 63, 64, 65, 255, 256, 257]
    full_check(attn, inputs.custom(lens, seed=12, device="cuda", gap_fraction=0.3), "page edges")


def test_single_position_returns_v_bits(attn):
    """L = 1: the softmax has one weight, exactly 1, so o is v's bits."""
    w = inputs.custom([1] * 37, seed=13, device="cuda")
    o, _ = full_check(attn, w, "L=1")
    v_bits = w.qkv[:, 3072:].reshape(37, 8, 1, 128).expand(37, 8, 2, 128).reshape(37, 16, 128)
    assert torch.equal(o.view(torch.int16), v_bits.contiguous().view(torch.int16))


def test_max_batch_ragged(attn):
    g = torch.Generator().manual_seed(14)
    lens = torch.randint(1, 700, (256,), generator=g).tolist()
    full_check(attn, inputs.custom(lens, seed=14, device="cuda", gap_fraction=0.1), "B=256 ragged")


def test_maximum_context(attn):
    w = inputs.custom([40960, 40959, 1], seed=15, device="cuda", stride=2560)
    full_check(attn, w, "L=40960")


def test_positions_argument(attn):
    w = inputs.custom([5, 100, 1234], seed=16, device="cuda")
    o_default, _ = full_check(attn, inputs.custom([5, 100, 1234], seed=16, device="cuda"), "positions NULL")
    o_same, _ = full_check(attn, w, "positions = L-1", positions=w.seq_lens - 1)
    assert torch.equal(o_default, o_same)
    full_check(attn, inputs.custom([5, 100, 1234], seed=16, device="cuda"), "positions shifted",
               positions=torch.tensor([0, 7000, 40000], dtype=torch.int32))


def test_zero_query_slice_attends_uniformly(attn):
    """nnterp qwen3, "An edit to q_proj.output is renormalized": a zero slice gives a
    zero query, so the head's output is the mean of v over the sequence."""
    w = inputs.custom([200], seed=17, device="cuda")
    w.qkv[0, 128 * 3:128 * 4] = 0
    _, ref = full_check(attn, w, "zero query")
    bt, L = w.block_table[0], 200
    vc = ref["v_cache"]
    mean_v = np.mean([oracle_bf16(vc[bt[t // 16], t % 16, 1]) for t in range(L)], axis=0)
    assert np.allclose(ref["o"][0, 3], mean_v, atol=1e-12)


def oracle_bf16(bits):
    import oracle
    return oracle.bf16_to_f64(bits)


def test_locality(attn):
    """Bytes the step must not read (other pages, rows past the sequence, table
    entries past its last page) do not change o or the appended rows at all."""
    import dataclasses
    w = inputs.custom([7, 12, 40], seed=18, device="cuda", pool_pages=12, stride=6)
    ka, va = w.k_cache.clone(), w.v_cache.clone()
    kb, vb = w.k_cache.clone(), w.v_cache.clone()
    bt2 = w.block_table.clone()
    used, slots = set(), []
    for b, L in enumerate(w.seq_lens.tolist()):
        n = (L + 15) // 16
        used.update(w.block_table[b, :n].tolist())
        last, row = int(w.block_table[b, n - 1]), (L - 1) % 16
        slots.append((last, row))
        kb[last, row + 1:] = float("nan")
        vb[last, row + 1:] = float("nan")
        bt2[b, n:] = 10 ** 6
    for p in range(w.num_pages):
        if p not in used:
            kb[p] = float("nan")
            vb[p] = float("nan")
    o1 = ph.run(attn, w, DEV, ka, va)
    o2 = ph.run(attn, dataclasses.replace(w, block_table=bt2), DEV, kb, vb)
    assert attn.check() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    for page, row in slots:
        assert torch.equal(ka[page, row].view(torch.int16), kb[page, row].view(torch.int16))
        assert torch.equal(va[page, row].view(torch.int16), vb[page, row].view(torch.int16))


def test_deterministic(attn):
    w = inputs.custom([3000, 17, 900], seed=19, device="cuda")
    k0, v0 = w.k_cache.clone(), w.v_cache.clone()
    o1 = ph.run(attn, w, DEV, w.k_cache, w.v_cache)
    o2 = ph.run(attn, w, DEV, k0, v0)
    assert attn.check() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))


def test_host_buffer_entry_point(attn):
    w = inputs.custom([77, 1, 16, 513], seed=20, device="cuda")
    k0, v0 = w.k_cache.clone(), w.v_cache.clone()
    o_dev = ph.run(attn, w, DEV, w.k_cache, w.v_cache)
    pin = lambda t: t.cpu().pin_memory()
    o_host = torch.empty((4, 16, 128), dtype=torch.bfloat16).pin_memory()
    binding.qwen3_decode_attn_append_and_attend_host(
        attn.handle, pin(w.qkv), w.q_norm_w, w.k_norm_w, pin(w.seq_lens), None, pin(w.block_table),
        k0, v0, o_host)
    assert attn.check() == 0
    assert torch.equal(o_host.view(torch.int16), o_dev.cpu().view(torch.int16))
    assert torch.equal(k0.view(torch.int16), w.k_cache.view(torch.int16))


def test_host_buffer_calls_back_to_back(attn):
    """Consecutive host-buffer calls on one stream, no synchronization between
    them: each call's stage-in may run while the previous call's attention
    still reads its staging set (alternate calls use alternate sets). Five
    calls, each on a different batch appending into the same caches (the next
    token of the same sequences), give the bytes of five device-entry calls."""
    lens0 = torch.tensor([77, 1, 16, 513, 2000, 33], dtype=torch.int32)
    w = inputs.custom((lens0 + 5).tolist(), seed=26, device="cuda", gap_fraction=0.2)
    kd, vd = w.k_cache.clone(), w.v_cache.clone()
    kh, vh = w.k_cache.clone(), w.v_cache.clone()
    steps = []
    for i in range(5):
        qkv = inputs.custom((lens0 + 5).tolist(), seed=27 + i, device="cuda").qkv
        steps.append(dataclasses.replace(w, qkv=qkv, seq_lens=(lens0 + 1 + i).contiguous()))
    o_dev = [ph.run(attn, wi, DEV, kd, vd) for wi in steps]
    torch.cuda.synchronize(DEV)
    pin = lambda t: t.cpu().pin_memory()
    host_in = [(pin(wi.qkv), pin(wi.seq_lens), pin(wi.block_table)) for wi in steps]
    o_host = [torch.empty((6, 16, 128), dtype=torch.bfloat16).pin_memory() for _ in steps]
    for (qkv_h, sl_h, bt_h), oh in zip(host_in, o_host):
        binding.qwen3_decode_attn_append_and_attend_host(attn.handle, qkv_h, w.q_norm_w, w.k_norm_w, sl_h, None, bt_h,
                                                         kh, vh, oh)
    assert attn.check() == 0
    for i in range(5):
        assert torch.equal(o_host[i].view(torch.int16), o_dev[i].cpu().view(torch.int16)), i
    assert torch.equal(kh.view(torch.int16), kd.view(torch.int16))
    assert torch.equal(vh.view(torch.int16), vd.view(torch.int16))


def pinned_at_offset(t):
    """A page-locked copy of int32 `t` starting 4 bytes past a 16-byte boundary."""
    flat = torch.empty(t.numel() + 1, dtype=t.dtype).pin_memory()
    v = flat[1:].view(t.shape)
    v.copy_(t)
    assert v.data_ptr() % 16 == 4
    return v


@pytest.mark.parametrize("mapped", ["none", "inputs", "o", "all", "offset"])
def test_host_buffer_entry_point_mixed_memory(attn, mapped):
    """Pageable buffers go through copies, page-locked ones through the
    stage-in launch (inputs) or in place (o), at 16-byte or only 4-byte
    alignment; any mix gives the bytes of the device entry point."""
    w = inputs.custom([300, 2, 16, 1025, 40], seed=25, device="cuda", gap_fraction=0.3)
    positions = (w.seq_lens - 1 + torch.tensor([0, 5, 0, 1000, 7], dtype=torch.int32)).contiguous()
    k0, v0 = w.k_cache.clone(), w.v_cache.clone()
    a = ph.device_args(w, DEV)
    o_dev = attn(a["qkv"], a["q_norm_w"], a["k_norm_w"], a["seq_lens"], a["block_table"], w.k_cache, w.v_cache,
                 positions=positions.to(DEV))
    torch.cuda.synchronize(DEV)
    pin_in = mapped in ("inputs", "all")
    host = lambda t, pin: t.cpu().pin_memory() if pin else t.cpu().clone()
    ints = pinned_at_offset if mapped == "offset" else (lambda t: host(t, pin_in))
    o_host = torch.full((5, 16, 128), 3.0, dtype=torch.bfloat16)
    if mapped in ("o", "all"):
        o_host = o_host.pin_memory()
    binding.qwen3_decode_attn_append_and_attend_host(
        attn.handle, host(w.qkv, pin_in or mapped == "offset"), w.q_norm_w, w.k_norm_w, ints(w.seq_lens),
        ints(positions), ints(w.block_table), k0, v0, o_host)
    torch.cuda.synchronize(DEV)
    assert attn.check() == 0
    assert torch.equal(o_host.view(torch.int16), o_dev.cpu().view(torch.int16))
    assert torch.equal(k0.view(torch.int16), w.k_cache.view(torch.int16))
    assert torch.equal(v0.view(torch.int16), w.v_cache.view(torch.int16))


# ----------------------------------------------------------------------------
# device-side errors: recorded in the status word, no out-of-range access

def test_out_of_range_seq_lens_skip_the_sequence(attn):
    w = inputs.custom([9, 20, 5, 33], seed=21, device="cuda", pool_pages=8, stride=3)
    for bad in (0, -5, 49, 40961):          # 49 > 16 * stride
        k, v = w.k_cache.clone(), w.v_cache.clone()
        lens = w.seq_lens.clone()
        lens[2] = bad
        o = torch.full((4, 16, 128), 7.0, dtype=torch.bfloat16, device=DEV)
        a = ph.device_args(w, DEV)
        attn(a["qkv"], a["q_norm_w"], a["k_norm_w"], lens.to(DEV), a["block_table"], k, v, o=o)
        assert attn.check() == binding.QDA_ERR_BOUNDS, bad
        assert torch.all(o[2] == 7.0)
        # the valid sequences are still right
        keep = [0, 1, 3]
        ref = ph.oracle_sampled(w, keep, w.k_cache, w.v_cache)
        ph.assert_o_close(o[keep], ref, f"seq_len {bad}")
    assert attn.check() == 0


def test_out_of_range_page_ids_are_not_dereferenced(attn):
    w = inputs.custom([40, 20, 30], seed=22, device="cuda", pool_pages=8, stride=3)
    for bad in (-1, 8, 1 << 30):
        k, v = w.k_cache.clone(), w.v_cache.clone()
        bt = w.block_table.clone()
        bt[1, 1] = bad                      # the last page of sequence 1 (its append slot)
        a = ph.device_args(w, DEV)
        o = attn(a["qkv"], a["q_norm_w"], a["k_norm_w"], a["seq_lens"], bt.to(DEV), k, v)
        assert attn.check() == binding.QDA_ERR_BOUNDS
        ref = ph.oracle_sampled(w, [0, 2], w.k_cache, w.v_cache)
        ph.assert_o_close(o[[0, 2]], ref, f"page id {bad}")
        # only sequences 0 and 2 appended
        changed = (k.view(torch.int16) != w.k_cache.view(torch.int16)).any(dim=(1, 2, 3)).nonzero().flatten()
        for p in changed.tolist():
            assert p in (int(w.block_table[0, 2]), int(w.block_table[2, 1]))
    assert attn.check() == 0


def test_wait_timeout_is_reported_and_the_handle_recovers():
    """A wait on a barrier nothing completes ends after the configured limit with
    QDA_ERR_TIMEOUT; the call's result is still right and the handle still works."""
    a = binding.DecodeAttention(device=0, flags=binding.QDA_FLAG_INJECT_WAIT_TIMEOUT, wait_timeout_ns=2_000_000)
    w = inputs.custom([100, 5], seed=23, device="cuda")
    k, v = w.k_cache.clone(), w.v_cache.clone()
    ref = ph.oracle_full(w, k.clone(), v.clone())
    o = ph.run(a, w, DEV, k, v)
    assert a.check() == binding.QDA_ERR_TIMEOUT
    ph.assert_o_close(o, ref["o"], "timeout injection")
    a.close()
    b = binding.DecodeAttention(device=0)
    full_check(b, inputs.custom([100, 5], seed=23, device="cuda"), "after timeout")
    b.close()


# ----------------------------------------------------------------------------
# full-size workloads, in the benchmark's launch configuration

def full_size_check(attn, w, sample, label):
    k_pre, v_pre = w.k_cache.clone(), w.v_cache.clone()
    o = ph.run(attn, w, DEV, w.k_cache, w.v_cache)
    assert attn.check() == 0
    k_rows, v_rows, k64 = ph.oracle_appended_rows(w, k_pre, v_pre)
    k_exp, v_exp = ph.expected_cache(w, k_pre, v_pre, k_rows, v_rows)
    ph.assert_cache_equal(w.k_cache, w.v_cache, k_exp, v_exp, k64, w)
    del k_exp, v_exp
    ref = ph.oracle_sampled(w, sample, k_pre, v_pre)
    return ph.assert_o_close(o[torch.as_tensor(sample)], ref, label)


def test_config2_full_size(attn):
    w = inputs.config2("cuda")
    full_size_check(attn, w, list(range(32)), "cfg2")


def test_config4_full_size(attn):
    w = inputs.config4("cuda")
    full_size_check(attn, w, [0, 1, 2, 3], "cfg4")


def test_config5_full_size(attn):
    w = inputs.config5("cuda")
    g = torch.Generator().manual_seed(5)
    sample = sorted(set(torch.randint(0, 256, (24,), generator=g).tolist()) |
                    {int(w.seq_lens.argmax()), int(w.seq_lens.argmin())})
    full_size_check(attn, w, sample, "cfg5")


def test_config3_all_layers(attn):
    """28 independent layer caches, one call per layer back to back (the benchmark's
    step); three layers get a whole-cache comparison, every layer its appended rows
    and 8 sampled sequences."""
    layers = [inputs.config3_layer(i, "cuda") for i in range(inputs.CONFIG3_LAYERS)]
    full = {0, 13, 27}
    pre = {i: (layers[i].k_cache.clone(), layers[i].v_cache.clone()) for i in full}
    appended = {}
    for i, w in enumerate(layers):
        appended[i] = ph.oracle_appended_rows(w, w.k_cache, w.v_cache)
    outs = [ph.run(attn, w, DEV, w.k_cache, w.v_cache) for w in layers]
    assert attn.check() == 0
    g = torch.Generator().manual_seed(3)
    for i, w in enumerate(layers):
        k_rows, v_rows, k64 = appended[i]
        if i in full:
            k_exp, v_exp = ph.expected_cache(w, *pre[i], k_rows, v_rows)
            ph.assert_cache_equal(w.k_cache, w.v_cache, k_exp, v_exp, k64, w)
            del k_exp, v_exp
        for b in range(w.batch):
            page, row = int(w.block_table[b, 127]), 15
            assert np.array_equal(inputs.bf16_bits(w.k_cache[page, row]), k_rows[b, 0])
            assert np.array_equal(inputs.bf16_bits(w.v_cache[page, row]), v_rows[b, 0])
        sample = torch.randint(0, 256, (8,), generator=g).tolist()
        # the oracle reads the pre-call cache; rows other than the appended ones are unchanged
        ref = ph.oracle_sampled(w, sample, w.k_cache, w.v_cache)
        ph.assert_o_close(outs[i][torch.as_tensor(sample)], ref, f"cfg3 layer {i}")


def test_rope_theta_is_a_runtime_parameter():
    """nnterp qwen3, "What loads as this family": rope_theta is 1e6 everywhere but the
    4B-2507 pair (5e6). The base is a create-time parameter; the oracle takes the same."""
    a = binding.DecodeAttention(device=0, rope_theta=5.0e6)
    w = inputs.custom([40960, 3, 1000, 17], seed=24, device="cuda", stride=2560)
    k, v = w.k_cache.clone(), w.v_cache.clone()
    ref = ph.oracle.append_and_attend(
        inputs.bf16_bits(w.qkv), inputs.bf16_bits(w.q_norm_w), inputs.bf16_bits(w.k_norm_w),
        w.seq_lens.numpy(), w.block_table.numpy(), inputs.bf16_bits(k), inputs.bf16_bits(v), rope_theta=5.0e6)
    o = ph.run(a, w, DEV, k, v)
    assert a.check() == 0
    assert np.array_equal(inputs.bf16_bits(k), ref["k_cache"]) and np.array_equal(inputs.bf16_bits(v), ref["v_cache"])
    ph.assert_o_close(o, ref["o"], "theta 5e6")
    a.close()
