"""Parity of the larger-Qwen3 kernels (32, 40, 64 query heads over 8 kv heads)
with the float64 oracle, through the C ABI.

nnterp qwen3, "Grouped-query attention, with 128-wide heads on every size":
4B and 8B have 32 query heads, 14B 40, 32B 64, all over 8 kv heads of 128.
The same checks as the 16-head kernel: the whole cache bit for bit, o within
the gate and the strict bound.
"""
import dataclasses

import numpy as np
import pytest
import torch

from decode_attention_qk_b200 import binding, inputs
import parity_helpers as ph

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
HEADS = [32, 40, 64]


@pytest.fixture(scope="module")
def handles():
    from decode_attention_qk_b200 import build
    build.build_library()
    hs = {hq: binding.DecodeAttention(device=0, num_q_heads=hq) for hq in HEADS}
    yield hs
    for h in hs.values():
        h.close()


def full_check(attn, w, label, positions=None):
    k, v = w.k_cache.to(DEV), w.v_cache.to(DEV)
    ref = ph.oracle_full(w, k, v, positions=positions)
    o = ph.run(attn, w, DEV, k, v, positions=positions)
    assert attn.check() == 0
    assert o.shape == (w.batch, w.num_q_heads, 128)
    got_k, got_v = inputs.bf16_bits(k), inputs.bf16_bits(v)
    if not np.array_equal(got_k, ref["k_cache"]):
        bad = np.argwhere(got_k != ref["k_cache"])[:8].tolist()
        raise AssertionError(f"{label}: k cache differs at {bad}")
    assert np.array_equal(got_v, ref["v_cache"]), f"{label}: v cache differs"
    ph.assert_o_close(o, ref["o"], label)
    return o, ref


@pytest.mark.parametrize("hq", HEADS)
def test_page_edges(handles, hq):
    lens = [1, 2, 15, 16, 17, 31, 33, 64, 65, 300, 1000]
    full_check(handles[hq], inputs.custom(lens, seed=40 + hq, device="cuda", gap_fraction=0.2, num_q_heads=hq),
               f"Hq={hq} page edges")


@pytest.mark.parametrize("hq", HEADS)
def test_gains_at_a_4_byte_aligned_address(handles, hq):
    w = inputs.custom([1, 17, 300, 33], seed=45, device="cuda", num_q_heads=hq)
    full_check(handles[hq], ph.gains_at_a_4_byte_offset(w), f"Hq={hq} gains at +4 bytes")


@pytest.mark.parametrize("hq", HEADS)
def test_single_position_returns_v_bits(handles, hq):
    w = inputs.custom([1] * 9, seed=41, device="cuda", num_q_heads=hq)
    o, _ = full_check(handles[hq], w, f"Hq={hq} L=1")
    G = hq // 8
    v = w.qkv[:, (hq + 8) * 128:].reshape(9, 8, 1, 128).expand(9, 8, G, 128).reshape(9, hq, 128)
    assert torch.equal(o.view(torch.int16), v.contiguous().view(torch.int16))


@pytest.mark.parametrize("grid", [1, 3, 148, 1024])
def test_split_count_does_not_change_the_result(grid):
    a = binding.DecodeAttention(device=0, num_q_heads=64, grid_ctas=grid)
    w = inputs.custom([1, 16, 17, 300, 2000, 33], seed=42, device="cuda", gap_fraction=0.2, num_q_heads=64)
    full_check(a, w, f"Hq=64 grid {grid}")
    a.close()


def test_maximum_context(handles):
    w = inputs.custom([40960, 40959, 7], seed=43, device="cuda", stride=2560, num_q_heads=64)
    full_check(handles[64], w, "Hq=64 L=40960")


def test_positions_argument(handles):
    full_check(handles[40], inputs.custom([5, 100, 1234], seed=44, device="cuda", num_q_heads=40),
               "Hq=40 positions", positions=torch.tensor([0, 7000, 40000], dtype=torch.int32))


def test_locality_with_nan_in_unread_bytes(handles):
    """Rows past a sequence, pages it does not own and table entries past its last
    page may hold anything (here NaN): o and the appended rows do not change.
    The value product must not turn a stale NaN into NaN at probability 0."""
    attn = handles[64]
    w = inputs.custom([7, 12, 40, 16], seed=45, device="cuda", pool_pages=14, stride=6, num_q_heads=64)
    ka, va = w.k_cache.clone(), w.v_cache.clone()
    kb, vb = w.k_cache.clone(), w.v_cache.clone()
    bt2 = w.block_table.clone()
    used, slots = set(), []
    for b, L in enumerate(w.seq_lens.tolist()):
        n = (L + 15) // 16
        used.update(w.block_table[b, :n].tolist())
        last, row = int(w.block_table[b, n - 1]), (L - 1) % 16
        slots.append((last, row))
        kb[last, row:] = float("nan")     # the new row too: it is written, never read
        vb[last, row:] = float("nan")
        bt2[b, n:] = 10 ** 6
    for p in range(w.num_pages):
        if p not in used:
            kb[p] = float("nan")
            vb[p] = float("nan")
    o1 = ph.run(attn, w, DEV, ka, va)
    o2 = ph.run(attn, dataclasses.replace(w, block_table=bt2), DEV, kb, vb)
    assert attn.check() == 0
    assert not torch.isnan(o2.float()).any()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    for page, row in slots:
        assert torch.equal(ka[page, row].view(torch.int16), kb[page, row].view(torch.int16))
        assert torch.equal(va[page, row].view(torch.int16), vb[page, row].view(torch.int16))


def test_out_of_range_page_ids_are_not_dereferenced(handles):
    attn = handles[32]
    w = inputs.custom([40, 20, 30], seed=46, device="cuda", pool_pages=8, stride=3, num_q_heads=32)
    k, v = w.k_cache.clone(), w.v_cache.clone()
    bt = w.block_table.clone()
    bt[1, 1] = 8
    a = ph.device_args(w, DEV)
    o = attn(a["qkv"], a["q_norm_w"], a["k_norm_w"], a["seq_lens"], bt.to(DEV), k, v)
    assert attn.check() == binding.QDA_ERR_BOUNDS
    ref = ph.oracle_sampled(w, [0, 2], w.k_cache, w.v_cache)
    ph.assert_o_close(o[[0, 2]], ref, "Hq=32 bad page id")
    assert attn.check() == 0


def test_host_buffer_entry_point(handles):
    attn = handles[64]
    w = inputs.custom([77, 1, 16, 513], seed=47, device="cuda", num_q_heads=64)
    k0, v0 = w.k_cache.clone(), w.v_cache.clone()
    o_dev = ph.run(attn, w, DEV, w.k_cache, w.v_cache)
    pin = lambda t: t.cpu().pin_memory()
    o_host = torch.empty((4, 64, 128), dtype=torch.bfloat16).pin_memory()
    binding.qwen3_decode_attn_append_and_attend_host(
        attn.handle, pin(w.qkv), w.q_norm_w, w.k_norm_w, pin(w.seq_lens), None, pin(w.block_table),
        k0, v0, o_host)
    assert attn.check() == 0
    assert torch.equal(o_host.view(torch.int16), o_dev.cpu().view(torch.int16))
    assert torch.equal(k0.view(torch.int16), w.k_cache.view(torch.int16))


def test_handle_refuses_a_row_of_another_size(handles):
    w = inputs.custom([5], seed=48, device="cuda")   # 16-head rows
    with pytest.raises(ValueError):
        ph.run(handles[64], w, DEV, w.k_cache, w.v_cache)


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


@pytest.mark.parametrize("hq", HEADS)
def test_config2_shape_full_size(handles, hq):
    w = inputs.config2("cuda", num_q_heads=hq)
    full_size_check(handles[hq], w, list(range(0, 32, 3)), f"cfg2 Hq={hq}")


def test_config4_shape_full_size(handles):
    w = inputs.config4("cuda", num_q_heads=64)
    full_size_check(handles[64], w, [0, 3], "cfg4 Hq=64")
