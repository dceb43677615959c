"""Parity of the step with several new tokens per sequence (causal inside the
new block) with the float64 oracle, through the C ABI: up to 16 query rows per
kv head in one launch of the decode-shaped kernel, longer blocks as the chunked
prefill (128 query rows per kv head per chunk).

Token t of sequence b goes to cache slot L - T + t (L = seq_lens[b] counts the
new tokens) and its query attends over slots 0 .. L - T + t (Qwen3-0.6B Model
Spec, "What to watch for": every layer is full causal attention). The checks
are those of the one-token step: the whole cache bit for bit, o within the
gate and the strict bound. Instances with more than 8 query rows per kv head
(T * Hq / 8 > 8) take q and the probabilities as bf16; their o is held to the
gate against the oracle and to the bound of parity_helpers.emulated_bf16_q_check.
"""
import dataclasses

import numpy as np
import pytest
import torch

from decode_attention_qk_b200 import binding, inputs
import parity_helpers as ph

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
CASES = list(binding.SUPPORTED_MULTI_TOKEN)   # (query heads, new tokens)


@pytest.fixture(scope="module")
def handles():
    from decode_attention_qk_b200 import build
    build.build_library()
    hs = {hq: binding.DecodeAttention(device=0, num_q_heads=hq) for hq in (16, 32, 40, 64)}
    yield hs
    for h in hs.values():
        h.close()


def check_o(o, ref, w, label):
    """The required gate against the oracle over all of o; then, per new
    token, the one-token step's strict bound, or for tokens whose launch took
    q as bf16 (more than 8 query rows per kv head) the bf16-q bound."""
    if not ph.is_wide(w):
        return ph.assert_o_close(o, ref["o"], label)
    max_abs, rel, _ = ph.o_errors(o, ref["o"])
    assert max_abs <= ph.GATE_ABS and rel <= ph.GATE_REL, f"{label}: max abs {max_abs:.3g}, rel rms {rel:.3g}"
    flags = ph.wide_tokens(w)
    narrow = [t for t, f in enumerate(flags) if not f]
    if narrow:
        ph.assert_o_close(o[:, narrow], ref["o"][:, narrow], label + " (two-term rows)")
    ph.emulated_bf16_q_check(o, ref["q"], ref["seq_lens"], ref["block_table"], ref["k_cache"], ref["v_cache"],
                             w.new_tokens, label, tokens=[t for t, f in enumerate(flags) if f])
    return max_abs, rel


def full_check(attn, w, label, positions=None):
    k, v = w.k_cache.to(DEV), w.v_cache.to(DEV)
    ref = ph.oracle_full(w, k, v, positions=positions)
    ref["seq_lens"], ref["block_table"] = w.seq_lens.numpy(), w.block_table.numpy()
    o = ph.run(attn, w, DEV, k, v, positions=positions)
    assert attn.check() == 0
    assert o.shape == (w.batch, w.new_tokens, w.num_q_heads, 128)
    got_k, got_v = inputs.bf16_bits(k), inputs.bf16_bits(v)
    if not np.array_equal(got_k, ref["k_cache"]):
        bad = np.argwhere(got_k != ref["k_cache"])[:8].tolist()
        raise AssertionError(f"{label}: k cache differs at {bad}")
    assert np.array_equal(got_v, ref["v_cache"]), f"{label}: v cache differs"
    check_o(o, ref, w, label)
    return o, ref


@pytest.mark.parametrize("hq,T", CASES)
def test_page_edges(handles, hq, T):
    """New blocks that start, end or straddle a page boundary."""
    lens = [T, T + 1, 15, 16, 17, 18, 19, 20, 31, 32, 33, 34, 64, 65, 300, 1000]
    w = inputs.custom(lens, seed=60 + 4 * hq + T, device="cuda", gap_fraction=0.2, num_q_heads=hq, new_tokens=T)
    full_check(handles[hq], w, f"Hq={hq} T={T} page edges")


@pytest.mark.parametrize("hq,T", [(16, 4), (32, 2), (16, 8)])
def test_gains_at_a_4_byte_aligned_address(handles, hq, T):
    """The norm gains need only be 4-byte aligned (the ABI's requirement)."""
    w = inputs.custom([T, 17, 300, 33], seed=62, device="cuda", num_q_heads=hq, new_tokens=T)
    full_check(handles[hq], ph.gains_at_a_4_byte_offset(w), f"Hq={hq} T={T} gains at +4 bytes")


@pytest.mark.parametrize("hq,T", CASES)
def test_an_empty_cache_gives_the_first_token_its_own_v(handles, hq, T):
    """L = T: the first new token sees only itself, so its o is its v, bit for bit."""
    w = inputs.custom([T] * 5, seed=61, device="cuda", num_q_heads=hq, new_tokens=T)
    o, _ = full_check(handles[hq], w, f"Hq={hq} T={T} L=T")
    G = hq // 8
    v0 = w.qkv[:, 0, (hq + 8) * 128:].reshape(5, 8, 1, 128).expand(5, 8, G, 128).reshape(5, hq, 128)
    assert torch.equal(o[:, 0].contiguous().view(torch.int16), v0.contiguous().view(torch.int16))


@pytest.mark.parametrize("hq", [16, 32])
def test_one_token_through_the_tokens_entry_is_the_decode_step(handles, hq):
    """new_tokens = 1 is the one-token step: same o and cache bits."""
    w = inputs.custom([1, 17, 300, 45], seed=62, device="cuda", num_q_heads=hq)
    k1, v1 = w.k_cache.clone(), w.v_cache.clone()
    k2, v2 = w.k_cache.clone(), w.v_cache.clone()
    o1 = ph.run(handles[hq], w, DEV, k1, v1)
    o2 = ph.run(handles[hq], dataclasses.replace(w, qkv=w.qkv[:, None].contiguous()), DEV, k2, v2)
    assert handles[hq].check() == 0
    assert o2.shape == (4, 1, hq, 128)
    assert torch.equal(o1.view(torch.int16), o2[:, 0].view(torch.int16))
    assert torch.equal(k1.view(torch.int16), k2.view(torch.int16))
    assert torch.equal(v1.view(torch.int16), v2.view(torch.int16))


@pytest.mark.parametrize("hq,T", [(16, 4), (32, 2)])
def test_successive_one_token_steps_append_the_same_rows(handles, hq, T):
    """T one-token calls (L growing by one) leave the same cache bits as one
    T-token call, and the last one's o equals the T-token call's last row
    within the tolerance (two different kernels)."""
    lens = torch.tensor([T, 16, 17, 40, 333], dtype=torch.int32)
    w = inputs.custom(lens, seed=63, device="cuda", num_q_heads=hq, new_tokens=T)
    ks, vs = w.k_cache.clone(), w.v_cache.clone()
    for t in range(T):
        wt = dataclasses.replace(w, qkv=w.qkv[:, t].contiguous(), seq_lens=lens - (T - 1 - t))
        o_last = ph.run(handles[hq], wt, DEV, ks, vs)
    km, vm = w.k_cache.clone(), w.v_cache.clone()
    o = ph.run(handles[hq], w, DEV, km, vm)
    assert handles[hq].check() == 0
    assert torch.equal(ks.view(torch.int16), km.view(torch.int16))
    assert torch.equal(vs.view(torch.int16), vm.view(torch.int16))
    ref = ph.oracle_full(w, w.k_cache, w.v_cache)["o"]
    ph.assert_o_close(o, ref, f"Hq={hq} T={T}")
    ph.assert_o_close(o_last, ref[:, T - 1], f"Hq={hq} last of {T} single steps")


@pytest.mark.parametrize("grid", [1, 3, 148, 1024])
def test_split_count_does_not_change_the_result(grid):
    """Any cut of the key range, including cuts inside the new block (then two
    CTAs each append the new rows on their own pages)."""
    a = binding.DecodeAttention(device=0, grid_ctas=grid)
    w = inputs.custom([4, 16, 17, 18, 19, 300, 2000, 33], seed=64, device="cuda", gap_fraction=0.2, new_tokens=4)
    full_check(a, w, f"T=4 grid {grid}")
    a.close()


@pytest.mark.parametrize("hq,T", [(16, 9), (16, 20), (32, 9), (40, 4), (64, 5), (64, 3)])
def test_blocks_longer_than_one_launch(handles, hq, T):
    """A block of more than 16 query rows per kv head runs as the prefill: the
    same cache bits and the same causal attention as the oracle's single pass
    over the block."""
    lens = [T, T + 1, 16, 31, 33, 47, 48, 300, 1000]
    lens = [max(L, T) for L in lens]
    w = inputs.custom(lens, seed=72 + hq + T, device="cuda", gap_fraction=0.2, num_q_heads=hq, new_tokens=T)
    full_check(handles[hq], w, f"Hq={hq} T={T} in chunks")


def test_a_long_block_over_a_long_cache(handles):
    """64 new tokens (one prefill chunk of 128 rows at 16 heads) after up to 5000 cached ones, with positions."""
    w = inputs.custom([64, 100, 5064, 777], seed=73, device="cuda", gap_fraction=0.1, new_tokens=64)
    full_check(handles[16], w, "T=64 in chunks", positions=torch.tensor([0, 36, 9000, 713], dtype=torch.int32))


@pytest.mark.parametrize("grid", [1, 5, 148])
def test_split_count_does_not_change_the_result_wide(handles, grid):
    """The same with 8 new tokens at 16 heads (16 query rows per kv head)."""
    a = binding.DecodeAttention(device=0, grid_ctas=grid)
    w = inputs.custom([8, 16, 17, 23, 24, 25, 300, 2000, 33], seed=70, device="cuda", gap_fraction=0.2,
                      new_tokens=8)
    full_check(a, w, f"T=8 grid {grid}")
    a.close()


@pytest.mark.parametrize("hq,T", [(16, 8), (64, 2)])
def test_maximum_context_wide(handles, hq, T):
    w = inputs.custom([40960, 40955, 9], seed=71, device="cuda", stride=2560, new_tokens=T, num_q_heads=hq)
    full_check(handles[hq], w, f"Hq={hq} T={T} L=40960")


def test_positions_argument(handles):
    full_check(handles[16], inputs.custom([5, 100, 1234], seed=65, device="cuda", new_tokens=3),
               "T=3 positions", positions=torch.tensor([0, 7000, 40000], dtype=torch.int32))


def test_maximum_context(handles):
    w = inputs.custom([40960, 40959, 7], seed=66, device="cuda", stride=2560, new_tokens=4)
    full_check(handles[16], w, "T=4 L=40960")


@pytest.mark.parametrize("hq,T", [(16, 4), (16, 8), (16, 20), (64, 5), (32, 40)])
def test_locality_with_nan_in_unread_bytes(handles, hq, T):
    """The new tokens' rows (written, never read before), rows past a sequence,
    pages it does not own and table entries past its last page may hold
    anything (here NaN): o and the appended rows do not change. T * Hq / 8 > 16
    runs the prefill, whose stages also hold rows past a piece's last page."""
    attn = handles[hq]
    lens = [max(L, T) for L in [8, 12, 40, 16, 18, 70]]
    w = inputs.custom(lens, seed=67, device="cuda", pool_pages=24, stride=6, new_tokens=T, num_q_heads=hq)
    ka, va = w.k_cache.clone(), w.v_cache.clone()
    kb, vb = w.k_cache.clone(), w.v_cache.clone()
    bt2 = w.block_table.clone()
    used, slots = set(), []
    for b, L in enumerate(w.seq_lens.tolist()):
        n = (L + 15) // 16
        used.update(w.block_table[b, :n].tolist())
        for s in range(L - T, 16 * n):
            page, row = int(w.block_table[b, s // 16]), s % 16
            kb[page, row] = float("nan")
            vb[page, row] = float("nan")
            if s < L:
                slots.append((page, row))
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


@pytest.mark.parametrize("T", [4, 20])
def test_a_sequence_shorter_than_the_new_block_is_skipped(handles, T):
    """seq_lens[b] < T is out of range on the device: that sequence is skipped
    (its cache untouched), the others are computed, and the status says BOUNDS."""
    attn = handles[16]
    w = inputs.custom([40, 3, 30], seed=68, device="cuda", new_tokens=T)
    lens = w.seq_lens.clone()
    k, v = w.k_cache.clone(), w.v_cache.clone()
    k0, v0 = w.k_cache.clone(), w.v_cache.clone()
    o = ph.run(attn, w, DEV, k, v)
    assert attn.check() == binding.QDA_ERR_BOUNDS
    sampled_check(o, w, [0, 2], w.k_cache, w.v_cache, f"T={T} with a short sequence")
    page1 = int(w.block_table[1, 0])
    assert torch.equal(k[page1].view(torch.int16), k0[page1].view(torch.int16))
    assert torch.equal(v[page1].view(torch.int16), v0[page1].view(torch.int16))
    assert int(lens[1]) == 3
    assert attn.check() == 0


@pytest.mark.parametrize("hq,T", [(16, 20), (64, 5)])
def test_prefill_out_of_range_page_ids_are_not_dereferenced(handles, hq, T):
    """A block-table entry outside [0, num_pages) among a sequence's older
    pages: not copied, the status says BOUNDS, the other sequences are
    computed."""
    attn = handles[hq]
    w = inputs.custom([40, 70, 30], seed=69, device="cuda", pool_pages=16, stride=5, new_tokens=T, num_q_heads=hq)
    k, v = w.k_cache.clone(), w.v_cache.clone()
    bt = w.block_table.clone()
    bt[1, 1] = 16
    a = ph.device_args(w, DEV)
    o = attn(a["qkv"], a["q_norm_w"], a["k_norm_w"], a["seq_lens"], bt.to(DEV), k, v)
    assert attn.check() == binding.QDA_ERR_BOUNDS
    sampled_check(o, w, [0, 2], w.k_cache, w.v_cache, f"Hq={hq} T={T} bad page id")
    assert attn.check() == 0


def test_prefill_wait_timeout_is_reported_and_the_handle_recovers():
    """The prefill's bounded waits: a wait on a barrier nothing completes ends
    after the configured limit with QDA_ERR_TIMEOUT, the call's result is still
    right, and a new handle works."""
    a = binding.DecodeAttention(device=0, flags=binding.QDA_FLAG_INJECT_WAIT_TIMEOUT, wait_timeout_ns=2_000_000)
    w = inputs.custom([100, 40, 300], seed=74, device="cuda", new_tokens=20)
    k, v = w.k_cache.clone(), w.v_cache.clone()
    o = ph.run(a, w, DEV, k, v)
    assert a.check() == binding.QDA_ERR_TIMEOUT
    sampled_check(o, w, [0, 1, 2], w.k_cache, w.v_cache, "prefill timeout injection")
    a.close()
    b = binding.DecodeAttention(device=0)
    full_check(b, inputs.custom([100, 40, 300], seed=74, device="cuda", new_tokens=20), "prefill after timeout")
    b.close()


def test_host_side_errors(handles):
    w = inputs.custom([20, 30], seed=69, device="cuda", new_tokens=2)
    a = ph.device_args(w, DEV)
    call = lambda h, qkv, o: binding.qwen3_decode_attn_append_and_attend_tokens(
        h, qkv, a["q_norm_w"], a["k_norm_w"], a["seq_lens"], None, a["block_table"], w.k_cache, w.v_cache, o)
    small = binding.DecodeAttention(device=0, max_seq_len=8, max_pages_per_seq=8)
    qkv9 = torch.zeros((2, 9, 4096), dtype=torch.bfloat16, device=DEV)   # more new tokens than max_seq_len
    with pytest.raises(binding.QdaError) as e:
        call(small.handle, qkv9, torch.empty((2, 9, 16, 128), dtype=torch.bfloat16, device=DEV))
    assert e.value.code == binding.QDA_ERR_INVALID_ARG
    small.close()
    with pytest.raises(ValueError):   # several tokens are not taken by the one-token entry point
        binding.qwen3_decode_attn_append_and_attend(
            handles[16].handle, a["qkv"], a["q_norm_w"], a["k_norm_w"], a["seq_lens"], None, a["block_table"],
            w.k_cache, w.v_cache, torch.empty((2, 2, 16, 128), dtype=torch.bfloat16, device=DEV))
    assert handles[16].check() == 0


def full_size_check(attn, w, sample, label):
    k_pre, v_pre = w.k_cache.clone(), w.v_cache.clone()
    o = ph.run(attn, w, DEV, w.k_cache, w.v_cache)
    assert attn.check() == 0
    k_rows, v_rows, k64 = ph.oracle_appended_rows(w, k_pre, v_pre)
    k_exp, v_exp = ph.expected_cache(w, k_pre, v_pre, k_rows, v_rows)
    ph.assert_cache_equal(w.k_cache, w.v_cache, k_exp, v_exp, k64, w)
    del k_exp, v_exp
    return sampled_check(o, w, sample, k_pre, v_pre, label)


def sampled_check(o, w, sample, k_pre, v_pre, label):
    """o of the sequences `sample` against the oracle over those sequences
    alone (caches before the call): the gate, then the strict bound or, for
    tokens that took q as bf16, the bf16-q bound."""
    if ph.is_wide(w):
        ref, lens, bt = ph.oracle_sampled_qk(w, sample, k_pre, v_pre)
        ref["seq_lens"], ref["block_table"] = lens, bt
        sub = o[torch.as_tensor(sample)]
        max_abs, rel, _ = ph.o_errors(sub, ref["o"])
        assert max_abs <= ph.GATE_ABS and rel <= ph.GATE_REL, f"{label}: max abs {max_abs:.3g}, rel rms {rel:.3g}"
        flags = ph.wide_tokens(w)
        narrow = [t for t, f in enumerate(flags) if not f]
        if narrow:
            ph.assert_o_close(sub[:, narrow], ref["o"][:, narrow], label + " (two-term rows)")
        ph.emulated_bf16_q_check(sub, ref["q"], lens, bt, ref["k_cache"], ref["v_cache"], w.new_tokens, label,
                                 tokens=[t for t, f in enumerate(flags) if f])
        return max_abs, rel
    ref = ph.oracle_sampled(w, sample, k_pre, v_pre)
    return ph.assert_o_close(o[torch.as_tensor(sample)], ref, label)


@pytest.mark.parametrize("hq,T", CASES)
def test_config2_shape_full_size(handles, hq, T):
    w = inputs.config2("cuda", num_q_heads=hq, new_tokens=T)
    full_size_check(handles[hq], w, list(range(1, 32, 4)), f"cfg2 Hq={hq} T={T}")


def test_config4_shape_full_size(handles):
    w = inputs.config4("cuda", new_tokens=4)
    full_size_check(handles[16], w, [1, 2], "cfg4 T=4")


@pytest.mark.parametrize("hq,T", [(16, 130), (32, 70), (40, 30), (64, 40)])
def test_prefill_in_several_chunks(handles, hq, T):
    """Blocks of more than 128 query rows per kv head: several prefill launches
    (128 / G tokens each), each seeing the block's tokens up to its own."""
    lens = [T, T + 1, T + 15, T + 16, T + 17, T + 700, T + 1500]
    w = inputs.custom(lens, seed=90 + hq + T, device="cuda", gap_fraction=0.2, num_q_heads=hq, new_tokens=T)
    full_check(handles[hq], w, f"Hq={hq} T={T} prefill chunks")


def test_prefill_with_positions(handles):
    w = inputs.custom([33, 40, 2000, 600], seed=95, device="cuda", gap_fraction=0.1, num_q_heads=32, new_tokens=33)
    full_check(handles[32], w, "Hq=32 T=33 positions", positions=torch.tensor([0, 7, 4000, 100], dtype=torch.int32))


@pytest.mark.parametrize("hq,T", [(16, 16), (16, 64), (64, 16)])
def test_config2_shape_full_size_prefill(handles, hq, T):
    w = inputs.config2("cuda", num_q_heads=hq, new_tokens=T)
    full_size_check(handles[hq], w, list(range(2, 32, 5)), f"cfg2 Hq={hq} T={T} prefill")


def test_config4_shape_full_size_prefill(handles):
    w = inputs.config4("cuda", new_tokens=32)
    full_size_check(handles[16], w, [0, 3], "cfg4 T=32 prefill")
