"""The shortcuts the full-size parity tests take through the oracle (a
sub-batch over a compacted pool, or only the pages from the first new token
on) give what the oracle gives on the whole batch. CPU only."""
import numpy as np
import pytest
import torch

from decode_attention_qk_b200 import inputs
import parity_helpers as ph


@pytest.mark.parametrize("hq,T", [(16, 1), (16, 3), (32, 2)])
def test_appended_rows_from_the_tail_pages_match_the_whole_batch(hq, T):
    w = inputs.custom([T, 15, 16, 17, 18, 33, 70], seed=90 + T, gap_fraction=0.3, num_q_heads=hq, new_tokens=T)
    full = ph.oracle_full(w, w.k_cache, w.v_cache)
    k_rows, v_rows, k64 = ph.oracle_appended_rows(w, w.k_cache, w.v_cache)
    k_exp, v_exp = ph.expected_cache(w, w.k_cache, w.v_cache, k_rows, v_rows)
    assert np.array_equal(inputs.bf16_bits(k_exp), full["k_cache"])
    assert np.array_equal(inputs.bf16_bits(v_exp), full["v_cache"])
    assert np.array_equal(k64.reshape(full["k"].shape), full["k"])


@pytest.mark.parametrize("hq,T", [(16, 1), (16, 4), (40, 1)])
def test_sampled_sequences_match_the_whole_batch(hq, T):
    w = inputs.custom([T, 20, 47, 16, 100], seed=95, gap_fraction=0.5, num_q_heads=hq, new_tokens=T)
    full = ph.oracle_full(w, w.k_cache, w.v_cache)
    sample = [1, 4, 0]
    got = ph.oracle_sampled(w, sample, w.k_cache, w.v_cache)
    assert got.shape == full["o"][sample].shape
    assert np.array_equal(got, full["o"][sample])


def test_appended_rows_with_positions():
    w = inputs.custom([9, 31], seed=97, new_tokens=2, positions=[100, 5000])
    full = ph.oracle_full(w, w.k_cache, w.v_cache)
    k_rows, v_rows, _ = ph.oracle_appended_rows(w, w.k_cache, w.v_cache)
    k_exp, _ = ph.expected_cache(w, w.k_cache, w.v_cache, k_rows, v_rows)
    assert np.array_equal(inputs.bf16_bits(k_exp), full["k_cache"])
    assert not np.array_equal(inputs.bf16_bits(k_exp), ph.oracle_full(
        w, w.k_cache, w.v_cache, positions=torch.tensor([0, 0], dtype=torch.int32))["k_cache"])
