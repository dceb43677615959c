"""Parity of attn.o_proj (the attention step's consumer) with the float64
oracle, through the C ABI.

y is rounded once to bf16. The products of two bf16 values are exact and the
tensor cores sum them in float, so the error of a sum is bounded by a small
multiple of 2^-24 times S = sum_k |x_k W[n,k]|, not of |y| (the sum can
cancel). The bound checked is |y - y_ref| <= ulp(y_ref) + 2^-17 S for every
element, and y equals the oracle's rounding for all but 0.5% of elements.
"""
import numpy as np
import pytest
import torch

from decode_attention_qk_b200 import binding, inputs
import oracle
import parity_helpers as ph

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module")
def handles():
    from decode_attention_qk_b200 import build
    build.build_library()
    hs = {hq: binding.DecodeAttention(device=0, num_q_heads=hq) for hq in (16, 32, 64)}
    yield hs
    for h in hs.values():
        h.close()


def ulp(y):
    a = np.abs(y)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def check_y(got, x, w, label):
    ref = oracle.o_proj(inputs.bf16_bits(x), inputs.bf16_bits(w))
    got = got.float().cpu().numpy().astype(np.float64)
    y = ref["y"]
    assert np.all(np.isfinite(got)), label
    S = x.double().cpu().reshape(x.shape[0], -1).abs() @ w.double().cpu().abs().T
    excess = np.abs(got - y) - (ulp(y) + 2.0 ** -17 * S.numpy())
    assert np.all(excess <= 0), f"{label}: beyond the bound at {np.argwhere(excess > 0)[:5]}, by up to {excess.max():.3g}"
    off = float(np.mean(got != oracle.bf16_to_f64(ref["bits"])))
    assert off <= 0.005, f"{label}: {off:.4%} not the correctly rounded value"


@pytest.mark.parametrize("B", [1, 2, 3, 4, 7, 8, 9, 16, 32, 33, 64, 65, 128, 200, 256])
def test_parity_at_batch_sizes(handles, B):
    d = inputs.o_proj_inputs(B, seed=200 + B, device="cuda")
    y = handles[16].o_proj(d["x"], d["w_o"])
    assert handles[16].check() == 0
    check_y(y, d["x"], d["w_o"], f"B={B}")


@pytest.mark.parametrize("B", [3, 24])
@pytest.mark.parametrize("hq,hidden", [(16, 2048), (32, 2560), (64, 5120)])
def test_parity_at_larger_sizes(handles, hq, hidden, B):
    """Qwen3-1.7B (hidden 2048), 4B (2560, 32 heads), 32B (5120, 64 heads);
    B = 3 runs the small-batch product with its K range in parts."""
    d = inputs.o_proj_inputs(B, seed=hidden + hq + B, device="cuda", hidden=hidden, num_q_heads=hq)
    y = handles[hq].o_proj(d["x"], d["w_o"])
    assert handles[hq].check() == 0
    check_y(y, d["x"], d["w_o"], f"Hq={hq} hidden={hidden}")


def test_o_proj_directly_after_the_attention(handles):
    """The attention step, then o_proj on its o on the same stream (the
    projection's weight copies overlap the attention's end; it reads o only
    after the attention has completed): y against the oracle's o_proj of the
    o the device produced, which itself passes the attention parity check."""
    attn = handles[16]
    lens = [1, 17, 300, 2000, 45, 4096, 40960]
    w = inputs.custom(lens, seed=21, device="cuda", gap_fraction=0.2)
    d = inputs.o_proj_inputs(len(lens), seed=22, device="cuda")
    k, v = w.k_cache.clone(), w.v_cache.clone()
    o = ph.run(attn, w, DEV, k, v)
    y = attn.o_proj(o, d["w_o"])
    assert attn.check() == 0
    ref = ph.oracle_full(w, w.k_cache, w.v_cache)
    ph.assert_o_close(o, ref["o"], "attention o")
    check_y(y, o, d["w_o"], "o_proj after the attention")


def test_host_side_errors(handles):
    attn = handles[16]
    d = inputs.o_proj_inputs(4, seed=23, device="cuda")
    y = torch.empty((4, 1024), dtype=torch.bfloat16, device=DEV)
    lib = binding.load_library()
    p = binding._ptr
    s = binding._stream(None, DEV)
    assert lib.qwen3_decode_attn_o_proj(attn.handle, p(d["x"]), p(d["w_o"]), 1000, p(y), 4, s) == \
        binding.QDA_ERR_INVALID_ARG
    assert lib.qwen3_decode_attn_o_proj(attn.handle, p(d["x"]), p(d["w_o"]), 1024, p(y), 0, s) == \
        binding.QDA_ERR_INVALID_ARG
    assert lib.qwen3_decode_attn_o_proj(attn.handle, p(d["x"]), p(d["w_o"]), 1024, p(y), 257, s) == \
        binding.QDA_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        attn.o_proj(d["x"], d["w_o"][:, :1000])
    assert attn.check() == 0
