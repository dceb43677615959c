"""Pins of the oracle's attn.o_proj (the node that consumes the attention
step's output; Qwen3-0.6B Model Spec, "Compute-graph nodes": attn.o_proj
linear K=2048 N=1024, y[t,n] = sum_k x[t,k] w[n,k]; "Tensors of the main
nodes": attn.core's o [B, 16, 128] and attn.o_proj's x [T, 2048]). CPU only.

Each pin ties the oracle to something other than itself: the float64 library
routine (torch linear), transformers' own Qwen3 attention o_proj with the
reshape it applies to the heads, a one-hot closed form, and error returns.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from decode_attention_qk_b200 import inputs


def as64(t):
    return t.to(torch.float64)


def run(oracle_mod, x, w):
    return oracle_mod.o_proj(inputs.bf16_bits(x), inputs.bf16_bits(w))


@pytest.mark.parametrize("hq,hidden", [(16, 1024), (32, 2560)])
def test_matches_torch_linear_in_float64(oracle_mod, hq, hidden):
    d = inputs.o_proj_inputs(5, seed=1, hidden=hidden, num_q_heads=hq)
    out = run(oracle_mod, d["x"], d["w_o"])
    ref = F.linear(as64(d["x"]), as64(d["w_o"])).numpy()
    assert out["y"].shape == (5, hidden)
    assert np.abs(out["y"] - ref).max() / np.abs(ref).max() <= 1e-12
    assert np.array_equal(out["bits"], oracle_mod.f64_to_bf16_rne(out["y"]))


def test_matches_transformers_qwen3_attention_o_proj(oracle_mod):
    """transformers' Qwen3 attention as a library: its o_proj is a bias-free
    Linear(16 * 128 -> 1024) applied to the heads' outputs reshaped from
    [..., 16, 128] to [..., 2048] (head-major), which is the row layout the
    oracle reads o in."""
    from transformers import Qwen3Config
    from transformers.models.qwen3 import modeling_qwen3
    cfg = Qwen3Config(hidden_size=1024, num_attention_heads=16, num_key_value_heads=8, head_dim=128,
                      intermediate_size=64, num_hidden_layers=1, rms_norm_eps=1e-6, vocab_size=32)
    attn = modeling_qwen3.Qwen3Attention(cfg, 0).to(torch.float64)
    assert attn.o_proj.bias is None
    assert tuple(attn.o_proj.weight.shape) == (1024, 2048)
    d = inputs.o_proj_inputs(4, seed=2)
    heads = as64(d["x"]).reshape(4, 16, 128)       # o [B, 16, 128]
    with torch.no_grad():
        attn.o_proj.weight.copy_(as64(d["w_o"]))
        ref = attn.o_proj(heads.reshape(4, -1))    # the reshape the attention module applies
    out = oracle_mod.o_proj(inputs.bf16_bits(d["x"].reshape(4, 16, 128)), inputs.bf16_bits(d["w_o"]))
    assert np.abs(out["y"] - ref.numpy()).max() / np.abs(ref.numpy()).max() <= 1e-12


def test_closed_form_with_one_hot_weight_rows(oracle_mod):
    """w[n, k] = 1 at k = (5n + 1) mod K, else 0: y[b, n] = x[b, k] exactly, so
    the rounded output has x's bits."""
    K, N = 2048, 1024
    d = inputs.o_proj_inputs(3, seed=3)
    cols = (5 * np.arange(N) + 1) % K
    w = torch.zeros((N, K), dtype=torch.bfloat16)
    w[np.arange(N), cols] = 1.0
    out = run(oracle_mod, d["x"], w)
    xb = inputs.bf16_bits(d["x"])
    assert np.array_equal(out["bits"], xb[:, cols])
    assert np.array_equal(out["y"], oracle_mod.bf16_to_f64(xb[:, cols]))


def test_linear_in_x(oracle_mod):
    """y(2x) = 2 y(x) exactly (scaling by a power of two is exact), and a zero row gives 0."""
    d = inputs.o_proj_inputs(3, seed=4)
    x = d["x"].clone()
    x[1] = 0
    a = run(oracle_mod, x, d["w_o"])
    b = run(oracle_mod, x * 2, d["w_o"])
    assert np.array_equal(b["y"], 2 * a["y"])
    assert np.all(a["y"][1] == 0.0)


def test_rejects_bad_arguments(oracle_mod):
    d = inputs.o_proj_inputs(1, seed=5)
    with pytest.raises(AssertionError):
        oracle_mod.o_proj(inputs.bf16_bits(d["x"]), inputs.bf16_bits(d["w_o"][:, :100]))
