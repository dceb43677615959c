"""Pins of the oracle's input_norm + attn.qkv_proj (the nodes that produce
the attention step's qkv row; Qwen3-0.6B Model Spec, "Compute-graph nodes":
input_norm rmsnorm H=1024 eps=1e-6, attn.qkv_proj linear K=1024 N=4096,
y[t,n] = sum_k x[t,k] w[n,k]). CPU only.

Each pin ties the oracle to something other than itself: float64 library
routines (torch rms_norm and linear; transformers' own Qwen3 RMSNorm and
q/k/v projections), closed forms, an exact invariance, and error returns.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from decode_attention_qk_b200 import inputs


def as64(bits_tensor):
    return bits_tensor.to(torch.float64)


def run(oracle_mod, x, g, w, eps=1e-6):
    return oracle_mod.input_norm_qkv_proj(inputs.bf16_bits(x), inputs.bf16_bits(g), inputs.bf16_bits(w), eps)


@pytest.mark.parametrize("hq", [16, 32])
def test_matches_torch_rms_norm_and_linear_in_float64(oracle_mod, hq):
    d = inputs.hidden_inputs(5, seed=1, num_q_heads=hq)
    out = run(oracle_mod, d["x"], d["input_norm_w"], d["w_qkv"])
    ref = F.linear(F.rms_norm(as64(d["x"]), (inputs.HIDDEN,), as64(d["input_norm_w"]), eps=1e-6), as64(d["w_qkv"]))
    assert out["y"].shape == (5, inputs.qkv_width(hq))
    err = np.abs(out["y"] - ref.numpy()).max() / np.abs(ref.numpy()).max()
    assert err <= 1e-12, err
    assert np.array_equal(out["bits"], oracle_mod.f64_to_bf16_rne(out["y"]))


def test_matches_transformers_qwen3_norm_and_projections(oracle_mod):
    """transformers' Qwen3 decoder layer as a library: input_layernorm, then
    q_proj | k_proj | v_proj; the fused weight is their rows stacked in that
    order. Its RMSNorm computes in float32 internally, hence the 1e-6 bound."""
    from transformers import Qwen3Config
    from transformers.models.qwen3 import modeling_qwen3
    cfg = Qwen3Config(hidden_size=1024, num_attention_heads=16, num_key_value_heads=8, head_dim=128,
                      intermediate_size=64, num_hidden_layers=1, rms_norm_eps=1e-6, vocab_size=32)
    layer = modeling_qwen3.Qwen3DecoderLayer(cfg, 0).to(torch.float64)
    d = inputs.hidden_inputs(6, seed=2)
    w = as64(d["w_qkv"])
    with torch.no_grad():
        layer.input_layernorm.weight.copy_(as64(d["input_norm_w"]))
        layer.self_attn.q_proj.weight.copy_(w[:2048])
        layer.self_attn.k_proj.weight.copy_(w[2048:3072])
        layer.self_attn.v_proj.weight.copy_(w[3072:])
        h = layer.input_layernorm(as64(d["x"])[None])
        ref = torch.cat([layer.self_attn.q_proj(h), layer.self_attn.k_proj(h), layer.self_attn.v_proj(h)], -1)[0]
    assert layer.self_attn.q_proj.bias is None
    out = run(oracle_mod, d["x"], d["input_norm_w"], d["w_qkv"])
    err = np.abs(out["y"] - ref.numpy()).max() / np.abs(ref.numpy()).max()
    assert err <= 1e-6, err


def test_closed_form_with_one_hot_weight_rows(oracle_mod):
    """w[n, k] = 1 at k = (7n + 3) mod K, else 0: y[b, n] = x[b, k] g[k] / r_b with
    r_b = sqrt(mean_k x[b,k]^2 + eps). A small constant row (x = 1e-3, where
    eps = 1e-6 weighs as much as the mean square) pins eps inside the root."""
    K, N = 1024, 4096
    d = inputs.hidden_inputs(3, seed=3)
    x = d["x"].clone()
    x[2] = 1e-3
    g = d["input_norm_w"]
    cols = (7 * np.arange(N) + 3) % K
    w = torch.zeros((N, K), dtype=torch.bfloat16)
    w[np.arange(N), cols] = 1.0
    out = run(oracle_mod, x, g, w)
    xs, gs = as64(x).numpy(), as64(g).numpy()
    for b in range(3):
        r = math.sqrt(float(np.mean(xs[b] ** 2)) + 1e-6)
        want = xs[b, cols] * gs[cols] / r
        assert np.allclose(out["y"][b], want, rtol=1e-15, atol=0), b
    c = float(as64(x[2, :1])[0])
    assert np.allclose(out["y"][2] / gs[cols], c / math.sqrt(c * c + 1e-6), rtol=1e-15)
    assert abs(c / math.sqrt(c * c + 1e-6) - 1 / math.sqrt(2)) < 1e-3


def test_zero_row_gives_zero(oracle_mod):
    d = inputs.hidden_inputs(2, seed=4)
    x = d["x"].clone()
    x[1] = 0
    out = run(oracle_mod, x, d["input_norm_w"], d["w_qkv"])
    assert np.all(out["y"][1] == 0.0) and np.all(np.isfinite(out["y"]))


def test_power_of_two_scaling_changes_no_bit_at_zero_eps(oracle_mod):
    """With eps = 0 the norm is scale-invariant (nnterp qwen3, RMSNorm scale
    invariance); scaling x by 2^12 is exact in binary, so every bit stays."""
    d = inputs.hidden_inputs(3, seed=5)
    a = run(oracle_mod, d["x"], d["input_norm_w"], d["w_qkv"], eps=0.0)
    b = run(oracle_mod, d["x"] * 4096, d["input_norm_w"], d["w_qkv"], eps=0.0)
    assert np.array_equal(a["y"], b["y"])


def test_rejects_bad_arguments(oracle_mod):
    d = inputs.hidden_inputs(1, seed=6)
    with pytest.raises(ValueError):
        oracle_mod.input_norm_qkv_proj(inputs.bf16_bits(d["x"]), inputs.bf16_bits(d["input_norm_w"]),
                                       inputs.bf16_bits(d["w_qkv"]), rms_eps=-1.0)
