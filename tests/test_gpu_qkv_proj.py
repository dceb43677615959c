"""Parity of input_norm + attn.qkv_proj (and of the attention fed by it) with
the float64 oracle, through the C ABI.

qkv is rounded once to bf16. The kernel's products are exact and its sums
are float: 2K terms x_k g_k W[n,k] / r (split in two exact halves), so the
sum's error is bounded by a small multiple of 2^-24 times S = sum_k |x_k g_k
W[n,k]| / r, not of |y| (the sum can cancel). The bound checked is
|qkv - y| <= ulp(y) + 2^-17 S for every element (one rounding of y to bf16
plus the float sum at 128x its per-operation error), and qkv equals the
oracle's rounding for all but 0.5% of elements.
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


def abs_sum(d):
    """S[b, n] = sum_k |x[b,k] g[k] W[n,k]| / r_b, in float64."""
    x = d["x"].double().cpu()
    g = d["input_norm_w"].double().cpu()
    w = d["w_qkv"].double().cpu()
    r = torch.sqrt((x * x).mean(-1, keepdim=True) + 1e-6)
    return ((x * g).abs() / r) @ w.abs().T


def check_qkv(got, ref, label, d):
    got = got.float().cpu().numpy().astype(np.float64)
    y, bits = ref["y"], ref["bits"]
    assert np.all(np.isfinite(got)), label
    bound = ulp(y) + 2.0 ** -17 * abs_sum(d).numpy()
    excess = np.abs(got - y) - bound
    assert np.all(excess <= 0), f"{label}: beyond the bound at {np.argwhere(excess > 0)[:5]}, by up to {excess.max():.3g}"
    off = float(np.mean(got != oracle.bf16_to_f64(bits)))
    assert off <= 0.005, f"{label}: {off:.4%} not the correctly rounded value"
    return off


def run_proj(attn, d):
    x, g, w = d["x"].to(DEV), d["input_norm_w"].to(DEV), d["w_qkv"].to(DEV)
    qkv = attn.qkv_proj(x, g, w)
    assert attn.check() == 0
    return qkv


@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 8, 9, 16, 17, 32, 33, 64, 65, 128, 129, 200, 256])
def test_parity_at_batch_sizes(handles, B):
    d = inputs.hidden_inputs(B, seed=100 + B)
    ref = oracle.input_norm_qkv_proj(inputs.bf16_bits(d["x"]), inputs.bf16_bits(d["input_norm_w"]),
                                     inputs.bf16_bits(d["w_qkv"]))
    check_qkv(run_proj(handles[16], d), ref, f"B={B}", d)


@pytest.mark.parametrize("B", [3, 24])
@pytest.mark.parametrize("hq,hidden", [(16, 2048), (32, 2560), (64, 5120)])
def test_parity_at_larger_sizes(handles, hq, hidden, B):
    """Qwen3-1.7B (hidden 2048), 4B (2560, 32 heads), 32B (5120, 64 heads);
    B = 3 runs the small-batch product with its K range in parts."""
    d = inputs.hidden_inputs(B, seed=hidden + B, hidden=hidden, num_q_heads=hq)
    ref = oracle.input_norm_qkv_proj(inputs.bf16_bits(d["x"]), inputs.bf16_bits(d["input_norm_w"]),
                                     inputs.bf16_bits(d["w_qkv"]))
    check_qkv(run_proj(handles[hq], d), ref, f"Hq={hq} hidden={hidden}", d)


def test_zero_and_tiny_rows(handles):
    d = inputs.hidden_inputs(3, seed=7)
    d["x"][1] = 0
    d["x"][2] = 1e-3   # the mean square equals eps here
    ref = oracle.input_norm_qkv_proj(inputs.bf16_bits(d["x"]), inputs.bf16_bits(d["input_norm_w"]),
                                     inputs.bf16_bits(d["w_qkv"]))
    qkv = run_proj(handles[16], d)
    assert torch.all(qkv[1].float() == 0)
    check_qkv(qkv, ref, "zero and tiny rows", d)


def test_attention_fed_by_the_projection(handles):
    """from_hidden = qkv_proj, then the attention step on that qkv: qkv as
    above; the cache bit for bit and o within the gate against the oracle's
    attention over the qkv the device produced."""
    attn = handles[16]
    lens = [1, 17, 300, 2000, 45, 4096]
    w = inputs.custom(lens, seed=8, device="cuda", gap_fraction=0.2)
    d = inputs.hidden_inputs(len(lens), seed=9)
    x, g, wq = d["x"].to(DEV), d["input_norm_w"].to(DEV), d["w_qkv"].to(DEV)
    k, v = w.k_cache.clone(), w.v_cache.clone()
    a = ph.device_args(w, DEV)
    o, qkv = attn.from_hidden(x, g, wq, a["q_norm_w"], a["k_norm_w"], a["seq_lens"], a["block_table"], k, v)
    assert attn.check() == 0
    ref_qkv = oracle.input_norm_qkv_proj(inputs.bf16_bits(d["x"]), inputs.bf16_bits(d["input_norm_w"]),
                                         inputs.bf16_bits(d["w_qkv"]))
    check_qkv(qkv, ref_qkv, "from_hidden qkv", d)
    import dataclasses
    w_dev = dataclasses.replace(w, qkv=qkv)
    ref = ph.oracle_full(w_dev, w.k_cache, w.v_cache)
    assert np.array_equal(inputs.bf16_bits(k), ref["k_cache"])
    assert np.array_equal(inputs.bf16_bits(v), ref["v_cache"])
    ph.assert_o_close(o, ref["o"], "from_hidden o")


@pytest.mark.parametrize("hq,hidden", [(32, 2560), (64, 5120)])
def test_attention_fed_by_the_projection_at_larger_sizes(handles, hq, hidden):
    """Qwen3-4B (hidden 2560, 32 heads) and 32B (hidden 5120, 64 heads) from the
    hidden state: the projection, then the tensor-core attention on its qkv."""
    attn = handles[hq]
    lens = [1, 33, 700, 17]
    w = inputs.custom(lens, seed=11 + hq, device="cuda", gap_fraction=0.2, num_q_heads=hq)
    d = inputs.hidden_inputs(len(lens), seed=12 + hq, hidden=hidden, num_q_heads=hq)
    x, g, wq = d["x"].to(DEV), d["input_norm_w"].to(DEV), d["w_qkv"].to(DEV)
    k, v = w.k_cache.clone(), w.v_cache.clone()
    a = ph.device_args(w, DEV)
    o, qkv = attn.from_hidden(x, g, wq, a["q_norm_w"], a["k_norm_w"], a["seq_lens"], a["block_table"], k, v)
    assert attn.check() == 0
    ref_qkv = oracle.input_norm_qkv_proj(inputs.bf16_bits(d["x"]), inputs.bf16_bits(d["input_norm_w"]),
                                         inputs.bf16_bits(d["w_qkv"]))
    check_qkv(qkv, ref_qkv, f"Hq={hq} from_hidden qkv", d)
    import dataclasses
    ref = ph.oracle_full(dataclasses.replace(w, qkv=qkv), w.k_cache, w.v_cache)
    assert np.array_equal(inputs.bf16_bits(k), ref["k_cache"])
    assert np.array_equal(inputs.bf16_bits(v), ref["v_cache"])
    ph.assert_o_close(o, ref["o"], f"Hq={hq} from_hidden o")


def test_host_side_errors(handles):
    attn = handles[16]
    d = inputs.hidden_inputs(4, seed=10)
    x, g, wq = d["x"].to(DEV), d["input_norm_w"].to(DEV), d["w_qkv"].to(DEV)
    qkv = torch.empty((4, 4096), dtype=torch.bfloat16, device=DEV)
    lib = binding.load_library()
    p = lambda t: binding._ptr(t)
    s = binding._stream(None, DEV)
    assert lib.qwen3_decode_attn_qkv_proj(attn.handle, p(x), p(g), p(wq), 1000, p(qkv), 4, s) == \
        binding.QDA_ERR_INVALID_ARG
    assert lib.qwen3_decode_attn_qkv_proj(attn.handle, p(x), p(g), p(wq), 1024, p(qkv), 0, s) == \
        binding.QDA_ERR_INVALID_ARG
    xo = torch.empty(4 * 1024 + 8, dtype=torch.bfloat16, device=DEV)[1:4 * 1024 + 1]   # 2-byte aligned only
    assert lib.qwen3_decode_attn_qkv_proj(attn.handle, binding._ptr(xo), p(g), p(wq), 1024, p(qkv), 4, s) == \
        binding.QDA_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        attn.qkv_proj(x, g, wq[:1000])
    assert attn.check() == 0
