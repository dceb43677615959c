"""Pins of the float64 oracle to facts that do not come from the oracle itself.

Each test ties one oracle function to a closed form, an identity the pages
prove, a library routine run as an independent implementation, or brute force
on a tiny input. The pages print no worked input -> output example of the
step, so no end-to-end value is pinned by the pages directly; together these
pins are chosen so that a dropped term, a wrong sign, a misplaced epsilon, a
wrong head mapping or a transposed operand fails at least one of them.

Citations name the page and its section:
  Spec     = Qwen3-0.6B Model Spec (docs.theformalera.com/models/qwen3-0-6b)
  nnterp   = nnterp encyclopedia, qwen3 (ndif-team.github.io/nnterp/encyclopedia/qwen3)
  Models   = Supported models (docs.theformalera.com/models/index), "Facts proved about the specs"
  Conform  = Model conformance (docs.theformalera.com/conformance/overview)
"""
import json
import math
import os

import numpy as np
import pytest
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
SPEC = {k: v["value"] for k, v in json.load(open(os.path.join(HERE, "golden", "qwen3_0_6b_spec.json"))).items()
        if not k.startswith("_")}
D = SPEC["head_dim"]
THETA = SPEC["rope_theta"]
EPS = SPEC["rms_norm_eps"]
pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def rng(seed=0):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------
# bf16 conversions
# ----------------------------------------------------------------------------

def _bf16_table():
    """All finite non-negative bf16 values, from their bit patterns, by numpy."""
    bits = np.arange(0, 0x7F80, dtype=np.uint32)           # +0 .. largest finite
    return (bits << 16).view(np.float32).astype(np.float64), bits.astype(np.uint16)


def test_bf16_widening_known_patterns(oracle_mod):
    pats = np.array([0x3F80, 0xC000, 0x0001, 0x0080, 0x7F7F, 0x7F80, 0xFF80, 0x8000], dtype=np.uint16)
    want = [1.0, -2.0, 2.0 ** -133, 2.0 ** -126, (2 - 2 ** -7) * 2.0 ** 127, math.inf, -math.inf, -0.0]
    got = oracle_mod.bf16_to_f64(pats)
    for g, w in zip(got, want):
        assert g == w and math.copysign(1, g) == math.copysign(1, w)


def test_bf16_rne_brute_force_nearest(oracle_mod):
    """Every result is the nearest bf16 value; ties go to the even pattern."""
    vals, bits = _bf16_table()
    r = rng(1)
    x = np.concatenate([
        r.standard_normal(20000) * 10.0 ** r.integers(-6, 6, 20000),
        r.uniform(2.0 ** -140, 2.0 ** -120, 2000),          # subnormal range
        r.uniform(1e37, 3.39e38, 2000),                      # top of the range
    ])
    # exact midpoints between neighbours, and points just off them
    i = r.integers(1, len(vals) - 2, 4000)
    mids = (vals[i] + vals[i + 1]) / 2
    x = np.concatenate([x, mids, np.nextafter(mids, np.inf), np.nextafter(mids, -np.inf)])
    got = oracle_mod.f64_to_bf16_rne(x)
    a = np.abs(x)
    j = np.clip(np.searchsorted(vals, a), 1, len(vals) - 1)
    lo, hi = vals[j - 1], vals[j]
    pick_hi = (a - lo > hi - a) | ((a - lo == hi - a) & (bits[j] % 2 == 0))
    want = np.where(pick_hi, bits[j], bits[j - 1]) | np.where(x < 0, 0x8000, 0).astype(np.uint16)
    assert np.array_equal(got, want.astype(np.uint16))


def test_bf16_rne_is_not_double_rounded(oracle_mod):
    # 1 + 2^-8 + 2^-30 lies above the midpoint between 1 and 1 + 2^-7, so it
    # rounds up; going through float first would land on the midpoint and tie
    # down to 1.0.
    x = np.array([1 + 2.0 ** -8 + 2.0 ** -30, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8 + 2.0 ** -30)])
    assert list(oracle_mod.f64_to_bf16_rne(x)) == [0x3F81, 0x3F80, 0x3F82, 0xBF81]


def test_bf16_rne_special_values(oracle_mod):
    x = np.array([0.0, -0.0, math.inf, -math.inf, math.nan, 3.39e38, 3.40e38, 2.0 ** -134, 2.0 ** -134 * 3])
    got = list(oracle_mod.f64_to_bf16_rne(x))
    assert got[:4] == [0x0000, 0x8000, 0x7F80, 0xFF80]
    assert (got[4] & 0x7F80) == 0x7F80 and (got[4] & 0x7F) != 0     # a NaN
    assert got[5] == 0x7F7F and got[6] == 0x7F80                    # largest finite / overflow
    assert got[7] == 0x0000 and got[8] == 0x0002                    # half the smallest subnormal ties to 0


# ----------------------------------------------------------------------------
# attn.qk_norm (Spec, "Compute-graph nodes", rmsnorm / attn.qk_norm rows)
# ----------------------------------------------------------------------------

def test_rmsnorm_closed_form_rms(oracle_mod):
    """With w = 1, RMS(y) = sqrt(m / (m + eps)) where m = mean(x^2)."""
    x = rng(2).standard_normal(D) * 0.01
    y = oracle_mod.rmsnorm(x, np.ones(D), EPS)
    m = float(np.mean(x * x))
    assert math.isclose(math.sqrt(float(np.mean(y * y))), math.sqrt(m / (m + EPS)), rel_tol=1e-14)


def test_rmsnorm_epsilon_inside_the_root(oracle_mod):
    # x = 1e-3 everywhere: mean(x^2) = 1e-6 = eps, so y = 1e-3 / sqrt(2e-6) = 1/sqrt(2).
    # With eps outside the root y would be 1e-3 / (1e-3 + 1e-6) ~ 0.999.
    y = oracle_mod.rmsnorm(np.full(D, 1e-3), np.ones(D), EPS)
    assert np.allclose(y, 1 / math.sqrt(2), rtol=1e-14, atol=0)


def test_rmsnorm_scale_invariance_and_gain(oracle_mod):
    """nnterp, "Queries and keys are normed per head": the norm undoes the input's scale."""
    r = rng(3)
    x, w = r.standard_normal(D), 1 + r.uniform(-0.5, 0.5, D)
    y1 = oracle_mod.rmsnorm(x, w, EPS)
    y2 = oracle_mod.rmsnorm(1e4 * x, w, EPS)          # eps / c^2 -> 1e-14
    y0 = oracle_mod.rmsnorm(x, w, 0.0)
    assert np.allclose(y2, y0, rtol=1e-12, atol=0)
    assert not np.allclose(y1, y0, rtol=1e-9, atol=0)  # eps does act at scale 1
    assert np.allclose(oracle_mod.rmsnorm(x, np.ones(D), EPS) * w, y1, rtol=1e-15, atol=0)


def test_rmsnorm_zero_input(oracle_mod):
    """nnterp, "No projection has a bias": zero input gives zero queries and keys."""
    assert np.array_equal(oracle_mod.rmsnorm(np.zeros(D), np.ones(D), EPS), np.zeros(D))


def test_rmsnorm_matches_torch_library(oracle_mod):
    r = rng(4)
    for _ in range(20):
        x, w = r.standard_normal(D) * r.uniform(0.01, 100), 1 + r.uniform(-0.5, 0.5, D)
        ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (D,), torch.from_numpy(w), EPS).numpy()
        got = oracle_mod.rmsnorm(x, w, EPS)
        assert np.max(np.abs(got - ref)) / np.max(np.abs(ref)) <= 1e-15


def test_rmsnorm_tiled_equals_untiled(oracle_mod):
    """Models, rmsNormTiled_eq: summing the squares block by block gives the same norm."""
    r = rng(5)
    x, w = r.standard_normal(D), 1 + r.uniform(-0.5, 0.5, D)
    got = oracle_mod.rmsnorm(x, w, EPS)
    for block in (1, 4, 16, 32, 128):
        ss = sum(float(np.sum(x[i:i + block] ** 2)) for i in range(0, D, block))
        ref = x / math.sqrt(ss / D + EPS) * w
        assert np.allclose(got, ref, rtol=1e-14, atol=0)


# ----------------------------------------------------------------------------
# attn.rope (Spec, "Compute-graph nodes", attn.rope row)
# ----------------------------------------------------------------------------

def test_rope_position_zero_is_identity(oracle_mod):
    x = rng(6).standard_normal(D)
    assert np.array_equal(oracle_mod.rope(x, 0, THETA), x)


def test_rope_closed_form_unit_vectors(oracle_mod):
    """Pair i is (x_i, x_{i+64}), rotated by pos * theta^(-2i/128)."""
    for i in (0, 1, 17, 63):
        for pos in (1, 5, 40959):
            a = pos * THETA ** (-2.0 * i / D)
            e = np.zeros(D)
            e[i] = 1.0
            y = oracle_mod.rope(e, pos, THETA)
            want = np.zeros(D)
            want[i], want[i + 64] = math.cos(a), math.sin(a)
            assert np.allclose(y, want, rtol=0, atol=1e-15)
            e = np.zeros(D)
            e[i + 64] = 1.0
            y = oracle_mod.rope(e, pos, THETA)
            want = np.zeros(D)
            want[i], want[i + 64] = -math.sin(a), math.cos(a)
            assert np.allclose(y, want, rtol=0, atol=1e-15)


def test_rope_isometry(oracle_mod):
    """Models, rope_isometry: RoPE preserves inner products (and norms)."""
    r = rng(7)
    q, k = r.standard_normal(D), r.standard_normal(D)
    for pos in (1, 77, 4096, 40959):
        rq, rk = oracle_mod.rope(q, pos, THETA), oracle_mod.rope(k, pos, THETA)
        assert math.isclose(float(rq @ rk), float(q @ k), rel_tol=1e-12)
        assert math.isclose(float(np.linalg.norm(rq)), float(np.linalg.norm(q)), rel_tol=1e-14)


def test_rope_relative_positions(oracle_mod):
    """Models, rope_relative: <R_p q, R_p' k> = <R_(p-p') q, k>."""
    r = rng(8)
    q, k = r.standard_normal(D), r.standard_normal(D)
    for p, pp in ((5, 3), (100, 0), (2048, 2047), (40959, 17), (3, 5)):
        lhs = float(oracle_mod.rope(q, p, THETA) @ oracle_mod.rope(k, pp, THETA))
        rhs = float(oracle_mod.rope(q, p - pp, THETA) @ k)
        assert math.isclose(lhs, rhs, rel_tol=1e-9, abs_tol=1e-9)


def test_rope_matches_transformers_convention(oracle_mod):
    """The rotation direction matches the official implementation's RoPE.

    The Spec page states the official transformers Qwen3ForCausalLM agrees with
    the spec ("Conformance"); its rotary embedding module and
    apply_rotary_pos_emb are run here as a library. Its cos/sin are computed
    in float32, hence the tolerance; a wrong direction is off by O(1).
    """
    mq = pytest.importorskip("transformers.models.qwen3.modeling_qwen3")
    from transformers import Qwen3Config
    cfg = Qwen3Config(hidden_size=1024, num_attention_heads=16, num_key_value_heads=8, head_dim=D,
                      max_position_embeddings=40960,
                      rope_parameters={"rope_type": "default", "rope_theta": THETA})
    emb = mq.Qwen3RotaryEmbedding(cfg)
    r = rng(9)
    positions = torch.tensor([[0, 1, 2, 9, 33, 100, 511]])
    x = torch.from_numpy(r.standard_normal((1, 1, positions.shape[1], D)))
    cos, sin = emb(x.float(), positions)
    ref, _ = mq.apply_rotary_pos_emb(x, x, cos.double(), sin.double())
    for t, pos in enumerate(positions[0].tolist()):
        got = oracle_mod.rope(x[0, 0, t].numpy(), pos, THETA)
        assert np.allclose(got, ref[0, 0, t].numpy(), rtol=0, atol=2e-4)


# ----------------------------------------------------------------------------
# attn.core (Spec, "Compute-graph nodes", attn.core row: decodeGQA)
# ----------------------------------------------------------------------------

def _bits(a):
    return np.asarray(a).astype(np.float32).view(np.uint32).__rshift__(16).astype(np.uint16)


def _small_cache(pages, r):
    kc = _bits(r.standard_normal((pages, 16, 8, D)))
    vc = _bits(r.standard_normal((pages, 16, 8, D)))
    return kc, vc


def test_decode_head_single_position_returns_v(oracle_mod):
    r = rng(10)
    kc, vc = _small_cache(2, r)
    o = oracle_mod.decode_head(r.standard_normal(D), 1, np.array([1, 0], np.int32), kc, vc, 3)
    assert np.array_equal(o, oracle_mod.bf16_to_f64(vc[1, 0, 3]))


def test_decode_head_weights_sum_to_one(oracle_mod):
    """Models, attnWeights_distribution: with every v = 1 the output is exactly 1."""
    r = rng(11)
    kc, _ = _small_cache(3, r)
    vc = np.full_like(kc, 0x3F80)
    o = oracle_mod.decode_head(r.standard_normal(D) * 3, 41, np.array([2, 0, 1], np.int32), kc, vc, 5)
    assert np.allclose(o, 1.0, rtol=0, atol=1e-14)


def test_decode_head_equal_keys_and_zero_query_give_mean_v(oracle_mod):
    """nnterp, "An edit to q_proj.output is renormalized": a zero query attends uniformly."""
    r = rng(12)
    kc, vc = _small_cache(2, r)
    bt = np.array([1, 0], np.int32)
    L = 23
    rows = [(bt[t // 16], t % 16) for t in range(L)]
    mean_v = np.mean([oracle_mod.bf16_to_f64(vc[p, s, 2]) for p, s in rows], axis=0)
    o0 = oracle_mod.decode_head(np.zeros(D), L, bt, kc, vc, 2)
    assert np.allclose(o0, mean_v, rtol=0, atol=1e-14)
    kc_eq = kc.copy()
    for p, s in rows:
        kc_eq[p, s, 2] = kc[1, 0, 2]
    o1 = oracle_mod.decode_head(r.standard_normal(D), L, bt, kc_eq, vc, 2)
    assert np.allclose(o1, mean_v, rtol=0, atol=1e-14)


def test_decode_head_shift_invariance(oracle_mod):
    """Models, softmax_shift: a key component shared by every position cancels."""
    r = rng(13)
    L = 30
    small = r.integers(-8, 9, (2, 16, 8, D)).astype(np.float64)   # exact in bf16
    shared = r.integers(-8, 9, D).astype(np.float64)
    kc = _bits(small)
    kc_shift = _bits(small + shared)
    _, vc = _small_cache(2, r)
    q = r.standard_normal(D) * 0.05
    bt = np.array([0, 1], np.int32)
    o = oracle_mod.decode_head(q, L, bt, kc, vc, 4)
    o_shift = oracle_mod.decode_head(q, L, bt, kc_shift, vc, 4)
    assert np.allclose(o, o_shift, rtol=1e-12, atol=1e-13)


def test_decode_head_matches_brute_force_softmax(oracle_mod):
    r = rng(14)
    kc, vc = _small_cache(3, r)
    bt = np.array([2, 0, 1], np.int32)
    q = r.standard_normal(D)
    L = 37
    K = np.stack([oracle_mod.bf16_to_f64(kc[bt[t // 16], t % 16, 6]) for t in range(L)])
    V = np.stack([oracle_mod.bf16_to_f64(vc[bt[t // 16], t % 16, 6]) for t in range(L)])
    s = K @ q / math.sqrt(128)
    w = np.exp(s) / np.sum(np.exp(s))
    assert np.allclose(oracle_mod.decode_head(q, L, bt, kc, vc, 6), w @ V, rtol=1e-13, atol=1e-14)


# ----------------------------------------------------------------------------
# the whole step
# ----------------------------------------------------------------------------

def _workload(seq_lens, seed=0, extra_pages=2, stride=None):
    from decode_attention_qk_b200 import inputs
    w = inputs.custom(seq_lens, seed=seed, stride=stride,
                      pool_pages=int(inputs.pages_for(torch.tensor(seq_lens)).sum()) + extra_pages)
    return dict(qkv=inputs.bf16_bits(w.qkv), q_norm_w=inputs.bf16_bits(w.q_norm_w),
                k_norm_w=inputs.bf16_bits(w.k_norm_w), seq_lens=w.seq_lens.numpy(),
                block_table=w.block_table.numpy(), k_cache=inputs.bf16_bits(w.k_cache),
                v_cache=inputs.bf16_bits(w.v_cache))


def test_step_matches_torch_sdpa_with_gqa(oracle_mod):
    """Dense brute force: scaled_dot_product_attention(enable_gqa=True) in float64
    over the gathered post-append cache, with the oracle's own q."""
    w = _workload([1, 5, 16, 17, 40], seed=21)
    out = oracle_mod.append_and_attend(**w, want_qk=True)
    kc, vc = out["k_cache"], out["v_cache"]
    for b, L in enumerate(w["seq_lens"].tolist()):
        bt = w["block_table"][b]
        K = np.stack([oracle_mod.bf16_to_f64(kc[bt[t // 16], t % 16]) for t in range(L)], axis=1)
        V = np.stack([oracle_mod.bf16_to_f64(vc[bt[t // 16], t % 16]) for t in range(L)], axis=1)
        q = torch.from_numpy(out["q"][b])[None, :, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, torch.from_numpy(K)[None], torch.from_numpy(V)[None], enable_gqa=True)[0, :, 0]
        assert np.max(np.abs(out["o"][b] - ref.numpy())) <= 1e-9 * np.max(np.abs(ref.numpy()))


def test_step_append_touches_only_the_new_slots(oracle_mod):
    """Brute force over the whole cache: only slot L-1 of each sequence changes,
    and it holds bf16_rne(new k) and the bits of v from the qkv row."""
    w = _workload([3, 16, 17, 32, 33], seed=22, extra_pages=3)
    out = oracle_mod.append_and_attend(**w, want_qk=True)
    kc0, vc0 = w["k_cache"], w["v_cache"]
    mask = np.zeros(kc0.shape[:2], dtype=bool)
    for b, L in enumerate(w["seq_lens"].tolist()):
        page, row = w["block_table"][b][(L - 1) // 16], (L - 1) % 16
        mask[page, row] = True
        assert np.array_equal(out["k_cache"][page, row], oracle_mod.f64_to_bf16_rne(out["k"][b]))
        assert np.array_equal(out["v_cache"][page, row], w["qkv"][b, 3072:].reshape(8, 128))
    assert np.array_equal(out["k_cache"][~mask], kc0[~mask])
    assert np.array_equal(out["v_cache"][~mask], vc0[~mask])


def test_step_qkv_split_and_new_k_closed_form(oracle_mod):
    """q | k | v order of the fused row (Spec attn.qkv_proj N=4096 = 2048+1024+1024;
    nnterp "Queries and keys are normed per head"): with L = 1 the position is 0, so
    the appended k is bf16(x / sqrt(mean(x^2) + eps) * w) of the k slice, and o = v."""
    w = _workload([1, 1], seed=23)
    out = oracle_mod.append_and_attend(**w)
    wk = oracle_mod.bf16_to_f64(w["k_norm_w"])
    for b in range(2):
        page = w["block_table"][b][0]
        for j in range(8):
            x = oracle_mod.bf16_to_f64(w["qkv"][b, 2048 + 128 * j:2048 + 128 * (j + 1)])
            want = x / math.sqrt(float(np.mean(x * x)) + EPS) * wk
            assert np.array_equal(out["k_cache"][page, 0, j], oracle_mod.f64_to_bf16_rne(want))
            v = oracle_mod.bf16_to_f64(w["qkv"][b, 3072 + 128 * j:3072 + 128 * (j + 1)])
            assert np.array_equal(out["o"][b, 2 * j], v) and np.array_equal(out["o"][b, 2 * j + 1], v)


def test_step_zero_query_slice_attends_uniformly(oracle_mod):
    """nnterp, "An edit to q_proj.output is renormalized": zeroing a head's slice gives
    a zero query and that head attends uniformly over the prefix."""
    w = _workload([29], seed=24)
    w["qkv"][0, 128 * 5:128 * 6] = 0
    out = oracle_mod.append_and_attend(**w)
    bt, vc = w["block_table"][0], out["v_cache"]
    mean_v = np.mean([oracle_mod.bf16_to_f64(vc[bt[t // 16], t % 16, 2]) for t in range(29)], axis=0)
    assert np.allclose(out["o"][0, 5], mean_v, rtol=0, atol=1e-14)


def test_step_gqa_head_mapping(oracle_mod):
    """nnterp, "Grouped-query attention": an edit to kv head j reaches q heads 2j, 2j+1 only."""
    w = _workload([20, 9], seed=25)
    base = oracle_mod.append_and_attend(**w)["o"]
    for j in (0, 3, 7):
        w2 = dict(w)
        vc = w["v_cache"].copy()
        for b, L in enumerate(w["seq_lens"].tolist()):
            for t in range(L - 1):
                vc[w["block_table"][b][t // 16], t % 16, j] ^= 0x0100
        w2["v_cache"] = vc
        o = oracle_mod.append_and_attend(**w2)["o"]
        changed = [h for h in range(16) if not np.array_equal(o[:, h], base[:, h])]
        assert changed == [2 * j, 2 * j + 1]


def test_step_locality(oracle_mod):
    """Models, attnHead_local / forward_causal and Conform "Causality": bytes the step
    must not read (other pages, rows at or past seq_len, table entries past the last
    page) do not change o at all."""
    w = _workload([7, 12], seed=26, extra_pages=3, stride=3)
    base = oracle_mod.append_and_attend(**w)
    w2 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in w.items()}
    used = set()
    for b, L in enumerate(w["seq_lens"].tolist()):
        page = w["block_table"][b][0]
        used.add(page)
        w2["k_cache"][page, L:] ^= 0x1234
        w2["v_cache"][page, L:] ^= 0x4321
        w2["block_table"][b][1:] = 10 ** 6           # never read
    for p in range(w["k_cache"].shape[0]):
        if p not in used:
            w2["k_cache"][p] = 0x7FC0                 # NaN pages
            w2["v_cache"][p] = 0x7FC0
    got = oracle_mod.append_and_attend(**w2)
    assert np.array_equal(got["o"], base["o"])


def test_step_positions_argument(oracle_mod):
    """Explicit positions equal to seq_len-1 give the default result; others rotate."""
    w = _workload([9, 40], seed=27)
    a = oracle_mod.append_and_attend(**w)["o"]
    b = oracle_mod.append_and_attend(**w, positions=w["seq_lens"] - 1)["o"]
    c = oracle_mod.append_and_attend(**w, positions=w["seq_lens"] + 100)["o"]
    assert np.array_equal(a, b) and not np.allclose(a, c)


def test_step_rejects_out_of_range_indices(oracle_mod):
    w = _workload([5, 18], seed=28)
    for bad in ({"seq_lens": np.array([0, 18], np.int32)},
                {"seq_lens": np.array([5, 40961], np.int32)},
                {"seq_lens": np.array([5, 10 ** 4], np.int32)}):      # past the table row
        with pytest.raises(ValueError):
            oracle_mod.append_and_attend(**{**w, **bad})
    bt = w["block_table"].copy()
    bt[1, 1] = w["k_cache"].shape[0]
    with pytest.raises(ValueError):
        oracle_mod.append_and_attend(**{**w, "block_table": bt})


def test_parameter_count_fixes_shared_head_gains():
    """Spec "At a glance" (596,049,920 parameters) decomposed with the Spec's node
    shapes: it balances only with one [128] q_norm and one [128] k_norm gain per layer
    (shared by every head) and no biases, the reading the oracle takes."""
    H, I, V, N = SPEC["hidden_size"], SPEC["intermediate_size"], SPEC["vocab_size"], SPEC["num_hidden_layers"]
    per_layer = (H * SPEC["qkv_proj_out"] + SPEC["o_proj_in"] * H    # attention projections
                 + 2 * D                                              # q_norm, k_norm gains
                 + H * 2 * I + I * H                                  # gate_up, down
                 + 2 * H)                                             # input / post-attention norms
    assert V * H + N * per_layer + H == SPEC["parameters"]
    per_head_gains = per_layer - 2 * D + (SPEC["num_attention_heads"] + SPEC["num_key_value_heads"]) * D
    assert V * H + N * per_head_gains + H != SPEC["parameters"]


# ----------------------------------------------------------------------------
# larger Qwen3 sizes: 32, 40 or 64 query heads over the same 8 kv heads
# (nnterp qwen3, "Grouped-query attention, with 128-wide heads on every size")

@pytest.mark.parametrize("num_q_heads", [32, 40, 64])
def test_step_with_larger_groups_matches_torch_sdpa(oracle_mod, num_q_heads):
    from decode_attention_qk_b200 import inputs
    w = inputs.custom([1, 17, 40], seed=30, num_q_heads=num_q_heads, pool_pages=6)
    out = oracle_mod.append_and_attend(inputs.bf16_bits(w.qkv), inputs.bf16_bits(w.q_norm_w),
                                       inputs.bf16_bits(w.k_norm_w), w.seq_lens.numpy(), w.block_table.numpy(),
                                       inputs.bf16_bits(w.k_cache), inputs.bf16_bits(w.v_cache), want_qk=True)
    assert out["o"].shape == (3, num_q_heads, 128)
    kc, vc = out["k_cache"], out["v_cache"]
    for b, L in enumerate(w.seq_lens.tolist()):
        bt = w.block_table[b].numpy()
        K = np.stack([oracle_mod.bf16_to_f64(kc[bt[t // 16], t % 16]) for t in range(L)], axis=1)
        V = np.stack([oracle_mod.bf16_to_f64(vc[bt[t // 16], t % 16]) for t in range(L)], axis=1)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(out["q"][b])[None, :, None, :], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
            enable_gqa=True)[0, :, 0].numpy()
        assert np.max(np.abs(out["o"][b] - ref)) <= 1e-9 * np.max(np.abs(ref))


@pytest.mark.parametrize("num_q_heads", [32, 40, 64])
def test_larger_group_head_mapping(oracle_mod, num_q_heads):
    """kv head j serves query heads G*j .. G*j+G-1, G = num_q_heads / 8."""
    from decode_attention_qk_b200 import inputs
    G = num_q_heads // 8
    w = inputs.custom([20], seed=31, num_q_heads=num_q_heads)
    args = [inputs.bf16_bits(w.qkv), inputs.bf16_bits(w.q_norm_w), inputs.bf16_bits(w.k_norm_w),
            w.seq_lens.numpy(), w.block_table.numpy()]
    kc, vc = inputs.bf16_bits(w.k_cache), inputs.bf16_bits(w.v_cache)
    base = oracle_mod.append_and_attend(*args, kc, vc)["o"]
    for j in (0, 5, 7):
        vc2 = vc.copy()
        for t in range(19):
            vc2[w.block_table[0, t // 16], t % 16, j] ^= 0x0100
        o = oracle_mod.append_and_attend(*args, kc, vc2)["o"]
        changed = [h for h in range(num_q_heads) if not np.array_equal(o[0, h], base[0, h])]
        assert changed == list(range(G * j, G * j + G))


# ----------------------------------------------------------------------------
# several new tokens per sequence, causal inside the new block
# (Model Spec, "What to watch for": every layer is full causal attention;
#  "At a glance": T tokens; Supported models: forward_causal)

def _tok_args(w, oracle_mod):
    from decode_attention_qk_b200 import inputs
    return dict(qkv=inputs.bf16_bits(w.qkv), q_norm_w=inputs.bf16_bits(w.q_norm_w),
                k_norm_w=inputs.bf16_bits(w.k_norm_w), seq_lens=w.seq_lens.numpy(),
                block_table=w.block_table.numpy(), k_cache=inputs.bf16_bits(w.k_cache),
                v_cache=inputs.bf16_bits(w.v_cache))


@pytest.mark.parametrize("T,hq", [(2, 16), (3, 16), (4, 16), (2, 32), (8, 16), (5, 64), (24, 16)])
def test_tokens_match_sdpa_with_bottom_right_causal_mask(oracle_mod, T, hq):
    from decode_attention_qk_b200 import inputs
    w = inputs.custom([T, max(17, T), max(40, T + 16)], seed=50 + T, num_q_heads=hq, new_tokens=T, pool_pages=8)
    out = oracle_mod.append_and_attend_tokens(**_tok_args(w, oracle_mod), want_qk=True)
    kc, vc = out["k_cache"], out["v_cache"]
    for b, L in enumerate(w.seq_lens.tolist()):
        bt = w.block_table[b].numpy()
        K = np.stack([oracle_mod.bf16_to_f64(kc[bt[t // 16], t % 16]) for t in range(L)], axis=1)
        V = np.stack([oracle_mod.bf16_to_f64(vc[bt[t // 16], t % 16]) for t in range(L)], axis=1)
        mask = torch.tensor([[s <= L - T + t for s in range(L)] for t in range(T)])   # query t, key s
        q = torch.from_numpy(out["q"][b]).permute(1, 0, 2)[None]                   # [1, Hq, T, 128]
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, torch.from_numpy(K)[None], torch.from_numpy(V)[None], attn_mask=mask, enable_gqa=True)
        ref = ref[0].permute(1, 0, 2).numpy()                                      # [T, Hq, 128]
        assert np.max(np.abs(out["o"][b] - ref)) <= 1e-9 * np.max(np.abs(ref))


def test_tokens_equal_successive_single_token_steps(oracle_mod):
    """T new tokens in one step give exactly what T one-token steps give, one after
    the other: same cache, same outputs (the decode step is the T = 1 case)."""
    from decode_attention_qk_b200 import inputs
    T = 3
    w = inputs.custom([20, 3, 50], seed=53, new_tokens=T, pool_pages=7)
    a = _tok_args(w, oracle_mod)
    multi = oracle_mod.append_and_attend_tokens(**a)
    kc, vc = a["k_cache"].copy(), a["v_cache"].copy()
    for t in range(T):
        lens = w.seq_lens.numpy() - (T - 1 - t)
        one = oracle_mod.append_and_attend(a["qkv"][:, t], a["q_norm_w"], a["k_norm_w"], lens, a["block_table"],
                                           kc, vc, inplace=True)
        assert np.array_equal(one["o"], multi["o"][:, t])
    assert np.array_equal(kc, multi["k_cache"]) and np.array_equal(vc, multi["v_cache"])


def test_tokens_causality(oracle_mod):
    """Model conformance, "Causality": changing a later new token's q, k and v never
    changes an earlier new token's output (the earlier outputs stay bit-identical)."""
    from decode_attention_qk_b200 import inputs
    T = 4
    w = inputs.custom([30, 4], seed=54, new_tokens=T)
    a = _tok_args(w, oracle_mod)
    base = oracle_mod.append_and_attend_tokens(**a)["o"]
    for t in range(T):
        a2 = dict(a)
        qkv = a["qkv"].copy()
        qkv[:, t, :] ^= 0x0040          # perturb token t's whole row
        a2["qkv"] = qkv
        o = oracle_mod.append_and_attend_tokens(**a2)["o"]
        assert np.array_equal(o[:, :t], base[:, :t])
        assert not np.array_equal(o[:, t], base[:, t])


def test_tokens_default_positions(oracle_mod):
    from decode_attention_qk_b200 import inputs
    w = inputs.custom([9, 33], seed=55, new_tokens=2)
    a = _tok_args(w, oracle_mod)
    o1 = oracle_mod.append_and_attend_tokens(**a)["o"]
    o2 = oracle_mod.append_and_attend_tokens(**a, positions=w.seq_lens.numpy() - 2)["o"]
    assert np.array_equal(o1, o2)


def test_thread_count_does_not_change_the_result(oracle_mod):
    """The step's attention loop may run on several threads (for the timed CPU
    baseline); every row is the same sequential computation either way."""
    from decode_attention_qk_b200 import inputs
    w = inputs.custom([300, 1000, 17, 2, 64], seed=77, gap_fraction=0.3, num_q_heads=32, new_tokens=2)
    args = (inputs.bf16_bits(w.qkv), inputs.bf16_bits(w.q_norm_w), inputs.bf16_bits(w.k_norm_w),
            w.seq_lens.numpy(), w.block_table.numpy(), inputs.bf16_bits(w.k_cache), inputs.bf16_bits(w.v_cache))
    one = oracle_mod.append_and_attend_tokens(*args)
    oracle_mod.set_threads(4)
    try:
        four = oracle_mod.append_and_attend_tokens(*args)
    finally:
        oracle_mod.set_threads(1)
    assert oracle_mod.get_threads() == 1
    assert np.array_equal(one["o"], four["o"])
    assert np.array_equal(one["k_cache"], four["k_cache"]) and np.array_equal(one["v_cache"], four["v_cache"])
