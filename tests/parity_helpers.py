"""Helpers that compare the CUDA library with the float64 oracle.

Tolerances for o (bf16 output of a float computation):
  gate    max |o - o_ref| <= 2e-2 and ||o - o_ref|| / ||o_ref|| <= 1e-2 over
          the whole output (the required tolerance);
  strict  |o - o_ref| <= 2^-8 |o_ref| + 1e-4 element by element: one bf16
          rounding of o (at most 2^-9 relative) plus float error in the
          scores, exp2 and sums (~1e-5 absolute at O(1) values). It catches
          a dropped or doubled token, which the gate alone would not.
The cache is compared bit for bit.
"""
from __future__ import annotations

import dataclasses
import numpy as np
import torch

import oracle
from decode_attention_qk_b200 import inputs

GATE_ABS, GATE_REL = 2e-2, 1e-2
STRICT_REL, STRICT_ABS = 2.0 ** -8, 1e-4


def device_args(w: inputs.Workload, dev, positions=None):
    """The per-step tensors of a workload on `dev` (caches are used in place)."""
    pos = positions if positions is not None else w.positions
    return dict(qkv=w.qkv.to(dev), q_norm_w=w.q_norm_w.to(dev), k_norm_w=w.k_norm_w.to(dev),
                seq_lens=w.seq_lens.to(dev), block_table=w.block_table.to(dev),
                positions=None if pos is None else pos.to(dev))


def gains_at_a_4_byte_offset(w: inputs.Workload) -> inputs.Workload:
    """The same workload with q_norm_w and k_norm_w on the device at addresses
    that are 4-byte but not 8-byte aligned (the alignment the ABI asks of them)."""
    def at4(t):
        buf = torch.empty(t.numel() + 8, dtype=t.dtype, device=t.device)
        view = buf[2:2 + t.numel()]
        view.copy_(t)
        assert view.data_ptr() % 8 == 4
        return view
    return dataclasses.replace(w, q_norm_w=at4(w.q_norm_w), k_norm_w=at4(w.k_norm_w))


def run(attn, w: inputs.Workload, dev, k_cache, v_cache, positions=None, o=None):
    a = device_args(w, dev, positions)
    o = attn(a["qkv"], a["q_norm_w"], a["k_norm_w"], a["seq_lens"], a["block_table"], k_cache, v_cache,
             o=o, positions=a["positions"])
    return o


def _qkv3(w: inputs.Workload) -> np.ndarray:
    """qkv bits as [B, T, W] (T = 1 for a single new token)."""
    bits = inputs.bf16_bits(w.qkv)
    return bits.reshape(w.batch, w.new_tokens, -1)


def _o_shape(w: inputs.Workload, o: np.ndarray) -> np.ndarray:
    """The oracle's [B, T, Hq, 128] o in the layout of the call: [B, Hq, 128] when T = 1."""
    return o[:, 0] if w.qkv.dim() == 2 else o


def oracle_full(w: inputs.Workload, k_cache_pre, v_cache_pre, positions=None):
    """The oracle on the whole batch; caches given as tensors (any device), pre-call."""
    pos = positions if positions is not None else w.positions
    out = oracle.append_and_attend_tokens(
        _qkv3(w), inputs.bf16_bits(w.q_norm_w), inputs.bf16_bits(w.k_norm_w),
        w.seq_lens.numpy(), w.block_table.numpy(), inputs.bf16_bits(k_cache_pre), inputs.bf16_bits(v_cache_pre),
        positions=None if pos is None else pos.cpu().numpy(), inplace=True, want_qk=True)
    out["o"] = _o_shape(w, out["o"])
    return out


def _compact(w, seqs, k_pre, v_pre, tail_only=False):
    """A sub-batch of the sequences `seqs` over a pool holding only their pages
    (with `tail_only`, only the pages from the one holding the first new token)."""
    lens = w.seq_lens[seqs]
    T = w.new_tokens
    rows, pages = [], []
    for b in seqs.tolist():
        L = int(w.seq_lens[b])
        n = (L + 15) // 16
        ids = w.block_table[b, (L - T) // 16:n] if tail_only else w.block_table[b, :n]
        rows.append(torch.arange(len(pages), len(pages) + len(ids), dtype=torch.int32))
        pages.extend(ids.tolist())
    stride = max(len(r) for r in rows)
    bt = torch.full((len(seqs), stride), -1, dtype=torch.int32)
    for i, r in enumerate(rows):
        bt[i, :len(r)] = r
    idx = torch.tensor(pages, dtype=torch.int64, device=k_pre.device)
    kc = inputs.bf16_bits(k_pre.index_select(0, idx))
    vc = inputs.bf16_bits(v_pre.index_select(0, idx))
    return lens, bt, kc, vc


def oracle_sampled(w: inputs.Workload, seqs, k_pre, v_pre):
    """Oracle o for the sequences `seqs` only ([len(seqs), (T,) Hq, 128] float64)."""
    seqs = torch.as_tensor(seqs, dtype=torch.int64)
    lens, bt, kc, vc = _compact(w, seqs, k_pre, v_pre)
    pos = None if w.positions is None else w.positions[seqs].numpy()
    out = oracle.append_and_attend_tokens(
        _qkv3(w)[seqs.numpy()], inputs.bf16_bits(w.q_norm_w),
        inputs.bf16_bits(w.k_norm_w), lens.numpy(), bt.numpy(), kc, vc, positions=pos, inplace=True)
    return _o_shape(w, out["o"])


def _new_slots(w: inputs.Workload):
    """(b, t, page, row) of every appended token: token t of sequence b goes to slot L - T + t."""
    T = w.new_tokens
    for b in range(w.batch):
        L = int(w.seq_lens[b])
        for t in range(T):
            slot = L - T + t
            yield b, t, int(w.block_table[b, slot // 16]), slot % 16


def oracle_appended_rows(w: inputs.Workload, k_pre, v_pre):
    """The oracle's appended k/v rows for every sequence, cheaply: each sequence is
    replaced by its pages from the first new token's on, with its true RoPE
    positions.

    Returns (k_rows, v_rows) uint16 [B, T, 8, 128] and k64, the new k in float64.
    """
    B, T = w.batch, w.new_tokens
    seqs = torch.arange(B)
    lens, bt, kc, vc = _compact(w, seqs, k_pre, v_pre, tail_only=True)
    short = (lens - (lens - T) // 16 * 16).to(torch.int32)
    pos = (w.seq_lens - T) if w.positions is None else w.positions
    out = oracle.append_and_attend_tokens(
        _qkv3(w), inputs.bf16_bits(w.q_norm_w), inputs.bf16_bits(w.k_norm_w), short.numpy(),
        bt.numpy(), kc, vc, positions=pos.numpy().astype(np.int32), inplace=True, want_qk=True)
    k_rows = np.empty((B, T, 8, 128), np.uint16)
    v_rows = np.empty((B, T, 8, 128), np.uint16)
    for b in range(B):
        for t in range(T):
            slot = int(short[b]) - T + t
            k_rows[b, t] = out["k_cache"][bt[b, slot // 16], slot % 16]
            v_rows[b, t] = out["v_cache"][bt[b, slot // 16], slot % 16]
    return k_rows, v_rows, out["k"]


def expected_cache(w: inputs.Workload, k_pre, v_pre, k_rows, v_rows):
    """The pre-call caches (device) with each sequence's appended rows written in."""
    k_exp, v_exp = k_pre.clone(), v_pre.clone()
    dev = k_pre.device
    for b, t, page, row in _new_slots(w):
        k_exp[page, row] = torch.from_numpy(k_rows[b, t].view(np.int16)).view(torch.bfloat16).to(dev)
        v_exp[page, row] = torch.from_numpy(v_rows[b, t].view(np.int16)).view(torch.bfloat16).to(dev)
    return k_exp, v_exp


def describe_k_mismatch(got_bits, want_bits, k64):
    """For a differing appended k, how far the float64 value sat from a bf16 midpoint."""
    bad = np.argwhere(got_bits != want_bits)
    lines = []
    for idx in bad[:8]:
        x = float(k64[tuple(idx)])
        lo = oracle.bf16_to_f64(np.array([want_bits[tuple(idx)]], np.uint16))[0]
        hi = oracle.bf16_to_f64(np.array([got_bits[tuple(idx)]], np.uint16))[0]
        mid = (lo + hi) / 2
        lines.append(f"{tuple(idx)}: k64={x!r} gpu={hi!r} oracle={lo!r} |k64-mid|/|k64|={abs(x - mid) / abs(x):.3g}")
    return f"{len(bad)} appended k values differ:\n" + "\n".join(lines)


def assert_cache_equal(k_got, v_got, k_exp, v_exp, k64=None, w=None):
    if torch.equal(k_got.view(torch.int16), k_exp.view(torch.int16)) and \
            torch.equal(v_got.view(torch.int16), v_exp.view(torch.int16)):
        return
    msg = "cache differs from the oracle"
    if k64 is not None and w is not None:
        T = w.new_tokens
        gb = np.empty((w.batch, T, 8, 128), np.uint16)
        wb = np.empty((w.batch, T, 8, 128), np.uint16)
        for b, t, page, row in _new_slots(w):
            gb[b, t] = inputs.bf16_bits(k_got[page, row])
            wb[b, t] = inputs.bf16_bits(k_exp[page, row])
        msg += "\n" + describe_k_mismatch(gb, wb, k64.reshape(gb.shape))
    kd = (k_got.view(torch.int16) != k_exp.view(torch.int16)).nonzero()[:5].tolist()
    vd = (v_got.view(torch.int16) != v_exp.view(torch.int16)).nonzero()[:5].tolist()
    raise AssertionError(f"{msg}; first k diffs {kd}, v diffs {vd}")


def o_errors(o_got, o_ref):
    got = o_got.detach().float().cpu().numpy().astype(np.float64)
    ref = np.asarray(o_ref, dtype=np.float64)
    err = np.abs(got - ref)
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    strict_excess = float(np.max(err - (STRICT_REL * np.abs(ref) + STRICT_ABS)))
    return float(err.max()), rel, strict_excess


def assert_o_close(o_got, o_ref, label=""):
    max_abs, rel, strict_excess = o_errors(o_got, o_ref)
    assert max_abs <= GATE_ABS and rel <= GATE_REL, f"{label}: max abs {max_abs:.3g}, rel rms {rel:.3g}"
    assert strict_excess <= 0.0, f"{label}: strict bound exceeded by {strict_excess:.3g} (max abs {max_abs:.3g})"
    return max_abs, rel


# ---------------------------------------------------------------------------
# Instances with more than 8 query rows per kv head ("wide": T * Hq / 8 > 8)
# enter q and the probabilities into the tensor cores as bf16. Their strict
# check compares o with a float64 attention that uses the oracle's q rounded
# the way the kernel rounds it (bf16 of q * log2(e) / sqrt(128), nearest-even),
# over the oracle's post-append cache. Rounding each probability to bf16
# (relative error <= 2^-9; the sums add the same rounded values) moves each
# normalised weight by at most ~2^-8 of itself, so
#   |o - o_emul| <= 2^-8 sum_t w_t |v_t - o_emul|,
# checked with a factor 2 of margin (a float q may round to the neighbouring
# bf16 value where the double one sits near a midpoint), plus o's own bf16
# rounding and float sums: 2^-7 sum_t w_t |v_t - o| + 2^-8 |o| + 2e-4.

Q_SCALE = 1.4426950408889634 / np.sqrt(128.0)


def chunk_sizes(num_q_heads: int, T: int):
    """How the library runs a block of T new tokens: up to 16 query rows per kv
    head (T * Hq / 8) in one launch of the decode-shaped tensor-core kernel; a
    longer block as a chunked prefill, chunks of 128 / G tokens."""
    G = num_q_heads // 8
    if T * G <= 16:
        return [T]
    max_t = 128 // G
    return [min(max_t, T - c0) for c0 in range(0, T, max_t)]


def wide_tokens(w: inputs.Workload):
    """Per new token: whether its launch takes q and the probabilities into the
    tensor cores as bf16 (more than 8 query rows per kv head in a decode-shaped
    launch, and every prefill chunk)."""
    G = w.num_q_heads // 8
    if w.new_tokens == 1:
        return [False]
    if w.new_tokens * G > 16:
        return [True] * w.new_tokens
    return [w.new_tokens * G > 8] * w.new_tokens


def is_wide(w: inputs.Workload) -> bool:
    return any(wide_tokens(w))


def emulated_bf16_q_check(o_gpu, q64, seq_lens, block_table, k_bits, v_bits, T, label="", tokens=None):
    """o_gpu [B, T, Hq, 128] against the float64 attention with bf16-rounded
    scaled q (see above) for the new tokens `tokens` (default all); q64 the
    oracle's q [B, T, Hq, 128]; caches post-append."""
    got = o_gpu.detach().float().cpu().numpy().astype(np.float64)
    B, _, Hq, D = q64.shape
    G = Hq // 8
    qs = oracle.bf16_to_f64(oracle.f64_to_bf16_rne(q64 * Q_SCALE))
    worst = -np.inf
    for b in range(B):
        L = int(seq_lens[b])
        slots = np.arange(L)
        pages = block_table[b, slots // 16]
        K = oracle.bf16_to_f64(k_bits[pages, slots % 16])   # [L, 8, 128]
        V = oracle.bf16_to_f64(v_bits[pages, slots % 16])
        for t in (range(T) if tokens is None else tokens):
            n = L - T + t + 1
            for h in range(Hq):
                s = K[:n, h // G] @ qs[b, t, h]          # log2 units
                wgt = np.exp2(s - s.max())
                wgt /= wgt.sum()
                o_em = wgt @ V[:n, h // G]
                spread = wgt @ np.abs(V[:n, h // G] - o_em)
                bound = 2.0 ** -7 * spread + 2.0 ** -8 * np.abs(o_em) + 2e-4
                worst = max(worst, float(np.max(np.abs(got[b, t, h] - o_em) - bound)))
    assert worst <= 0.0, f"{label}: bf16-q bound exceeded by {worst:.3g}"


def oracle_sampled_qk(w: inputs.Workload, seqs, k_pre, v_pre):
    """The oracle over the sequences `seqs` only, with q and the compact
    post-append caches (for emulated_bf16_q_check)."""
    seqs = torch.as_tensor(seqs, dtype=torch.int64)
    lens, bt, kc, vc = _compact(w, seqs, k_pre, v_pre)
    pos = None if w.positions is None else w.positions[seqs].numpy()
    out = oracle.append_and_attend_tokens(
        _qkv3(w)[seqs.numpy()], inputs.bf16_bits(w.q_norm_w), inputs.bf16_bits(w.k_norm_w), lens.numpy(),
        bt.numpy(), kc, vc, positions=pos, inplace=True, want_qk=True)
    return out, lens.numpy(), bt.numpy()
