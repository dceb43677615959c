"""Seeded synthetic workloads for the Qwen3-0.6B decode-attention step.

This module is shared by the tests, the smoke check and the benchmark, and it
feeds the CUDA library and the float64 oracle the same bytes. It only draws
random numbers and lays out pages: none of the step's arithmetic (norm,
rotation, append, attention) is here.

Shapes and value recipes follow the Qwen3-0.6B Model Spec's shape domain
("At a glance": B in [1, 256] sequences, S in [1, 40960] cached positions,
page size 16) and the conformance method of the "Model conformance" page
("How the comparison works", step 1: norm weights perturbed away from their
identity value):

  qkv                 bf16 [B, (Hq + 16) * 128] ~ N(0, 1) (Hq = 16 for Qwen3-0.6B;
                      32, 40 or 64 for the 4B/8B, 14B and 32B sizes)
  q_norm_w, k_norm_w  bf16 [128] = 1 + U(-0.5, 0.5)
  k_cache, v_cache    bf16 [num_pages, 16, 8, 128] ~ N(0, 1)
  block_table         int32 [B, stride], distinct pages drawn from a random
                      permutation of the pool, -1 past each sequence's pages

Large tensors are drawn on the requested device with a generator of that
device, so a CUDA workload and a CPU workload with the same seed differ; the
tests hand the oracle the bytes the device holds.
"""
from __future__ import annotations

import dataclasses
import math

import torch

PAGE = 16
NUM_Q_HEADS = 16
NUM_KV_HEADS = 8
HEAD_DIM = 128
QKV_WIDTH = 4096
MAX_BATCH = 256
MAX_SEQ = 40960
MAX_PAGES_PER_SEQ = MAX_SEQ // PAGE


@dataclasses.dataclass
class Workload:
    name: str
    seq_lens: torch.Tensor          # int32 [B], CPU; counts the new token
    block_table: torch.Tensor       # int32 [B, stride], CPU; -1 where unused
    num_pages: int
    qkv: torch.Tensor               # bf16 [B, (Hq + 16) * 128], or [B, T, ...] for T new tokens, on `device`
    q_norm_w: torch.Tensor          # bf16 [128] on `device`
    k_norm_w: torch.Tensor          # bf16 [128] on `device`
    k_cache: torch.Tensor           # bf16 [num_pages, 16, 8, 128] on `device`
    v_cache: torch.Tensor           # bf16 [num_pages, 16, 8, 128] on `device`
    positions: torch.Tensor | None = None  # int32 [B], CPU, or None

    @property
    def batch(self) -> int:
        return int(self.seq_lens.numel())

    @property
    def device(self) -> torch.device:
        return self.qkv.device

    @property
    def num_q_heads(self) -> int:
        return int(self.qkv.shape[-1]) // HEAD_DIM - 2 * NUM_KV_HEADS

    @property
    def new_tokens(self) -> int:
        return 1 if self.qkv.dim() == 2 else int(self.qkv.shape[1])


def pages_for(seq_lens: torch.Tensor) -> torch.Tensor:
    """Pages each sequence occupies (ceil(L / 16))."""
    return (seq_lens.to(torch.int64) + PAGE - 1) // PAGE


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def assign_pages(seq_lens: torch.Tensor, pool_pages: int, seed: int,
                 stride: int | None = None, gap_fraction: float = 0.0) -> torch.Tensor:
    """Block table whose sequences own distinct pages of a shuffled pool.

    With `gap_fraction` > 0 a random subset of the pool (that fraction of the
    pages in use) is never referenced, so used pages are interleaved with gaps.
    """
    n = pages_for(seq_lens)
    need = int(n.sum())
    if pool_pages < need:
        raise ValueError(f"pool of {pool_pages} pages is smaller than the {need} pages needed")
    stride = int(stride if stride is not None else max(1, int(n.max())))
    g = _gen(seed, "cpu")
    perm = torch.randperm(pool_pages, generator=g).to(torch.int32)
    if gap_fraction > 0.0:
        keep = torch.ones(pool_pages, dtype=torch.bool)
        n_gap = min(pool_pages - need, int(math.ceil(gap_fraction * need)))
        gaps = torch.randperm(pool_pages, generator=g)[:n_gap]
        keep[gaps] = False
        perm = perm[keep[perm.to(torch.int64)]]
    bt = torch.full((seq_lens.numel(), stride), -1, dtype=torch.int32)
    off = 0
    for b, nb in enumerate(n.tolist()):
        bt[b, :nb] = perm[off:off + nb]
        off += nb
    return bt


def qkv_width(num_q_heads: int) -> int:
    """Width of the fused qkv row: Hq query heads, then 8 k and 8 v heads, of 128."""
    return (num_q_heads + 2 * NUM_KV_HEADS) * HEAD_DIM


def _values(B: int, num_pages: int, seed: int, device, num_q_heads: int = NUM_Q_HEADS,
            new_tokens: int = 1) -> dict:
    dev = torch.device(device)
    shape = (B, qkv_width(num_q_heads)) if new_tokens == 1 else (B, new_tokens, qkv_width(num_q_heads))
    qkv = torch.randn(shape, generator=_gen(seed * 16 + 1, dev), device=dev,
                      dtype=torch.float32).to(torch.bfloat16)
    gq = torch.rand(HEAD_DIM, generator=_gen(seed * 16 + 2, dev), device=dev, dtype=torch.float32)
    gk = torch.rand(HEAD_DIM, generator=_gen(seed * 16 + 3, dev), device=dev, dtype=torch.float32)
    shape = (num_pages, PAGE, NUM_KV_HEADS, HEAD_DIM)
    k_cache = torch.randn(shape, generator=_gen(seed * 16 + 4, dev), device=dev, dtype=torch.bfloat16)
    v_cache = torch.randn(shape, generator=_gen(seed * 16 + 5, dev), device=dev, dtype=torch.bfloat16)
    return dict(qkv=qkv, q_norm_w=(gq + 0.5).to(torch.bfloat16), k_norm_w=(gk + 0.5).to(torch.bfloat16),
                k_cache=k_cache, v_cache=v_cache)


def custom(seq_lens, seed: int = 0, device="cpu", pool_pages: int | None = None,
           stride: int | None = None, gap_fraction: float = 0.0, positions=None,
           name: str = "custom", num_q_heads: int = NUM_Q_HEADS, new_tokens: int = 1) -> Workload:
    """A workload with the given sequence lengths (counting the new tokens) and the
    standard value recipe; with new_tokens = T > 1, qkv is [B, T, width]."""
    seq_lens = torch.as_tensor(seq_lens, dtype=torch.int32).reshape(-1)
    need = int(pages_for(seq_lens).sum())
    if pool_pages is None:
        pool_pages = need + (int(math.ceil(gap_fraction * need)) if gap_fraction > 0 else 0)
    bt = assign_pages(seq_lens, pool_pages, seed, stride=stride, gap_fraction=gap_fraction)
    vals = _values(seq_lens.numel(), pool_pages, seed, device, num_q_heads, new_tokens)
    pos = None if positions is None else torch.as_tensor(positions, dtype=torch.int32).reshape(-1)
    return Workload(name=name, seq_lens=seq_lens, block_table=bt, num_pages=pool_pages,
                    positions=pos, **vals)


def config1(device="cpu") -> Workload:
    """B=2, seq_lens {7, 12} (with the new token), 4 pages, seed 0.

    The block table is a random permutation of the 4 pages viewed as [2, 2];
    the second column is real pages that the step must not read. Lengths 7 and
    12 are the reduced profile's token lengths on the "Model conformance" page.
    """
    seed = 0
    seq_lens = torch.tensor([7, 12], dtype=torch.int32)
    bt = torch.randperm(4, generator=_gen(seed, "cpu")).to(torch.int32).view(2, 2).contiguous()
    vals = _values(2, 4, seed, device)
    return Workload(name="cfg1: B=2, seq_lens={7,12}, 4 pages", seq_lens=seq_lens,
                    block_table=bt, num_pages=4, **vals)


def config2(device="cpu", seed: int = 2000, num_q_heads: int = NUM_Q_HEADS, new_tokens: int = 1) -> Workload:
    """B=32, seq_lens ~ U{1..4096} (at least new_tokens), pool of 32*256 shuffled pages."""
    seq_lens = torch.randint(1, 4097, (32,), generator=_gen(seed, "cpu"), dtype=torch.int64).to(torch.int32)
    seq_lens = seq_lens.clamp(min=new_tokens)
    pool = 32 * 256
    bt = assign_pages(seq_lens, pool, seed + 1, stride=256)
    vals = _values(32, pool, seed, device, num_q_heads, new_tokens)
    return Workload(name="cfg2: B=32, seq_lens~U[1,4096], page 16, shuffled pool of 8192 pages",
                    seq_lens=seq_lens, block_table=bt, num_pages=pool, **vals)


def config3_layer(layer: int, device="cpu", seed: int = 3000) -> Workload:
    """One of 28 independent layers: B=256, seq_len 2048, own pool of 32768 pages."""
    s = seed + layer
    seq_lens = torch.full((256,), 2048, dtype=torch.int32)
    pool = 256 * 128
    bt = assign_pages(seq_lens, pool, s + 100, stride=128)
    vals = _values(256, pool, s, device)
    return Workload(name=f"cfg3 layer {layer}: B=256, seq_len=2048, pool of 32768 pages",
                    seq_lens=seq_lens, block_table=bt, num_pages=pool, **vals)


CONFIG3_LAYERS = 28


def config4(device="cpu", seed: int = 4000, num_q_heads: int = NUM_Q_HEADS, new_tokens: int = 1) -> Workload:
    """B=4, seq_len 40960 (the maximum context), 10240 shuffled pages."""
    seq_lens = torch.full((4,), MAX_SEQ, dtype=torch.int32)
    pool = 4 * MAX_PAGES_PER_SEQ
    bt = assign_pages(seq_lens, pool, seed + 1, stride=MAX_PAGES_PER_SEQ)
    vals = _values(4, pool, seed, device, num_q_heads, new_tokens)
    return Workload(name="cfg4: B=4, seq_len=40960, 10240 shuffled pages",
                    seq_lens=seq_lens, block_table=bt, num_pages=pool, **vals)


def config5_lengths(seed: int = 5000) -> torch.Tensor:
    """B=256 lengths: round(lognormal(mu=7, sigma=1.5)) clipped to [1, 40960]."""
    z = torch.randn(256, generator=_gen(seed, "cpu"), dtype=torch.float64)
    return torch.exp(7.0 + 1.5 * z).round().clamp(1, MAX_SEQ).to(torch.int32)


def config5(device="cpu", seed: int = 5000, num_q_heads: int = NUM_Q_HEADS, new_tokens: int = 1) -> Workload:
    """B=256 ragged lognormal lengths (at least new_tokens); pool 1.1x the pages in use, gaps interleaved."""
    seq_lens = config5_lengths(seed).clamp(min=new_tokens)
    need = int(pages_for(seq_lens).sum())
    pool = int(math.ceil(1.1 * need))
    bt = assign_pages(seq_lens, pool, seed + 1, stride=MAX_PAGES_PER_SEQ, gap_fraction=0.1)
    vals = _values(256, pool, seed, device, num_q_heads, new_tokens)
    return Workload(name="cfg5: B=256, seq_lens lognormal(7,1.5) clipped, 10% gap pages",
                    seq_lens=seq_lens, block_table=bt, num_pages=pool, **vals)


HIDDEN = 1024   # Qwen3-0.6B hidden size (Model Spec, "Compute-graph nodes": input_norm H=1024)


def hidden_inputs(B: int, seed: int = 0, device="cpu", hidden: int = HIDDEN,
                  num_q_heads: int = NUM_Q_HEADS) -> dict:
    """Inputs of input_norm + attn.qkv_proj: x bf16 [B, hidden] ~ N(0, 1); the
    input_norm gain bf16 [hidden] = 1 + U(-0.5, 0.5) (perturbed away from 1, as
    the conformance method does); the qkv_proj weight bf16 [(Hq + 16) * 128,
    hidden] ~ N(0, 1/hidden), so that the outputs stay O(1)."""
    dev = torch.device(device)
    N = qkv_width(num_q_heads)
    x = torch.randn((B, hidden), generator=_gen(seed * 16 + 6, dev), device=dev).to(torch.bfloat16)
    g = (torch.rand(hidden, generator=_gen(seed * 16 + 7, dev), device=dev) + 0.5).to(torch.bfloat16)
    w = (torch.randn((N, hidden), generator=_gen(seed * 16 + 8, dev), device=dev) / math.sqrt(hidden)).to(torch.bfloat16)
    return dict(x=x, input_norm_w=g, w_qkv=w)


def o_proj_inputs(B: int, seed: int = 0, device="cpu", hidden: int = HIDDEN,
                  num_q_heads: int = NUM_Q_HEADS) -> dict:
    """Inputs of attn.o_proj: x bf16 [B, Hq * 128] ~ N(0, 1) (the attention output
    o [B, Hq, 128] read as rows); the o_proj weight bf16 [hidden, Hq * 128] ~
    N(0, 1/(Hq * 128)), so that the outputs stay O(1)."""
    dev = torch.device(device)
    K = num_q_heads * HEAD_DIM
    x = torch.randn((B, K), generator=_gen(seed * 16 + 9, dev), device=dev).to(torch.bfloat16)
    w = (torch.randn((hidden, K), generator=_gen(seed * 16 + 10, dev), device=dev) / math.sqrt(K)).to(torch.bfloat16)
    return dict(x=x, w_o=w)


def bf16_bits(t: torch.Tensor):
    """numpy uint16 view of a bf16 tensor's bits (copied to the host)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view("uint16")
