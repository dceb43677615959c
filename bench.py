"""Benchmark of the Qwen3-0.6B decode-attention step on B200.

One step is one pass of the whole path (q/k norm, RoPE, cache append,
decodeGQA) over one batch: one library call for a single-layer workload, 28
calls for the 28-layer one. Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload cfg2]
  python bench.py --impl reference ...   (the float64 CPU oracle, host cores)

Multi-GPU (torchrun, one process per GPU): every rank runs its own replica of
the workload (sequences are independent; no collective on the data path);
timing is the max over ranks, the value the sum of all ranks' bytes over it.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from decode_attention_qk_b200 import inputs  # noqa: E402

METRIC = "decode-attn KV GB/s and µs/call (1 B200) as fraction of HBM roofline"
PROJ_METRIC = "input_norm + qkv_proj GB/s (weight + x + gain + qkv bytes) and µs/call (1 B200)"
O_METRIC = "attn.o_proj GB/s (weight + x + y bytes) and µs/call (1 B200)"
KV_BYTES_PER_TOKEN = 2 * inputs.NUM_KV_HEADS * inputs.HEAD_DIM * 2      # K and V rows: 4096 B
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 2 ** 20
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
_CSRC = os.path.join(ROOT, "decode_attention_qk_b200", "csrc")
KERNEL_SOURCES = {   # the files each attention kernel is built from
    16: [os.path.join(_CSRC, f) for f in ("qda_decode_kernel.cu", "qda_device.cuh", "qda_internal.h")],
    "grouped": [os.path.join(_CSRC, f) for f in ("qda_decode_mma.cu", "qda_device.cuh", "qda_internal.h")],
    "qkv_proj": [os.path.join(_CSRC, f) for f in ("qda_qkv_proj.cu", "qda_device.cuh", "qda_internal.h")],
    "prefill": [os.path.join(_CSRC, f)
                for f in ("qda_prefill.cu", "qda_prefill.h", "qda_tc.cuh", "qda_device.cuh", "qda_internal.h")],
}

WORKLOADS = {
    "cfg1": "B=2, seq_lens={7,12} incl. new token, 4 pages, random block table",
    "cfg2": "B=32, seq_lens~U[1,4096], page 16, shuffled pool of 8192 pages",
    "cfg3": "B=256, seq_len=2048, 28 independent layer caches (2.15 GB KV each), one step = 28 calls",
    "cfg4": "B=4, seq_len=40960 (max context), 10240 shuffled pages",
    "cfg5": "B=256, seq_lens lognormal(7,1.5) clipped to [1,40960], 10% gap pages",
}


# ----------------------------------------------------------------------------
# workloads and byte counts

def make_layers(name: str, device, rank: int = 0, num_q_heads: int = 16, new_tokens: int = 1, layers: int = 0):
    """The layers of one step (one Workload per library call). num_q_heads picks the
    Qwen3 size: 16 (0.6B), 32 (4B/8B), 40 (14B) or 64 (32B); new_tokens > 1 gives
    every sequence that many new tokens (causal among themselves). cfg1 and cfg3
    are 0.6B with one new token only. layers > 0 keeps only the first `layers`
    layers of cfg3 (to profile one launch without holding all 28 layers)."""
    off = 100 * rank
    if name in ("cfg1", "cfg3") and (num_q_heads != 16 or new_tokens != 1):
        raise ValueError(f"{name} is defined for Qwen3-0.6B (16 query heads) and one new token")
    if name == "cfg1":
        return [inputs.config1(device)] if rank == 0 else [inputs.custom([7, 12], seed=off, device=device)]
    if name == "cfg2":
        return [inputs.config2(device, seed=2000 + off, num_q_heads=num_q_heads, new_tokens=new_tokens)]
    if name == "cfg3":
        n = inputs.CONFIG3_LAYERS if layers <= 0 else min(layers, inputs.CONFIG3_LAYERS)
        return [inputs.config3_layer(i, device, seed=3000 + off) for i in range(n)]
    if name == "cfg4":
        return [inputs.config4(device, seed=4000 + off, num_q_heads=num_q_heads, new_tokens=new_tokens)]
    if name == "cfg5":
        return [inputs.config5(device, seed=5000 + off, num_q_heads=num_q_heads, new_tokens=new_tokens)]
    raise ValueError(name)


def kv_bytes(seq_lens) -> int:
    """K and V bytes the attention reads: every position incl. the new one, 4096 B each."""
    return int(torch.as_tensor(seq_lens, dtype=torch.int64).sum()) * KV_BYTES_PER_TOKEN


def algorithmic_bytes(seq_lens, num_q_heads: int = 16, new_tokens: int = 1) -> int:
    """Least HBM traffic of one call with T = new_tokens: the cached K/V rows
    read (L-T per sequence), the T new k/v rows written, the T qkv rows read,
    o written, the block-table entries and seq_lens read, and the two gain
    vectors."""
    L = torch.as_tensor(seq_lens, dtype=torch.int64)
    B, T = int(L.numel()), new_tokens
    pages = int(((L + 15) // 16).sum())
    return (int((L - T).sum()) * KV_BYTES_PER_TOKEN + B * T * KV_BYTES_PER_TOKEN
            + B * T * inputs.qkv_width(num_q_heads) * 2 + B * T * num_q_heads * inputs.HEAD_DIM * 2
            + pages * 4 + B * 4 + 2 * inputs.HEAD_DIM * 2)


def proj_bytes(batch: int, hidden: int = inputs.HIDDEN, num_q_heads: int = 16) -> int:
    """Least HBM traffic of input_norm + qkv_proj: the weight, x, the gain and qkv."""
    N = inputs.qkv_width(num_q_heads)
    return N * hidden * 2 + batch * hidden * 2 + hidden * 2 + batch * N * 2


def o_bytes(batch: int, hidden: int = inputs.HIDDEN, num_q_heads: int = 16) -> int:
    """Least HBM traffic of attn.o_proj: the weight, x (the attention output) and y."""
    K = num_q_heads * inputs.HEAD_DIM
    return hidden * K * 2 + batch * K * 2 + batch * hidden * 2


def o_flops(batch: int, hidden: int = inputs.HIDDEN, num_q_heads: int = 16) -> int:
    return 2 * batch * hidden * num_q_heads * inputs.HEAD_DIM


def proj_flops(batch: int, hidden: int = inputs.HIDDEN, num_q_heads: int = 16) -> int:
    """Multiply-adds of the projection, 2 flops each (the hi/lo split doubles the tensor work)."""
    return 2 * batch * inputs.qkv_width(num_q_heads) * hidden


def tensor_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def chunk_tokens(args) -> list:
    """New tokens per launch of the tensor-core attention in one call: up to 16
    query rows per kv head (T * Hq / 8) in one decode-shaped launch; a longer
    block as a chunked prefill of 128 / G tokens per chunk."""
    T, G = args.new_tokens, args.num_q_heads // 8
    if T * G <= 16:
        return [T]
    max_t = 128 // G
    return [min(max_t, T - c0) for c0 in range(0, T, max_t)]


def n_chunks(args) -> int:
    return len(chunk_tokens(args))


def grouped_launches(args) -> int:
    """Kernel launches of a several-token call: the decode-shaped attention and
    its combine, or per prefill chunk the prep, the attention and the combine."""
    T, G = args.new_tokens, args.num_q_heads // 8
    return 2 if T * G <= 16 else 3 * n_chunks(args)


def kernel_key(num_q_heads: int = 16, new_tokens: int = 1):
    """Which attention kernel a call runs: the 16-head decode kernel, the
    decode-shaped tensor-core one (up to 16 query rows per kv head) or the
    prefill."""
    if num_q_heads == 16 and new_tokens == 1:
        return 16
    return "grouped" if new_tokens * (num_q_heads // 8) <= 16 else "prefill"


def workload_key(workload: str, num_q_heads: int = 16, new_tokens: int = 1) -> str:
    return workload + ("" if num_q_heads == 16 else f"-h{num_q_heads}") + ("" if new_tokens == 1 else f"-t{new_tokens}")


def kernel_source_hash(num_q_heads: int = 16, new_tokens: int = 1, key=None) -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES[key if key is not None else kernel_key(num_q_heads, new_tokens)]:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_per_launch(workload: str, num_q_heads: int = 16, new_tokens: int = 1, key=None):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, if it was taken on this kernel source and workload (else None)."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    entry = t.get(workload)
    if not entry or entry.get("kernel_source_sha256") != kernel_source_hash(num_q_heads, new_tokens, key):
        return None
    return entry.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------
# clocks

_REASONS = [(0x1, "gpu_idle"), (0x2, "applications_clocks_setting"), (0x4, "sw_power_cap"),
            (0x8, "hw_slowdown"), (0x10, "sync_boost"), (0x20, "sw_thermal_slowdown"),
            (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"), (0x100, "display_clock_setting")]
BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}


class ClockSampler:
    """Samples SM clock and clock-event reasons every ~5 ms (NVML) in a thread."""

    def __init__(self, device_index: int):
        self.samples = []   # (t, sm_mhz, reasons_mask)
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None

    def _run(self):
        n = self._nvml
        while not self._stop.is_set():
            try:
                mhz = n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM)
                reasons = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((time.perf_counter(), mhz, reasons))
            except Exception:
                pass
            self._stop.wait(0.005)

    def start(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def stop(self):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self, t0: float, t1: float, t_warm: float):
        if self._nvml is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "note": "NVML unavailable"}
        window = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "timed region"
        if len(window) < 3:
            window = [s for s in self.samples if t_warm <= s[0] <= t1]
            note = "warm-up + timed region (timed region shorter than the sampling period)"
        if not window:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "note": note}
        mask = 0
        for s in window:
            mask |= s[2]
        reasons = [name for bit, name in _REASONS if mask & bit]
        return {"sm_mhz": statistics.median(s[1] for s in window), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(window), "window": note}


# ----------------------------------------------------------------------------
# distributed plumbing (timing only; the data path has no collective)

def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return dist, int(os.environ["RANK"]), world, local
    if n_gpus != 1:
        raise SystemExit("--gpus N > 1 must be launched with torchrun, one process per GPU")
    return None, 0, 1, 0


def reduce_max(dist, value: float, device) -> float:
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(dist, value: float, device) -> float:
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(dist, device):
    if dist is not None:
        dist.barrier(device_ids=[device.index])
    torch.cuda.synchronize(device)


# ----------------------------------------------------------------------------
# the oracle on the host (CPU baseline and the reference arm)

def compact_host(w: inputs.Workload, seqs):
    """Host bytes of the sequences `seqs` over a pool holding only their pages."""
    pages, rows = [], []
    for b in seqs:
        n = (int(w.seq_lens[b]) + 15) // 16
        rows.append(list(range(len(pages), len(pages) + n)))
        pages.extend(w.block_table[b, :n].tolist())
    stride = max(len(r) for r in rows)
    bt = torch.full((len(seqs), stride), -1, dtype=torch.int32)
    for i, r in enumerate(rows):
        bt[i, :len(r)] = torch.tensor(r, dtype=torch.int32)
    idx = torch.tensor(pages, dtype=torch.int64, device=w.k_cache.device)
    sel = torch.tensor(list(seqs), dtype=torch.int64)
    return dict(qkv=inputs.bf16_bits(w.qkv[sel.to(w.qkv.device)]), q_norm_w=inputs.bf16_bits(w.q_norm_w),
                k_norm_w=inputs.bf16_bits(w.k_norm_w), seq_lens=w.seq_lens[sel].numpy(), block_table=bt.numpy(),
                k_cache=inputs.bf16_bits(w.k_cache.index_select(0, idx)),
                v_cache=inputs.bf16_bits(w.v_cache.index_select(0, idx)))


def time_oracle(batch: dict) -> float:
    import oracle
    step = oracle.append_and_attend_tokens if batch["qkv"].ndim == 3 else oracle.append_and_attend
    t0 = time.perf_counter()
    step(**batch, inplace=True)
    return time.perf_counter() - t0


def pick_sample(layers, budget_bytes: float):
    """(layer, sequences) pairs in order until the KV bytes reach `budget_bytes`
    (at least one sequence)."""
    picked, total = [], 0
    for li, w in enumerate(layers):
        seqs = []
        for b in range(w.batch):
            if total >= budget_bytes and (picked or seqs):
                break
            seqs.append(b)
            total += int(w.seq_lens[b]) * KV_BYTES_PER_TOKEN
        if seqs:
            picked.append((li, seqs))
        if total >= budget_bytes:
            break
    return picked, total


def host_cpu():
    """(usable cores, CPU model) of this host."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return cores, model


def cpu_baseline(layers, seconds: float = 12.0, threads: int = 1):
    """The oracle as it stands on a bounded sample of the step, its attention
    loop on `threads` threads (the result does not depend on the count)."""
    import oracle
    oracle.build()
    oracle.set_threads(threads)
    try:
        probe = min(range(layers[0].batch), key=lambda b: int(layers[0].seq_lens[b]))
        warm = compact_host(layers[0], [probe])
        dt = time_oracle(warm)
        rate = max(int(layers[0].seq_lens[probe]) * KV_BYTES_PER_TOKEN / max(dt, 1e-6), 1e6)
        picked, total_bytes = pick_sample(layers, rate * seconds)
        elapsed = 0.0
        for li, seqs in picked:
            elapsed += time_oracle(compact_host(layers[li], seqs))
    finally:
        oracle.set_threads(1)
    n_seq = sum(len(s) for _, s in picked)
    all_seq = sum(w.batch for w in layers)
    _, model = host_cpu()
    return {"value": total_bytes / elapsed / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{n_seq} of {all_seq} sequences of the step ({total_bytes / 1e9:.3f} GB of KV), "
                      f"{elapsed:.1f} s, {threads} thread{'s' if threads > 1 else ''}",
            "cpu_model": model, "seconds": elapsed}


def time_o_proj_oracle(w, rows) -> float:
    """Seconds the oracle's attn.o_proj takes for the given rows of layer w."""
    import oracle
    d = w.o_in
    sel = torch.tensor(list(rows), dtype=torch.int64, device=d["x"].device)
    x = inputs.bf16_bits(d["x"].index_select(0, sel))
    wo = inputs.bf16_bits(d["w_o"])
    t0 = time.perf_counter()
    oracle.o_proj(x, wo)
    return time.perf_counter() - t0


def time_proj_oracle(w, rows) -> float:
    """Seconds the oracle's input_norm + qkv_proj takes for the given rows of layer w."""
    import oracle
    if getattr(w, "o_in", None) is not None:
        return time_o_proj_oracle(w, rows)
    d = w.hidden_in
    sel = torch.tensor(list(rows), dtype=torch.int64, device=d["x"].device)
    x = inputs.bf16_bits(d["x"].index_select(0, sel))
    g, wq = inputs.bf16_bits(d["input_norm_w"]), inputs.bf16_bits(d["w_qkv"])
    t0 = time.perf_counter()
    oracle.input_norm_qkv_proj(x, g, wq)
    return time.perf_counter() - t0


def cpu_baseline_proj(layers, mode, seconds: float = 12.0, threads: int = 1):
    """The oracle on a bounded sample of the projection modes: qkv_proj alone
    (value = projection bytes / s), or from the hidden state (the projection
    of the sampled sequences plus their attention; value = K/V bytes / s)."""
    import oracle
    oracle.build()
    oracle.set_threads(threads)
    w0 = layers[0]
    hidden = w0.o_in["w_o"].shape[0] if mode == "o_proj" else w0.hidden_in["x"].shape[1]
    try:
        per_row = time_proj_oracle(w0, [0])
        if mode in ("qkv_proj", "o_proj"):
            rows = list(range(min(w0.batch, max(1, int(seconds / max(per_row, 1e-6))))))
            elapsed = time_proj_oracle(w0, rows)
            units = (o_bytes if mode == "o_proj" else proj_bytes)(len(rows), hidden, w0.num_q_heads)
            desc = f"{len(rows)} of {w0.batch} rows of one call"
        else:
            probe = min(range(w0.batch), key=lambda b: int(w0.seq_lens[b]))
            dt = time_oracle(compact_host(w0, [probe])) + per_row
            rate = max(int(w0.seq_lens[probe]) * KV_BYTES_PER_TOKEN / max(dt, 1e-6), 1e6)
            picked, units = pick_sample(layers, rate * seconds)
            elapsed = 0.0
            for li, seqs in picked:
                elapsed += time_proj_oracle(layers[li], seqs) + time_oracle(compact_host(layers[li], seqs))
            desc = f"{sum(len(q) for _, q in picked)} of {sum(w.batch for w in layers)} sequences of the step"
    finally:
        oracle.set_threads(1)
    _, model = host_cpu()
    return {"value": units / elapsed / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": f"{desc}, {elapsed:.1f} s, {threads} thread{'s' if threads > 1 else ''} "
                      "(the projection runs on one)", "cpu_model": model, "seconds": elapsed}


# ----------------------------------------------------------------------------
# GPU arm

def run_gpu(args):
    from decode_attention_qk_b200 import binding

    dist, rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    result = measure(args, dist, rank, world, dev, headline=True)
    per_config = (world == 1 and args.per_config and args.op == "step" and not args.from_hidden
                  and args.num_q_heads == 16 and args.new_tokens == 1)
    if per_config:
        # every other configuration of the workload set, each timed on its own
        # (graph replay of at least ~0.1 s, end to end through the host-buffer
        # entry point), so that one default run covers them all
        entries = {}
        for wl in sorted(WORKLOADS):
            if wl == args.workload:
                continue
            sub = argparse.Namespace(**vars(args))
            sub.workload, sub.warmup, sub.rotate = wl, 5, 0
            entries[wl] = measure(sub, dist, rank, world, dev, headline=False)
            torch.cuda.empty_cache()
        if rank == 0:
            result["per_config"] = entries
    if rank == 0:
        print(json.dumps(result), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def measure(args, dist, rank, world, dev, headline: bool):
    """Time one workload on this rank's GPU. headline: the K steps the command
    line asks for, with the eager comparison and a sustained leg; otherwise a
    per-configuration entry whose step count is chosen so that its timed
    region lasts at least ~0.1 s. Returns the result dict (rank 0) or None."""
    from decode_attention_qk_b200 import binding

    lib = binding.load_library()
    attn = binding.DecodeAttention(device=dev.index, num_q_heads=args.num_q_heads)
    T = args.new_tokens
    mode = args.op if args.op in ("qkv_proj", "o_proj") else ("from_hidden" if args.from_hidden else "attention")
    if mode != "attention" and T != 1:
        raise SystemExit("--op qkv_proj, --op o_proj and --from-hidden take one new token per sequence")

    # R resident copies of the step's inputs, so that a call never finds its
    # K/V in L2 from the previous call (each copy's KV is > L2 or R copies are).
    first = make_layers(args.workload, dev, rank, args.num_q_heads, T, args.layers)
    hidden = args.hidden
    if mode == "attention":
        step_bytes = sum(kv_bytes(w.seq_lens) for w in first)
    elif mode == "from_hidden":
        step_bytes = sum(kv_bytes(w.seq_lens) + proj_bytes(w.batch, hidden, args.num_q_heads) for w in first)
    elif mode == "o_proj":
        step_bytes = sum(o_bytes(w.batch, hidden, args.num_q_heads) for w in first)
    else:
        step_bytes = sum(proj_bytes(w.batch, hidden, args.num_q_heads) for w in first)
    cap = 8 if mode == "attention" else 64
    rotate = args.rotate or max(1, min(cap, math.ceil(4 * L2_BYTES / max(step_bytes, 1))))
    step_kv = step_bytes
    # the copies hold the same bytes in different memory, so every timed launch does the same work;
    # the projection modes rotate only their own inputs (the attention's cache is not read there)
    if mode in ("qkv_proj", "o_proj"):
        import dataclasses
        sets = [first] + [[dataclasses.replace(w) for w in first] for r in range(1, rotate)]
    else:
        sets = [first] + [make_layers(args.workload, dev, rank, args.num_q_heads, T, args.layers)
                          for r in range(1, rotate)]
    if mode in ("qkv_proj", "from_hidden"):
        for si, layers in enumerate(sets):
            for li, w in enumerate(layers):
                # per layer and copy: its hidden state, input_norm gain and qkv_proj weight
                w.hidden_in = inputs.hidden_inputs(w.batch, seed=7000 + 100 * rank + li, device=dev, hidden=hidden,
                                                   num_q_heads=args.num_q_heads)
    elif mode == "o_proj":
        for si, layers in enumerate(sets):
            for li, w in enumerate(layers):
                # per layer and copy: its attention output rows and o_proj weight
                w.o_in = inputs.o_proj_inputs(w.batch, seed=8000 + 100 * rank + li, device=dev, hidden=hidden,
                                              num_q_heads=args.num_q_heads)
    calls_per_step = len(first)
    stream = torch.cuda.current_stream(dev)
    sp = ctypes.c_void_p(stream.cuda_stream)

    def prepared(layers):
        out = []
        for w in layers:
            t = dict(qkv=w.qkv, q=w.q_norm_w, k=w.k_norm_w, sl=w.seq_lens.to(dev), bt=w.block_table.to(dev),
                     kc=w.k_cache, vc=w.v_cache,
                     o=torch.empty((*w.qkv.shape[:-1], w.num_q_heads, 128), dtype=torch.bfloat16, device=dev))
            vp = lambda k: ctypes.c_void_p(t[k].data_ptr())
            i32 = lambda k: ctypes.cast(ctypes.c_void_p(t[k].data_ptr()), ctypes.POINTER(ctypes.c_int32))
            if mode in ("qkv_proj", "from_hidden"):
                t.update(w.hidden_in)
                t["qkv"] = torch.empty_like(w.qkv)   # written by the projection
            if mode == "o_proj":
                t.update(ox=w.o_in["x"], w_o=w.o_in["w_o"],
                         y=torch.empty((w.batch, hidden), dtype=torch.bfloat16, device=dev))
            proj = (vp("x"), vp("input_norm_w"), vp("w_qkv"), hidden) if mode in ("qkv_proj", "from_hidden") else ()
            if mode == "o_proj":
                c = (attn.handle, vp("ox"), vp("w_o"), hidden, vp("y"), int(w.batch), sp)
            elif mode == "qkv_proj":
                c = (attn.handle, *proj, vp("qkv"), int(w.batch), sp)
            else:
                c = ((attn.handle, *proj, vp("qkv"), vp("q"), vp("k"), i32("sl"), None, i32("bt"),
                      int(w.block_table.shape[1]), vp("kc"), vp("vc"), int(w.num_pages), vp("o"), int(w.batch))
                     + ((T,) if T > 1 else ()) + (sp,))
            out.append((c, t))
        return out

    calls = [prepared(layers) for layers in sets]
    fn = {"qkv_proj": lib.qwen3_decode_attn_qkv_proj, "from_hidden": lib.qwen3_decode_attn_from_hidden,
          "o_proj": lib.qwen3_decode_attn_o_proj}.get(
        mode, lib.qwen3_decode_attn_append_and_attend_tokens if T > 1 else lib.qwen3_decode_attn_append_and_attend)

    def step(i):
        for c, _ in calls[i % rotate]:
            rc = fn(*c)
            if rc != 0:
                raise binding.QdaError(rc, "append_and_attend")

    clocks = ClockSampler(dev.index).start()
    t_warm = time.perf_counter()
    for i in range(args.warmup):
        step(i)
    rc = attn.check()
    if rc != 0:
        raise binding.QdaError(rc, "device status after warm-up")

    if not headline:
        # a step count whose graph-replayed region lasts at least ~0.1 s
        per0 = graph_plan(10 ** 6, rotate, calls_per_step)[0]
        g = capture_graphs(calls, fn, dev, rotate, per0)
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        est_ms = max(reduce_max(dist, e0.elapsed_time(e1), dev) / per0, 1e-4)
        del g
        args.steps = per0 * max(1, math.ceil(100.0 / (per0 * est_ms)))

    n_launch = args.steps * calls_per_step
    sustained = None
    if args.timing == "graph":
        # The timed region replays CUDA graphs that each hold `per_graph`
        # consecutive steps (step i runs rotation set i % rotate; per_graph is a
        # multiple of rotate, about 32 calls), plus one graph for the remainder:
        # exactly K steps, every call's kernel back to back with no host launch
        # between them. Events bracket the replays.
        per_graph, full, rest = graph_plan(args.steps, rotate, calls_per_step)
        g_full = capture_graphs(calls, fn, dev, rotate, per_graph) if full else None
        g_rest = capture_graphs(calls, fn, dev, rotate, rest) if rest else None
        for g in (g_full, g_rest):
            if g is not None:
                g.replay()
        torch.cuda.synchronize(dev)
        barrier(dist, dev)
        t0 = time.perf_counter()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(full):
            g_full.replay()
        if g_rest is not None:
            g_rest.replay()
        end.record(stream)
        torch.cuda.synchronize(dev)
        t1 = time.perf_counter()
        barrier(dist, dev)
        ms_local = start.elapsed_time(end)
        kernel_ms = [ms_local / n_launch] * n_launch
        del g_full, g_rest
        if headline:
            sustained = sustained_leg(calls, fn, dev, dist, stream, rotate, calls_per_step,
                                      ms_local / args.steps, clocks)
    else:
        t0, t1, ms_local, kernel_ms = timed_eager(args, calls, fn, dev, dist, stream, rotate, calls_per_step)
    clocks.stop()
    rc = attn.check()
    if rc != 0:
        raise binding.QdaError(rc, "device status after the timed region")

    ms = reduce_max(dist, ms_local, dev)
    ms_per_step = ms / args.steps
    # every rotation set has its own lengths (cfg2/cfg5 draw them); average the bytes per step
    def unit_bytes(w):   # what `value` counts: the K/V bytes attended, or the projection's bytes
        if mode == "o_proj":
            return o_bytes(w.batch, hidden, w.num_q_heads)
        return proj_bytes(w.batch, hidden, w.num_q_heads) if mode == "qkv_proj" else kv_bytes(w.seq_lens)

    def alg_bytes(w):
        if mode == "o_proj":
            return o_bytes(w.batch, hidden, w.num_q_heads)
        b = 0 if mode == "qkv_proj" else algorithmic_bytes(w.seq_lens, w.num_q_heads, T)
        return b + (proj_bytes(w.batch, hidden, w.num_q_heads) if mode != "attention" else 0)

    kv_per_step_local = sum(sum(unit_bytes(w) for w in s) for s in (sets[i % rotate] for i in range(args.steps))) / args.steps
    alg_per_step_local = sum(sum(alg_bytes(w) for w in s)
                             for s in (sets[i % rotate] for i in range(args.steps))) / args.steps
    kv_total = reduce_sum(dist, kv_per_step_local, dev)
    value = kv_total / (ms_per_step * 1e-3) / 1e9

    # dominant kernel roofline: algorithmic bytes per launch / mean launch duration
    mean_kernel_ms = reduce_max(dist, statistics.fmean(kernel_ms), dev)
    alg_per_launch = alg_per_step_local / calls_per_step
    peak, peak_kind = hbm_peak()
    achieved = alg_per_launch / (mean_kernel_ms * 1e-3) / 1e9
    if mode == "attention":
        traffic = traffic_per_launch(workload_key(args.workload, args.num_q_heads, T), args.num_q_heads, T)
    elif mode in ("qkv_proj", "o_proj") and args.num_q_heads == 16 and args.hidden == inputs.HIDDEN:
        traffic = traffic_per_launch(f"{args.workload}-{mode}", key="qkv_proj")   # the product launch's
    else:
        traffic = None

    # the other way of timing, for comparison: eager launches with an event pair around each
    if not headline:
        other = None
    elif args.timing == "graph":
        _, _, e_ms, e_kernel = timed_eager(args, calls, fn, dev, dist, stream, rotate, calls_per_step)
        other = {"timing": "eager launches, an event pair around each",
                 "us_per_call": round(reduce_max(dist, e_ms, dev) * 1e3 / n_launch, 3),
                 "kernel_us_mean": round(statistics.fmean(e_kernel) * 1e3, 3),
                 "kernel_us_median": round(statistics.median(e_kernel) * 1e3, 3)}
    else:
        graph = run_graph(args, attn, calls, fn, dev, dist, rotate, calls_per_step, kv_per_step_local)
        other = {"timing": "CUDA graph replay", **graph}
    if attn.check() != 0:
        raise RuntimeError("device status after the comparison timing")

    # end to end: per step the H2D copy of the step's inputs from pinned memory,
    # the call, and the D2H copy of o
    if mode != "attention":
        e2e = run_e2e_proj(args, attn, sets, dev, stream, dist, rotate, mode, fn, unit_bytes)
    elif T == 1:
        e2e = run_e2e(args, attn, sets, dev, stream, dist, rotate)
    else:
        e2e = run_e2e_tokens(args, attn, sets, dev, stream, dist, rotate)

    result = None
    proj_tensor = None
    if mode != "attention":
        tp, tp_kind = tensor_peak()
        flops = o_flops if mode == "o_proj" else proj_flops
        fl = sum(flops(w.batch, hidden, w.num_q_heads) for w in first) / calls_per_step
        t_ach = fl / (mean_kernel_ms * 1e-3) / 1e12
        proj_tensor = {"bound": "tensor", "achieved": round(t_ach, 1), "peak": tp, "unit": "TFLOP/s",
                       "frac": round(t_ach / tp, 4), "peak_kind": tp_kind,
                       "flops_per_launch": int(fl), "note": "algorithmic flops (2 per multiply-add)" + (
                           "" if mode == "o_proj" else "; the exact hi/lo split issues twice as many on the tensor pipe")}
    if rank == 0:
        clk = clocks.summary(t0, t1, t_warm)
        result = {
            "metric": {"qkv_proj": PROJ_METRIC, "o_proj": O_METRIC}.get(mode, METRIC), "value": round(value, 2),
            "unit": "GB/s",
            "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6),
            "us_per_call": round(ms_per_step * 1e3 / calls_per_step, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "io_dtype": "bf16", "data": "synthetic (seeded; N(0,1) bf16 qkv and cache, gains 1+U(-0.5,0.5))",
            "config": {"workload": f"{args.workload}: {WORKLOADS[args.workload]}"
                                   + ("" if not (args.workload == "cfg3" and args.layers > 0)
                                      else f" (first {calls_per_step} of the 28 layers only)")
                                   + ("" if args.num_q_heads == 16 else f", {args.num_q_heads} query heads")
                                   + ("" if T == 1 else f", {T} new tokens per sequence (causal among them)")
                                   + {"attention": "", "from_hidden": f", from the hidden state (input_norm + "
                                      f"qkv_proj of x [B, {hidden}], then the attention step)",
                                      "qkv_proj": f": input_norm + qkv_proj only (x [B, {hidden}] -> qkv)",
                                      "o_proj": f": attn.o_proj only (o [B, {args.num_q_heads} x 128] -> "
                                                f"y [B, {hidden}])"}[mode],
                       "op": mode, "batch": first[0].batch, "layers_per_step": calls_per_step, "new_tokens": T,
                       "sum_seq_lens_per_step": int(sum(int(w.seq_lens.sum()) for w in first)),
                       "page_size": 16, "heads": f"{args.num_q_heads} q / 8 kv, D=128",
                       "l2": f"{rotate} resident input sets rotated; {rotate * step_kv / 1e9:.2f} GB of KV cycled "
                             f"(> {L2_BYTES / 2**20:.0f} MiB L2)",
                       "grid_ctas": attn.grid_ctas, "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                         "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                         "traffic": traffic, "algorithmic_bytes_per_launch": int(alg_per_launch),
                         "kernel_us_mean": round(mean_kernel_ms * 1e3, 3),
                         "kernel_us_median": round(statistics.median(kernel_ms) * 1e3, 3)},
            "e2e": e2e,
            **({"roofline_tensor": proj_tensor} if proj_tensor is not None else {}),
            "timing": ("CUDA graph replay: graphs of %d consecutive steps (plus one for the remainder), "
                       "exactly K steps between two events; per-launch duration = region time / launches"
                       % graph_plan(args.steps, rotate, calls_per_step)[0]) if args.timing == "graph"
                      else "eager launches, an event pair around each; per-launch duration = mean of the pairs",
            ("eager" if args.timing == "graph" else "graph"): other,
            "seq_per_s": round(first[0].batch / (ms_per_step * 1e-3) * world, 1),
            # the 16-head attention: one launch per call, the tensor-core attention two (attention,
            # combine) or three per prefill chunk (grouped_launches); the projection two (split,
            # product), o_proj one
            "gpu_launches": n_launch * ({"qkv_proj": 2, "o_proj": 1, "from_hidden": 2}.get(mode, 0)
                                        + (0 if mode in ("qkv_proj", "o_proj") else
                                           (1 if kernel_key(args.num_q_heads, T) == 16 else grouped_launches(args)))),
            "clocks": clk,
        }
    if dist is not None:
        dist.barrier(device_ids=[dev.index])
    attn.close()
    if result is not None and sustained is not None:
        result["sustained"] = sustained
    if headline and rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores, _ = host_cpu()
        if mode == "attention":
            result["cpu_baseline"] = cpu_baseline(first)
            if cores > 1:
                result["cpu_baseline_all_cores"] = cpu_baseline(first, seconds=8.0, threads=cores)
        else:
            result["cpu_baseline"] = cpu_baseline_proj(first, mode)
    if result is not None and not headline:
        # the per-configuration entry: the same figures as the headline, for this workload
        keep = ("value", "unit", "steps", "warmup", "ms_per_step", "us_per_call", "seq_per_s", "roofline", "e2e",
                "clocks", "gpu_launches")
        result = {"config": result["config"]["workload"], "sum_seq_lens_per_step":
                  result["config"]["sum_seq_lens_per_step"], "l2": result["config"]["l2"],
                  **{k: result[k] for k in keep},
                  "timing": "CUDA graph replay of the steps, region of at least ~0.1 s between two events"}
    return result


def sustained_leg(calls, fn, dev, dist, stream, rotate, calls_per_step, est_ms_per_step, clocks):
    """Back-to-back replays of one graph for at least 0.5 s of device time, so
    that the clock sampler sees the timed region itself (the headline region
    can be shorter than its sampling period). Returns µs per call and the
    clocks of that window."""
    per = graph_plan(10 ** 6, rotate, calls_per_step)[0]
    g = capture_graphs(calls, fn, dev, rotate, per)
    g.replay()
    reps = max(1, math.ceil(500.0 / max(per * est_ms_per_step, 1e-4)))
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    t0 = time.perf_counter()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(reps):
        g.replay()
    end.record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.perf_counter()
    barrier(dist, dev)
    ms = reduce_max(dist, start.elapsed_time(end), dev)
    del g
    return {"steps": reps * per, "seconds": round(ms / 1e3, 3),
            "us_per_call": round(ms * 1e3 / (reps * per * calls_per_step), 3),
            "timing": f"{reps} back-to-back replays of one CUDA graph of {per} steps between two events",
            "clocks": clocks.summary(t0, t1, t0)}


def graph_plan(steps: int, rotate: int, calls_per_step: int):
    """(steps per graph, full graphs, steps in the remainder graph): the steps per
    graph are a multiple of the rotation count and hold about 32 calls."""
    per_graph = rotate * max(1, math.ceil(32 / (rotate * calls_per_step)))
    per_graph = min(per_graph, rotate * max(1, steps // rotate))
    full = steps // per_graph
    return per_graph, full, steps - full * per_graph


def capture_graphs(calls, fn, dev, rotate, steps):
    """One CUDA graph holding `steps` consecutive steps from step 0 (step i runs
    rotation set i % rotate)."""
    from decode_attention_qk_b200 import binding
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        sp = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
        for i in range(steps):
            for c, _ in calls[i % rotate]:
                rc = fn(*c[:-1], sp)
                if rc != 0:
                    raise binding.QdaError(rc, "capture")
    torch.cuda.current_stream(dev).wait_stream(cap)
    return g


def timed_eager(args, calls, fn, dev, dist, stream, rotate, calls_per_step):
    """K steps of eager launches with an event pair around every launch.
    Returns (t0, t1, region ms, per-launch ms list)."""
    from decode_attention_qk_b200 import binding
    n_launch = args.steps * calls_per_step
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * n_launch)]
    barrier(dist, dev)
    t0 = time.perf_counter()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    k = 0
    for i in range(args.steps):
        for c, _ in calls[i % rotate]:
            ev[2 * k].record(stream)
            rc = fn(*c)
            ev[2 * k + 1].record(stream)
            if rc != 0:
                raise binding.QdaError(rc, "append_and_attend")
            k += 1
    end.record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.perf_counter()
    barrier(dist, dev)
    return t0, t1, start.elapsed_time(end), [ev[2 * j].elapsed_time(ev[2 * j + 1]) for j in range(n_launch)]


def run_graph(args, attn, calls, fn, dev, dist, rotate, calls_per_step, kv_per_step):
    """µs per call when the K steps are replayed from CUDA graphs (as in the
    default timed region), for the line timed eagerly."""
    per_graph, full, rest = graph_plan(args.steps, rotate, calls_per_step)
    g_full = capture_graphs(calls, fn, dev, rotate, per_graph) if full else None
    g_rest = capture_graphs(calls, fn, dev, rotate, rest) if rest else None
    stream = torch.cuda.current_stream(dev)
    for g in (g_full, g_rest):
        if g is not None:
            g.replay()
    barrier(dist, dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(full):
        g_full.replay()
    if g_rest is not None:
        g_rest.replay()
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    if attn.check() != 0:
        raise RuntimeError("device status after the graph replays")
    ms = reduce_max(dist, start.elapsed_time(end), dev)
    ms_per_step = ms / args.steps
    kv_total = reduce_sum(dist, kv_per_step, dev)
    del g_full, g_rest
    return {"us_per_call": round(ms_per_step * 1e3 / calls_per_step, 3), "ms_per_step": round(ms_per_step, 6),
            "value": round(kv_total / (ms_per_step * 1e-3) / 1e9, 2), "unit": "GB/s", "steps": args.steps,
            "steps_per_graph": per_graph}


def run_e2e_proj(args, attn, sets, dev, stream, dist, rotate, mode, fn, unit_bytes):
    """End to end for the projection modes: x copied from pinned host memory into
    the device buffer, the call, and the result (qkv, or o) copied back."""
    from decode_attention_qk_b200 import binding
    sp = ctypes.c_void_p(stream.cuda_stream)
    host = []
    for layers in sets:
        hl = []
        for w in layers:
            x_dev = w.o_in["x"] if mode == "o_proj" else w.hidden_in["x"]
            if mode == "o_proj":
                out_dev = torch.empty((w.batch, w.o_in["w_o"].shape[0]), dtype=torch.bfloat16, device=dev)
            elif mode == "qkv_proj":
                out_dev = torch.empty_like(w.qkv)
            else:
                out_dev = torch.empty((w.batch, w.num_q_heads, 128), dtype=torch.bfloat16, device=dev)
            qkv_dev = out_dev if mode != "from_hidden" else torch.empty_like(w.qkv)
            h = dict(x=x_dev.cpu().pin_memory(), out=torch.empty(out_dev.shape, dtype=torch.bfloat16).pin_memory(),
                     sl=w.seq_lens.clone().pin_memory(), bt=w.block_table.clone().pin_memory())
            d = dict(x=x_dev, out=out_dev, sl=w.seq_lens.to(dev), bt=w.block_table.to(dev))
            vp = lambda t: ctypes.c_void_p(t.data_ptr())
            i32 = lambda t: ctypes.cast(ctypes.c_void_p(t.data_ptr()), ctypes.POINTER(ctypes.c_int32))
            if mode == "o_proj":
                c = (attn.handle, vp(d["x"]), vp(w.o_in["w_o"]), int(out_dev.shape[1]), vp(out_dev), int(w.batch), sp)
                hl.append((c, h, d, qkv_dev))
                continue
            proj = (vp(d["x"]), vp(w.hidden_in["input_norm_w"]), vp(w.hidden_in["w_qkv"]), int(d["x"].shape[1]))
            if mode == "qkv_proj":
                c = (attn.handle, *proj, vp(qkv_dev), int(w.batch), sp)
            else:
                c = (attn.handle, *proj, vp(qkv_dev), vp(w.q_norm_w), vp(w.k_norm_w), i32(d["sl"]), None,
                     i32(d["bt"]), int(w.block_table.shape[1]), vp(w.k_cache), vp(w.v_cache), int(w.num_pages),
                     vp(out_dev), int(w.batch), sp)
            hl.append((c, h, d, qkv_dev))
        host.append(hl)

    def call(c, h, d):
        d["x"].copy_(h["x"], non_blocking=True)
        if mode == "from_hidden":
            d["sl"].copy_(h["sl"], non_blocking=True)
            d["bt"].copy_(h["bt"], non_blocking=True)
        rc = fn(*c)
        if rc != 0:
            raise binding.QdaError(rc, mode)
        h["out"].copy_(d["out"], non_blocking=True)

    for i in range(args.warmup):
        for c, h, d, _ in host[i % rotate]:
            call(c, h, d)
    barrier(dist, dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    h2d = d2h = 0
    for i in range(args.steps):
        for c, h, d, _ in host[i % rotate]:
            call(c, h, d)
            h2d += h["x"].nbytes + (h["sl"].nbytes + h["bt"].nbytes if mode == "from_hidden" else 0)
            d2h += h["out"].nbytes
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    if attn.check() != 0:
        raise RuntimeError("device status after the e2e region")
    ms = reduce_max(dist, start.elapsed_time(end), dev) / args.steps
    units = sum(sum(unit_bytes(w) for w in sets[i % rotate]) for i in range(args.steps)) / args.steps
    total = reduce_sum(dist, units, dev)
    return {"value": round(total / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d // args.steps), "d2h_bytes_per_step": int(d2h // args.steps),
            "ms_per_step": round(ms, 6),
            "api": f"pinned host->device copy of x + qwen3_decode_attn_{mode} + result device->host"}


def run_e2e(args, attn, sets, dev, stream, dist, rotate):
    from decode_attention_qk_b200 import binding
    lib = binding.load_library()
    sp = ctypes.c_void_p(stream.cuda_stream)
    host = []
    for layers in sets:
        hl = []
        for w in layers:
            h = dict(qkv=w.qkv.cpu().pin_memory(), sl=w.seq_lens.clone().pin_memory(),
                     bt=w.block_table.clone().pin_memory(),
                     o=torch.empty((w.batch, w.num_q_heads, 128), dtype=torch.bfloat16).pin_memory())
            c = (attn.handle, ctypes.c_void_p(h["qkv"].data_ptr()), ctypes.c_void_p(w.q_norm_w.data_ptr()),
                 ctypes.c_void_p(w.k_norm_w.data_ptr()),
                 ctypes.cast(ctypes.c_void_p(h["sl"].data_ptr()), ctypes.POINTER(ctypes.c_int32)), None,
                 ctypes.cast(ctypes.c_void_p(h["bt"].data_ptr()), ctypes.POINTER(ctypes.c_int32)),
                 int(w.block_table.shape[1]), ctypes.c_void_p(w.k_cache.data_ptr()),
                 ctypes.c_void_p(w.v_cache.data_ptr()), int(w.num_pages), ctypes.c_void_p(h["o"].data_ptr()),
                 int(w.batch), sp)
            hl.append((c, h, w))
        host.append(hl)
    fn = lib.qwen3_decode_attn_append_and_attend_host
    for i in range(args.warmup):
        for c, _, _ in host[i % rotate]:
            fn(*c)
    h2d = sum(h["qkv"].nbytes + h["sl"].nbytes + h["bt"].nbytes for i in range(args.steps)
              for _, h, _ in host[i % rotate])
    d2h = sum(h["o"].nbytes for i in range(args.steps) for _, h, _ in host[i % rotate])

    def eager():
        for i in range(args.steps):
            for c, h, w in host[i % rotate]:
                rc = fn(*c)
                if rc != 0:
                    raise binding.QdaError(rc, "append_and_attend_host")

    ms_eager = time_region(dist, dev, stream, eager) / args.steps
    ms_graph, per_graph = None, None
    if args.timing == "graph":
        # the same calls (copies in, the step, o copied out) replayed from CUDA graphs
        calls = [[(c, None) for c, _, _ in hl] for hl in host]
        per_graph, full, rest = graph_plan(args.steps, rotate, len(host[0]))
        g_full = capture_graphs(calls, fn, dev, rotate, per_graph) if full else None
        g_rest = capture_graphs(calls, fn, dev, rotate, rest) if rest else None

        def replay():
            for _ in range(full):
                g_full.replay()
            if g_rest is not None:
                g_rest.replay()

        replay()
        ms_graph = time_region(dist, dev, stream, replay) / args.steps
        del g_full, g_rest
    if attn.check() != 0:
        raise RuntimeError("device status after the e2e region")
    kv = sum(sum(kv_bytes(w.seq_lens) for w in sets[i % rotate]) for i in range(args.steps)) / args.steps
    kv_total = reduce_sum(dist, kv, dev)
    ms = ms_graph if ms_graph is not None else ms_eager
    out = {"value": round(kv_total / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
           "h2d_bytes_per_step": int(h2d // args.steps), "d2h_bytes_per_step": int(d2h // args.steps),
           "ms_per_step": round(ms, 6), "api": "qwen3_decode_attn_append_and_attend_host",
           "host_buffers": "page-locked and mapped: qkv, seq_lens and the block table read across the host "
                           "link by one stage-in launch; o written there by the attention kernel"}
    if ms_graph is not None:
        out["timing"] = f"the calls replayed from CUDA graphs of {per_graph} steps, copies included"
        out["eager"] = {"value": round(kv_total / (ms_eager * 1e-3) / 1e9, 2), "ms_per_step": round(ms_eager, 6)}
    return out


def time_region(dist, dev, stream, body) -> float:
    """Milliseconds `body` takes on the device, between two events (max over ranks)."""
    barrier(dist, dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    body()
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    return reduce_max(dist, start.elapsed_time(end), dev)


def run_e2e_tokens(args, attn, sets, dev, stream, dist, rotate):
    """End to end for T new tokens: the per-step tensors (qkv, seq_lens, block
    table) copied from pinned host memory into device buffers, the call
    through qwen3_decode_attn_append_and_attend_tokens, and o copied back."""
    from decode_attention_qk_b200 import binding
    lib = binding.load_library()
    sp = ctypes.c_void_p(stream.cuda_stream)
    T = args.new_tokens
    host = []
    for layers in sets:
        hl = []
        for w in layers:
            h = dict(qkv=w.qkv.cpu().pin_memory(), sl=w.seq_lens.clone().pin_memory(),
                     bt=w.block_table.clone().pin_memory(),
                     o=torch.empty((w.batch, T, w.num_q_heads, 128), dtype=torch.bfloat16).pin_memory())
            d = {k: torch.empty_like(v, device=dev) for k, v in h.items()}
            c = (attn.handle, ctypes.c_void_p(d["qkv"].data_ptr()), ctypes.c_void_p(w.q_norm_w.data_ptr()),
                 ctypes.c_void_p(w.k_norm_w.data_ptr()),
                 ctypes.cast(ctypes.c_void_p(d["sl"].data_ptr()), ctypes.POINTER(ctypes.c_int32)), None,
                 ctypes.cast(ctypes.c_void_p(d["bt"].data_ptr()), ctypes.POINTER(ctypes.c_int32)),
                 int(w.block_table.shape[1]), ctypes.c_void_p(w.k_cache.data_ptr()),
                 ctypes.c_void_p(w.v_cache.data_ptr()), int(w.num_pages), ctypes.c_void_p(d["o"].data_ptr()),
                 int(w.batch), T, sp)
            hl.append((c, h, d))
        host.append(hl)
    fn = lib.qwen3_decode_attn_append_and_attend_tokens

    def call(c, h, d):
        for k in ("qkv", "sl", "bt"):
            d[k].copy_(h[k], non_blocking=True)
        rc = fn(*c)
        if rc != 0:
            raise binding.QdaError(rc, "append_and_attend_tokens")
        h["o"].copy_(d["o"], non_blocking=True)

    for i in range(args.warmup):
        for c, h, d in host[i % rotate]:
            call(c, h, d)
    barrier(dist, dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    h2d = d2h = 0
    for i in range(args.steps):
        for c, h, d in host[i % rotate]:
            call(c, h, d)
            h2d += h["qkv"].nbytes + h["sl"].nbytes + h["bt"].nbytes
            d2h += h["o"].nbytes
    end.record(stream)
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    if attn.check() != 0:
        raise RuntimeError("device status after the e2e region")
    ms = reduce_max(dist, start.elapsed_time(end), dev) / args.steps
    kv = sum(sum(kv_bytes(w.seq_lens) for w in sets[i % rotate]) for i in range(args.steps)) / args.steps
    kv_total = reduce_sum(dist, kv, dev)
    return {"value": round(kv_total / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d // args.steps), "d2h_bytes_per_step": int(d2h // args.steps),
            "ms_per_step": round(ms, 6),
            "api": "pinned host->device copies + qwen3_decode_attn_append_and_attend_tokens + o device->host"}


# ----------------------------------------------------------------------------
# reference arm: the float64 oracle on the host cores

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    cores, cpu_model = host_cpu()
    if args.op in ("qkv_proj", "o_proj") or args.from_hidden:
        run_reference_proj(args, cores, cpu_model)
        return
    oracle.set_threads(cores)
    layers = make_layers(args.workload, "cpu", 0, args.num_q_heads, args.new_tokens)
    # size each step's sample so that warm-up + timed steps take ~2 minutes
    probe = min(range(layers[0].batch), key=lambda b: int(layers[0].seq_lens[b]))
    dt = time_oracle(compact_host(layers[0], [probe]))
    rate = max(int(layers[0].seq_lens[probe]) * KV_BYTES_PER_TOKEN / max(dt, 1e-6), 1e6)
    per_step_budget = rate * min(20.0, 120.0 / max(1, args.steps + args.warmup))
    # a rotating window over the step's sequences
    flat = [(li, b) for li, w in enumerate(layers) for b in range(w.batch)]
    pos = 0

    def sample():
        nonlocal pos
        got, total = {}, 0
        while True:
            li, b = flat[pos % len(flat)]
            pos += 1
            got.setdefault(li, []).append(b)
            total += int(layers[li].seq_lens[b]) * KV_BYTES_PER_TOKEN
            if total >= per_step_budget or len(got.get(li, [])) >= layers[li].batch:
                return [(li, s) for li, s in got.items()], total

    for _ in range(args.warmup):
        picked, _ = sample()
        for li, s in picked:
            time_oracle(compact_host(layers[li], s))
    elapsed, nbytes, nseq = 0.0, 0, 0
    for _ in range(args.steps):
        picked, total = sample()
        for li, s in picked:
            elapsed += time_oracle(compact_host(layers[li], s))
            nseq += len(s)
        nbytes += total
    value = nbytes / elapsed / 1e9
    ms_per_step = elapsed * 1e3 / args.steps
    all_seq = sum(w.batch for w in layers)
    sample_desc = (f"per step a window of the step's sequences ({nbytes / args.steps / 1e6:.1f} MB of KV, "
                   f"{nseq / args.steps:.1f} of {all_seq} sequences on average), {cores} threads")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; same recipe as the GPU arm, drawn on the host)",
        "config": {"workload": f"{args.workload}: {WORKLOADS[args.workload]}"
                               + ("" if args.num_q_heads == 16 else f", {args.num_q_heads} query heads")
                               + ("" if args.new_tokens == 1 else
                                  f", {args.new_tokens} new tokens per sequence (causal among them)"),
                   "batch": layers[0].batch, "layers_per_step": len(layers), "new_tokens": args.new_tokens,
                   "page_size": 16,
                   "heads": f"{args.num_q_heads} q / 8 kv, D=128"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": sample_desc, "cpu_model": cpu_model},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_reference_proj(args, cores, cpu_model):
    """The reference arm of the projection modes: the oracle's input_norm +
    qkv_proj (and, from the hidden state, the attention too), per step a
    bounded sample."""
    mode = args.op if args.op in ("qkv_proj", "o_proj") else "from_hidden"
    layers = make_layers(args.workload, "cpu", 0, args.num_q_heads, 1)
    for li, w in enumerate(layers):
        if mode == "o_proj":
            w.o_in = inputs.o_proj_inputs(w.batch, seed=8000 + li, device="cpu", hidden=args.hidden,
                                          num_q_heads=args.num_q_heads)
        else:
            w.hidden_in = inputs.hidden_inputs(w.batch, seed=7000 + li, device="cpu", hidden=args.hidden,
                                               num_q_heads=args.num_q_heads)
    budget = min(20.0, 120.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline_proj(layers, mode, seconds=budget, threads=cores)
    runs = [cpu_baseline_proj(layers, mode, seconds=budget, threads=cores) for _ in range(args.steps)]
    elapsed = sum(r["seconds"] for r in runs)
    value = sum(r["value"] * r["seconds"] for r in runs) / elapsed
    print(json.dumps({
        "impl": "reference", "metric": {"qkv_proj": PROJ_METRIC, "o_proj": O_METRIC}.get(mode, METRIC),
        "value": round(value, 4),
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(elapsed * 1e3 / args.steps, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; same recipe as the GPU arm, drawn on the host)",
        "config": {"workload": f"{args.workload}: {WORKLOADS[args.workload]}, {mode}", "op": mode},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": runs[0]["sample"], "cpu_model": cpu_model},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="cfg2")
    ap.add_argument("--num-q-heads", type=int, choices=[16, 32, 40, 64], default=16,
                    help="query heads: 16 = Qwen3-0.6B (the default workload); 32/40/64 = 4B-8B/14B/32B")
    ap.add_argument("--new-tokens", type=int, default=1,
                    help="new tokens per sequence, causal among themselves (1 = decode; up to 16 query rows "
                         "per kv head in one launch of the decode-shaped kernel, longer blocks as the chunked "
                         "prefill)")
    ap.add_argument("--timing", choices=["graph", "eager"], default="graph",
                    help="timed region: CUDA graph replay of the steps (default) or eager launches with "
                         "an event pair around each; the line also carries the other figure")
    ap.add_argument("--op", choices=["step", "qkv_proj", "o_proj"], default="step",
                    help="step: the attention step (default); qkv_proj: input_norm + qkv_proj alone; "
                         "o_proj: attn.o_proj alone")
    ap.add_argument("--from-hidden", action="store_true",
                    help="each call starts from the hidden state: input_norm + qkv_proj, then the attention step")
    ap.add_argument("--hidden", type=int, default=inputs.HIDDEN,
                    help="hidden size of the projection modes (1024 for Qwen3-0.6B; 2560, 4096, 5120 for 4B/8B/14B-32B)")
    ap.add_argument("--rotate", type=int, default=0, help="resident input sets cycled (0: enough to defeat L2)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=0,
                    help="cfg3 only: time the first N of its 28 layers (0: all; for profiling one launch)")
    ap.add_argument("--no-per-config", dest="per_config", action="store_false",
                    help="skip the other configurations the default 1-GPU run also times (per_config)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
