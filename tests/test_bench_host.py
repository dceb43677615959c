"""Host logic of bench.py, on the CPU: byte counts, the JSON contract's
reductions over ranks (gloo, world size 2) and rank-distinct replicas."""
import os
import socket

import types

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from decode_attention_qk_b200 import inputs


def test_byte_counts():
    L = torch.tensor([1, 16, 17, 4096], dtype=torch.int32)
    assert bench.kv_bytes(L) == int(L.sum()) * 4096
    pages = 1 + 1 + 2 + 256
    want = (0 + 15 + 16 + 4095) * 4096 + 4 * 4096 + 4 * 8192 + 4 * 4096 + pages * 4 + 4 * 4 + 512
    assert bench.algorithmic_bytes(L) == want
    # T = 3 new tokens at 32 query heads: L - 3 cached rows read, 3 rows of qkv (12288 B each),
    # 3 k/v rows written and 3 o rows (8192 B each) per sequence
    L = torch.tensor([3, 16, 17, 4096], dtype=torch.int32)
    pages = 1 + 1 + 2 + 256
    want = (0 + 13 + 14 + 4093) * 4096 + 12 * 4096 + 12 * 12288 + 12 * 8192 + pages * 4 + 4 * 4 + 512
    assert bench.algorithmic_bytes(L, 32, 3) == want


def test_projection_byte_and_flop_counts():
    # Qwen3-0.6B: weight 4096 x 1024, x and qkv rows, the gain
    assert bench.proj_bytes(32) == 4096 * 1024 * 2 + 32 * 1024 * 2 + 1024 * 2 + 32 * 4096 * 2
    assert bench.proj_bytes(1, hidden=5120, num_q_heads=64) == 10240 * 5120 * 2 + 5120 * 2 + 5120 * 2 + 10240 * 2
    assert bench.proj_flops(256) == 2 * 256 * 4096 * 1024


def test_kernel_and_workload_keys():
    assert bench.kernel_key(16, 1) == 16
    assert bench.kernel_key(16, 2) == bench.kernel_key(64, 1) == bench.kernel_key(16, 8) == "grouped"
    assert bench.kernel_key(16, 9) == bench.kernel_key(40, 4) == bench.kernel_key(64, 3) == "prefill"
    # prefill chunks of 128 / G tokens, three launches each
    args = types.SimpleNamespace(new_tokens=130, num_q_heads=16)
    assert bench.chunk_tokens(args) == [64, 64, 2] and bench.grouped_launches(args) == 9
    args = types.SimpleNamespace(new_tokens=30, num_q_heads=40)
    assert bench.chunk_tokens(args) == [25, 5]
    args = types.SimpleNamespace(new_tokens=8, num_q_heads=16)
    assert bench.chunk_tokens(args) == [8] and bench.grouped_launches(args) == 2
    assert bench.workload_key("cfg2") == "cfg2"
    assert bench.workload_key("cfg2", 64) == "cfg2-h64"
    assert bench.workload_key("cfg2", 16, 4) == "cfg2-t4"
    with pytest.raises(ValueError):
        bench.make_layers("cfg3", "cpu", 0, 16, 2)
    w = bench.make_layers("cfg2", "cpu", 0, 16, 4)[0]
    assert w.new_tokens == 4 and int(w.seq_lens.min()) >= 4


def test_cpu_baseline_sample_is_bounded():
    layers = [inputs.custom([100, 200, 300, 400], seed=1)]
    picked, total = bench.pick_sample(layers, 250 * 4096)
    assert picked == [(0, [0, 1])] and total == 300 * 4096
    picked, total = bench.pick_sample(layers, 1)
    assert picked == [(0, [0])]


def test_replicas_differ_by_rank():
    a = bench.make_layers("cfg1", "cpu", 0)[0]
    b = bench.make_layers("cfg1", "cpu", 1)[0]
    assert not torch.equal(a.qkv, b.qkv)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    ms = [3.0, 5.0][rank]                 # per-rank elapsed time
    nbytes = [100.0, 300.0][rank]         # per-rank KV bytes per step
    mx = bench.reduce_max(dist, ms, torch.device("cpu"))
    tot = bench.reduce_sum(dist, nbytes, torch.device("cpu"))
    q.put((rank, mx, tot))
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_reductions_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    assert got == [(0, 5.0, 400.0), (1, 5.0, 400.0)]


def test_graph_plan_covers_exactly_the_steps():
    """The timed region's graphs hold exactly K steps; each graph starts on a
    multiple of the rotation count, so step i always runs rotation set i % R."""
    for steps, rotate, calls in [(2000, 2, 1), (1000, 1, 1), (200, 1, 28), (5, 1, 1), (7, 2, 1), (3, 8, 1),
                                 (2000, 8, 1), (1, 1, 1)]:
        per_graph, full, rest = bench.graph_plan(steps, rotate, calls)
        assert per_graph * full + rest == steps
        assert per_graph % rotate == 0 and rest < per_graph or full == 0
        # the fewest rotation cycles that reach 32 calls (unless K steps are fewer)
        assert per_graph == steps or per_graph * calls >= 32 or per_graph == rotate * max(1, steps // rotate)
        assert per_graph == rotate or (per_graph - rotate) * calls < 32
