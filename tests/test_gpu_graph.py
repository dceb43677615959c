"""The handle's entry points captured in a CUDA graph and replayed give the
same bytes as eager calls (the bench times both ways)."""
import pytest
import torch

from decode_attention_qk_b200 import binding, inputs
import parity_helpers as ph

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


@pytest.mark.parametrize("hq,T", [(16, 1), (64, 1), (16, 4)])
def test_graph_replay_matches_eager_calls(hq, T):
    from decode_attention_qk_b200 import build
    build.build_library()
    attn = binding.DecodeAttention(device=0, num_q_heads=hq)
    w = inputs.custom([T, 17, 300, 2000, 45], seed=80 + hq + T, device="cuda", gap_fraction=0.2,
                      num_q_heads=hq, new_tokens=T)
    a = ph.device_args(w, DEV)
    k_eager, v_eager = w.k_cache.clone(), w.v_cache.clone()
    o_eager = attn(a["qkv"], a["q_norm_w"], a["k_norm_w"], a["seq_lens"], a["block_table"], k_eager, v_eager)
    assert attn.check() == 0

    k_graph, v_graph = w.k_cache.clone(), w.v_cache.clone()
    o_graph = torch.empty_like(o_eager)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(DEV)
    side.wait_stream(torch.cuda.current_stream(DEV))
    with torch.cuda.graph(g, stream=side):
        attn(a["qkv"], a["q_norm_w"], a["k_norm_w"], a["seq_lens"], a["block_table"], k_graph, v_graph,
             o=o_graph, stream=torch.cuda.current_stream(DEV))
    for _ in range(3):   # replays append the same rows again: the bytes do not change
        g.replay()
    torch.cuda.synchronize(DEV)
    assert attn.check() == 0
    assert torch.equal(o_graph.view(torch.int16), o_eager.view(torch.int16))
    assert torch.equal(k_graph.view(torch.int16), k_eager.view(torch.int16))
    assert torch.equal(v_graph.view(torch.int16), v_eager.view(torch.int16))
    del g
    attn.close()
