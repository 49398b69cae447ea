"""The attention and streaming calls are stream-ordered and capture into a
CUDA graph: replaying the graph gives the eager results bit for bit (the
library allocates nothing and synchronises nothing during a call)."""

from __future__ import annotations

import pytest
import torch

import head_attention_streaming_b200 as hasb
from head_attention_streaming_b200 import inputs
from head_attention_streaming_b200.inputs import rope_angle_table

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_ok):
    torch.cuda.set_device(0)
    yield
    assert hasb.device_fault(clear=True) == 0


def test_attention_replays_from_a_cuda_graph():
    q, k, v = (t.cuda() for t in inputs.make_qkv(1, 300, 700, 4, 2, 128, torch.bfloat16, seed=90))
    o_ref, l_ref = hasb.attn_fwd(q, k, v, causal=hasb.MASK_CAUSAL, kv_offset=400)
    o = torch.empty_like(q)
    lse = torch.empty_like(l_ref)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        hasb.attn_fwd(q, k, v, causal=hasb.MASK_CAUSAL, kv_offset=400, out=o, lse=lse, stream=s)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_prologue_and_cached_attention_replay_from_a_cuda_graph():
    B, C, H, d = 1, 128, 2, 128
    g = torch.Generator().manual_seed(91)
    q, k, v = (torch.randn(B, C, 4 if i == 0 else H, d, generator=g).to(torch.bfloat16).cuda()
               for i in range(3))
    ang = rope_angle_table(C, d, hasb.ROPE_SPLIT, 0).cuda()
    kc = torch.zeros(B, 2 * C, H, d, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)

    def step(stream=None, out=None, lse=None):
        qr = hasb.stream_update(k, v, kc, vc, 0, q=q, norm_scope=hasb.NORM_HEAD,
                                rope_style=hasb.ROPE_SPLIT, angles_q=ang, angles_k=ang, stream=stream)
        return hasb.attn_fwd_cache(qr, kc, vc, C, out=out, lse=lse, stream=stream)

    o_ref, l_ref = step()
    torch.cuda.synchronize()
    o = torch.empty_like(o_ref)
    lse = torch.empty_like(l_ref)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            step(stream=s, out=o, lse=lse)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
