"""attn_fwd_host on a B200: host operands in, the forward, host outputs back,
with the copies overlapped with the computation in chunks (row ranges of one
batch, or whole batches). Checked bit for bit against attn_fwd on device
operands (chunks are whole 256-row work units and take the whole call's
schedule, so nothing may differ) and against the FP64 oracle within the BF16 /
FP16 bars, for several chunks per batch, ragged tails, whole-batch chunks,
more than 16 batches, GQA and every mask mode."""

from __future__ import annotations

import math

import pytest
import torch

import head_attention_streaming_b200 as hasb
import oracle
from head_attention_streaming_b200 import inputs
from test_parity_gpu import _check, _pbound

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_ok):
    torch.cuda.set_device(0)
    yield
    assert hasb.device_fault(clear=True) == 0


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,d,dtype,mask,off", [
    (1, 5000, 5000, 16, 8, 128, torch.bfloat16, 0, 0),     # 7 row chunks of 768, ragged last
    # causal, two batches of 2 row chunks: the whole call (192 units) runs
    # unsplit, while a 1536-row chunk alone (48 units) would take the pair split
    (2, 3000, 3400, 8, 4, 128, torch.float16, 1, 400),
    (20, 512, 700, 8, 2, 128, torch.bfloat16, 2, 188),     # 10 chunks of 2 whole batches, chunk mask
    (40, 200, 200, 8, 4, 64, torch.float16, 1, 0),         # more than 16 batches: chunks of 14, 14, 12
    (1, 100, 77, 1, 1, 128, torch.bfloat16, 0, 0),         # one chunk smaller than a tile
    (1, 2048, 2048, 8, 8, 256, torch.bfloat16, 1, 0),      # head dim 256, causal, 4 row chunks
])
def test_host_path_equals_device_call_and_oracle(B, Lq, Lk, Hq, Hkv, d, dtype, mask, off):
    assert len(hasb.host_chunks(B, Lq, Hq, d)) == {5000: 7, 3000: 4, 512: 10, 200: 3, 100: 1, 2048: 4}[Lq]
    q, k, v = inputs.make_qkv(B, Lq, Lk, Hq, Hkv, d, dtype, seed=Lq + Lk + d)
    scale = 1.0 / math.sqrt(d)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.full_like(q, float("nan")).pin_memory()
    lh = torch.full((B, Hq, Lq), float("nan"), dtype=torch.float32).pin_memory()
    qd, kd, vd = torch.empty_like(q, device="cuda"), torch.empty_like(k, device="cuda"), torch.empty_like(v, device="cuda")
    od = torch.empty_like(qd)
    ld = torch.empty((B, Hq, Lq), dtype=torch.float32, device="cuda")
    hasb.attn_fwd_host(qh, kh, vh, oh, lh, qd, kd, vd, od, ld, scale=scale, causal=mask, kv_offset=off)
    torch.cuda.current_stream().synchronize()
    o_dev, l_dev = hasb.attn_fwd(q.cuda(), k.cuda(), v.cuda(), scale=scale, causal=mask, kv_offset=off)
    torch.cuda.synchronize()
    assert torch.equal(oh, o_dev.cpu()) and torch.equal(lh, l_dev.cpu())
    f64 = lambda t: t.to(torch.float64).numpy()
    tag = "bf16" if dtype == torch.bfloat16 else "fp16"
    o_ref, lse_ref = oracle.attention_fwd(f64(q), f64(k), f64(v), scale, mask, off)
    _check(oh, lh, o_ref, lse_ref, tag, what="host path", p_bound=_pbound(q, k, v, scale, tag, mask, off))


def test_host_path_without_lse_and_repeated_calls():
    """Two calls in a row into the same buffers (the second call's copies must
    wait for the first call's forwards), LSE not requested."""
    q1, k1, v1 = inputs.make_qkv(1, 1500, 1500, 4, 4, 128, torch.bfloat16, seed=1)
    q2, k2, v2 = inputs.make_qkv(1, 1500, 1500, 4, 4, 128, torch.bfloat16, seed=2)
    bufs = [torch.empty_like(q1, device="cuda") for _ in range(4)]
    outs, keep = [], []
    for q, k, v in ((q1, k1, v1), (q2, k2, v2)):
        oh = torch.empty_like(q).pin_memory()
        # the host buffers must outlive the queued copies (a freed pinned block
        # may be handed to the next pin_memory() before the copy has read it)
        hin = [q.pin_memory(), k.pin_memory(), v.pin_memory()]
        keep.append(hin)
        hasb.attn_fwd_host(*hin, oh, None, *bufs, None)
        outs.append(oh)
    torch.cuda.current_stream().synchronize()
    for (q, k, v), oh in zip(((q1, k1, v1), (q2, k2, v2)), outs):
        o_dev, _ = hasb.attn_fwd(q.cuda(), k.cuda(), v.cuda())
        torch.cuda.synchronize()
        assert torch.equal(oh, o_dev.cpu())
