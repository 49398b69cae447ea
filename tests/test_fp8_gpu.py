"""Unscaled FP8 attention on a B200 against the FP64 oracle (developer guide,
"OptimizedImplConfig": quantized_sdpa casts Q, K, V directly to
float8_e4m3fn and multiplies V by FP8 probabilities).

* The casts (attn_fp8_cast, attn_fp8_cast_vt) are byte work: bit-exact
  against the oracle's e4m3 rounding.
* The attention is compared with the exact attention of the cast values. The
  kernel rounds P to e4m3, which the oracle bounds per element
  (``p_rounding_bound``) and in variance (``p_rounding_var``). Bars: every
  element within that bound + 2^-8 |O| (the bf16 output) + 1e-3; the mean
  squared error within 1.5x the variance bound + the output rounding's; LSE
  (from the unrounded P, float32) within 1e-3.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import head_attention_streaming_b200 as hasb
import oracle
from head_attention_streaming_b200 import inputs
from oracle import fp8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_ok):
    torch.cuda.set_device(0)
    yield
    assert hasb.device_fault(clear=True) == 0


def _bytes_of_oracle(x: torch.Tensor) -> torch.Tensor:
    """e4m3 bytes of the oracle's rounding of x (its values are exact e4m3)."""
    ref = fp8.e4m3(x.to(torch.float64).numpy())
    return torch.from_numpy(ref).to(torch.float8_e4m3fn).view(torch.uint8)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_cast_is_bit_exact(dtype):
    g = torch.Generator().manual_seed(1)
    parts = [torch.randn(40000, generator=g) * s for s in (1e-3, 0.05, 1.0, 40.0, 600.0)]
    x = torch.cat(parts + [torch.tensor([0.0, -0.0, 448.0, -448.0, 464.0, 1e4, -1e4, 2.0 ** -10,
                                         -2.0 ** -10, 2.0 ** -11, 1.0625, 1.1875])])
    x = torch.cat([x, torch.zeros((-x.numel()) % 8)]).to(dtype)
    y = hasb.fp8_cast(x.cuda())
    torch.cuda.synchronize()
    got = y.cpu().view(torch.uint8)
    want = _bytes_of_oracle(x)
    assert torch.equal(got, want), int((got != want).sum())


@pytest.mark.parametrize("B,Lk,Hkv,d,pitch", [(2, 700, 3, 128, None), (1, 64, 1, 64, 128),
                                              (1, 1, 2, 128, None), (3, 129, 2, 192, 160)])
def test_transposed_cast_is_bit_exact_and_leaves_the_padding(B, Lk, Hkv, d, pitch):
    g = torch.Generator().manual_seed(Lk)
    v = (torch.randn(B, Lk, Hkv, d, generator=g) * 3.0).to(torch.bfloat16)
    pitch = pitch if pitch is not None else (Lk + 15) // 16 * 16
    out = torch.full((B, Hkv, d, pitch), 0x55, dtype=torch.uint8, device="cuda").view(torch.float8_e4m3fn)
    hasb.fp8_cast_vt(v.cuda(), pitch=pitch, out=out)
    torch.cuda.synchronize()
    got = out.cpu().view(torch.uint8)
    want = _bytes_of_oracle(v).permute(0, 2, 3, 1)           # [B, Hkv, d, Lk]
    assert torch.equal(got[..., :Lk], want)
    assert bool((got[..., Lk:] == 0x55).all())


def _fp8_case(B, Lq, Lk, Hq, Hkv, mask, off, seed, rows=None):
    d = 128
    q, k, v = inputs.make_qkv(B, Lq, Lk, Hq, Hkv, d, torch.bfloat16, seed=seed)
    scale = 1.0 / math.sqrt(d)
    q8, k8, vt8 = hasb.fp8_cast(q.cuda()), hasb.fp8_cast(k.cuda()), hasb.fp8_cast_vt(v.cuda())
    o, lse = hasb.attn_fwd_fp8(q8, k8, vt8, scale=scale, causal=mask, kv_offset=off)
    torch.cuda.synchronize()
    f64 = lambda t: t.to(torch.float64).numpy()
    o_ref, lse_ref = fp8.attention_fp8(f64(q), f64(k), f64(v), scale, mask, off, rows=rows)
    bound = fp8.p_rounding_bound(f64(q), f64(k), f64(v), scale, mask, off, rows=rows)
    var = fp8.p_rounding_var(f64(q), f64(k), f64(v), scale, mask, off, rows=rows)
    o_c, l_c = f64(o.cpu()), f64(lse.cpu())
    if rows is not None:
        o_c, l_c = o_c[:, rows], l_c[:, :, rows]
    err = np.abs(o_c - o_ref)
    what = f"fp8 {B}x{Lq}x{Lk} {Hq}/{Hkv} mask {mask}"
    assert np.isfinite(o_c).all(), what
    excess = err - (bound + 2.0 ** -8 * np.abs(o_ref) + 1e-3)
    assert excess.max() <= 0, f"{what}: above the P-rounding bound by {excess.max():.3g}"
    out_var = np.mean((2.0 ** -8 * o_ref) ** 2) / 3.0
    ratio = np.mean(err ** 2) / (np.mean(var) + out_var)
    assert ratio <= 1.5, f"{what}: mean squared error {ratio:.3g} x the variance bound"
    assert np.abs(l_c - lse_ref).max() <= 1e-3, what
    return ratio


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,mask,off", [
    (1, 300, 700, 4, 2, 0, 0),       # ragged query and key tails, GQA
    (2, 257, 900, 4, 1, 1, 643),     # causal with an offset, MQA
    (1, 256, 1000, 2, 2, 2, 300),    # streaming chunk
    (1, 1000, 1000, 2, 2, 1, 0),     # causal square
    (3, 64, 64, 2, 2, 0, 0),         # one query tile, mostly padding
    (1, 1, 1, 1, 1, 0, 0),           # one query, one key
])
def test_fp8_attention(B, Lq, Lk, Hq, Hkv, mask, off):
    _fp8_case(B, Lq, Lk, Hq, Hkv, mask, off, seed=11 + Lq)


def test_fp8_attention_video_shape_sampled_rows():
    """20480 tokens x 56 heads (the video DiT's attention shape), 64 sampled rows."""
    rows = inputs.sample_rows(20480, 64, seed=3).numpy()
    _fp8_case(1, 20480, 20480, 56, 56, 0, 0, seed=4, rows=rows)


def test_fp8_attention_is_deterministic_and_takes_the_caller_buffers():
    q, k, v = inputs.make_qkv(2, 500, 800, 8, 2, 128, torch.bfloat16, seed=21)
    q8, k8, vt8 = hasb.fp8_cast(q.cuda()), hasb.fp8_cast(k.cuda()), hasb.fp8_cast_vt(v.cuda())
    o1, l1 = hasb.attn_fwd_fp8(q8, k8, vt8)
    o2 = torch.empty_like(o1)
    l2 = torch.empty_like(l1)
    hasb.attn_fwd_fp8(q8, k8, vt8, out=o2, lse=l2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
