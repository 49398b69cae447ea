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
                                              (1, 1, 2, 128, None), (3, 129, 2, 256, 160),
                                              (2, 300, 2, 32, None), (1, 77, 3, 16, 96)])
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


def _fp8_case(B, Lq, Lk, Hq, Hkv, mask, off, seed, rows=None, d=128):
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


# ---------------------------------------------------------------- per-token scaled FP8

def _scaled_inputs(B, L, H, d, seed, mag=1.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(B, L, H, d, generator=g) * mag
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("d", [16, 64, 128, 256])
def test_quantize_tokens_is_bit_exact(d):
    from oracle import quantize as qz
    x = _scaled_inputs(2, 37, 3, d, seed=d)
    x[0, 5, 1] = 0.0                                   # an all-zero row takes the floor
    x[1, 7] *= 1e4
    x[1, 8] *= 1e-30
    codes, s = hasb.fp8_quantize_tokens(x.cuda())
    torch.cuda.synchronize()
    c_ref, s_ref = qz.quantize(x.to(torch.float64).numpy(), "e4m3", qz.SLICE, axis=-1)
    want = torch.from_numpy(c_ref).to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(codes.cpu().view(torch.uint8), want)
    got_s = s.cpu()[:, :, :37].numpy()                              # [B, H, L]
    np.testing.assert_array_equal(got_s, s_ref[..., 0].transpose(0, 2, 1))


@pytest.mark.parametrize("B,Lk,Hkv,d", [(2, 700, 3, 128), (1, 5, 2, 64), (1, 1000, 1, 256)])
def test_quantize_vt_is_bit_exact(B, Lk, Hkv, d):
    from oracle import quantize as qz
    v = _scaled_inputs(B, Lk, Hkv, d, seed=Lk)
    v[:, :, 0, 3] = 0.0                                # an all-zero channel
    v[:, :, -1, 5] *= 1e-6
    codes, sv = hasb.fp8_quantize_vt(v.cuda())
    torch.cuda.synchronize()
    c_ref, s_ref = qz.quantize(v.to(torch.float64).numpy(), "e4m3", qz.SLICE, axis=1)
    want = torch.from_numpy(c_ref).to(torch.float8_e4m3fn).view(torch.uint8).permute(0, 2, 3, 1)
    assert torch.equal(codes.cpu().view(torch.uint8)[..., :Lk], want)
    np.testing.assert_array_equal(sv.cpu().numpy(), s_ref[:, 0])


def _fp8_scaled_case(B, Lq, Lk, Hq, Hkv, mask, off, seed, rows=None, mag=1.0, v_scaled=True, d=128):
    q, k, v = inputs.make_qkv(B, Lq, Lk, Hq, Hkv, d, torch.float32, seed=seed)
    q, k, v = ((t * mag).to(torch.bfloat16) for t in (q, k, v))
    scale = 1.0 / math.sqrt(d) / mag ** 2
    q8, sq = hasb.fp8_quantize_tokens(q.cuda())
    k8, sk = hasb.fp8_quantize_tokens(k.cuda())
    if v_scaled:
        vt8, sv = hasb.fp8_quantize_vt(v.cuda())
    else:
        vt8, sv = hasb.fp8_cast_vt(v.cuda()), None
    o, lse = hasb.attn_fwd_fp8_scaled(q8, sq, k8, sk, vt8, sv, scale=scale, causal=mask, kv_offset=off)
    torch.cuda.synchronize()
    f64 = lambda t: t.to(torch.float64).numpy()
    qd, kd, vd = fp8.dequantized_attention_inputs(f64(q), f64(k), f64(v), v_scaled)
    o_ref, lse_ref = oracle.attention_fwd(qd, kd, vd, scale, mask, off, rows=rows)
    bound = fp8.p_rounding_bound(qd, kd, vd, scale, mask, off, rows=rows, cast=False)
    var = fp8.p_rounding_var(qd, kd, vd, scale, mask, off, rows=rows, cast=False)
    o_c, l_c = f64(o.cpu()), f64(lse.cpu())
    if rows is not None:
        o_c, l_c = o_c[:, rows], l_c[:, :, rows]
    err = np.abs(o_c - o_ref)
    what = f"fp8 scaled {B}x{Lq}x{Lk} {Hq}/{Hkv} mask {mask} mag {mag}"
    assert np.isfinite(o_c).all(), what
    excess = err - (bound + 2.0 ** -8 * np.abs(o_ref) + 1e-3 * mag)
    assert excess.max() <= 0, f"{what}: above the P-rounding bound by {excess.max():.3g}"
    out_var = np.mean((2.0 ** -8 * o_ref) ** 2) / 3.0
    ratio = np.mean(err ** 2) / (np.mean(var) + out_var)
    assert ratio <= 1.5, f"{what}: mean squared error {ratio:.3g} x the variance bound"
    assert np.abs(l_c - lse_ref).max() <= 1e-3, what
    return err


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,mask,off", [
    (1, 300, 700, 4, 2, 0, 0),
    (2, 257, 900, 4, 1, 1, 643),
    (1, 256, 1000, 2, 2, 2, 300),
    (3, 64, 64, 2, 2, 0, 0),
    (1, 1, 3, 1, 1, 0, 0),
])
def test_fp8_scaled_attention(B, Lq, Lk, Hq, Hkv, mask, off):
    _fp8_scaled_case(B, Lq, Lk, Hq, Hkv, mask, off, seed=31 + Lq)


def test_fp8_scaled_attention_unscaled_v():
    _fp8_scaled_case(1, 300, 700, 4, 2, 0, 0, seed=5, v_scaled=False)


def test_fp8_scaled_attention_keeps_small_magnitudes():
    """Inputs around 1e-3 (scale compensated): the scaled path stays within
    its bars where a direct e4m3 cast would flush most values to subnormals."""
    _fp8_scaled_case(1, 256, 512, 2, 2, 0, 0, seed=8, mag=1e-3)


def test_fp8_scaled_attention_video_shape_sampled_rows():
    rows = inputs.sample_rows(20480, 48, seed=6).numpy()
    _fp8_scaled_case(1, 20480, 20480, 56, 56, 0, 0, seed=9, rows=rows)


@pytest.mark.parametrize("d", [16, 32, 64])
def test_fp8_small_head_dims(d):
    """d < 128 through the 128-wide e4m3 kernel (zero-filled columns, O chunks
    past d not stored), unscaled and per-token scaled, causal and plain."""
    _fp8_case(2, 300, 700, 4, 2, 0, 0, seed=70 + d, d=d)
    _fp8_case(1, 257, 900, 2, 1, 1, 643, seed=71 + d, d=d)
    _fp8_scaled_case(1, 300, 700, 4, 2, 0, 0, seed=72 + d, d=d)


@pytest.mark.parametrize("B,Lk,Hkv,d", [(2, 700, 3, 32), (1, 65, 2, 16)])
def test_quantize_vt_small_head_dims_bit_exact(B, Lk, Hkv, d):
    from oracle import quantize as qz
    v = _scaled_inputs(B, Lk, Hkv, d, seed=Lk + d)
    codes, sv = hasb.fp8_quantize_vt(v.cuda())
    torch.cuda.synchronize()
    c_ref, s_ref = qz.quantize(v.to(torch.float64).numpy(), "e4m3", qz.SLICE, axis=1)
    want = torch.from_numpy(c_ref).to(torch.float8_e4m3fn).view(torch.uint8).permute(0, 2, 3, 1)
    assert torch.equal(codes.cpu().view(torch.uint8)[..., :Lk], want)
    np.testing.assert_array_equal(sv.cpu().numpy(), s_ref[:, 0])


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,mask,off", [
    (1, 300, 700, 4, 2, 0, 0),
    (2, 257, 900, 2, 1, 1, 643),
    (1, 256, 1000, 2, 2, 2, 300),
])
def test_fp8_head_dim_256(B, Lq, Lk, Hq, Hkv, mask, off):
    """d = 256 through the one-tile e4m3 kernel (two 128-byte chunks per row,
    P of each S buffer in shared memory)."""
    _fp8_case(B, Lq, Lk, Hq, Hkv, mask, off, seed=80 + Lq, d=256)


@pytest.mark.parametrize("mask,off", [(0, 0), (1, 400)])
def test_fp8_scaled_head_dim_256(mask, off):
    _fp8_scaled_case(1, 300, 700, 4, 2, mask, off, seed=85 + mask, d=256)
