"""Head dims 16 and 32 on a B200 against the FP64 oracle: plain, masked,
windowed, key-split and cache-prefix attention (the pages' contract allows
powers of two 16..256; these two run the 64-wide kernel with the columns past
d loaded as zero and not stored). Bars as in the attention parity tests."""

from __future__ import annotations

import math

import pytest
import torch

import head_attention_streaming_b200 as hasb
import oracle
from head_attention_streaming_b200 import inputs
from test_parity_gpu import _check, _pbound

pytestmark = pytest.mark.gpu

f64 = lambda t: t.to(torch.float64).numpy()


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_ok):
    torch.cuda.set_device(0)
    yield
    assert hasb.device_fault(clear=True) == 0


def _qkv(B, Lq, Lk, Hq, Hkv, d, dtype, seed):
    return inputs.make_qkv(B, Lq, Lk, Hq, Hkv, d, dtype, seed=seed)


@pytest.mark.parametrize("d", [16, 32])
@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,dtype,mask,off", [
    (1, 1, 1, 1, 1, torch.bfloat16, 0, 0),
    (2, 257, 300, 4, 2, torch.bfloat16, 0, 0),
    (1, 300, 300, 2, 1, torch.float16, 1, 0),
    (1, 77, 500, 4, 4, torch.bfloat16, 1, 423),
    (1, 200, 700, 8, 2, torch.float16, 2, 300),
])
def test_small_head_dims(d, B, Lq, Lk, Hq, Hkv, dtype, mask, off):
    q, k, v = _qkv(B, Lq, Lk, Hq, Hkv, d, dtype, seed=7 * d + Lq)
    scale = 1.0 / math.sqrt(d)
    o, lse = hasb.attn_fwd(q.cuda(), k.cuda(), v.cuda(), scale=scale, causal=mask, kv_offset=off)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_fwd(f64(q), f64(k), f64(v), scale, mask, off)
    tag = "bf16" if dtype == torch.bfloat16 else "fp16"
    _check(o.cpu(), lse.cpu(), o_ref, lse_ref, tag, what=f"d={d}",
           p_bound=_pbound(q, k, v, scale, tag, mask, off))


@pytest.mark.parametrize("d", [16, 32])
def test_small_head_dims_neighbours_untouched(d):
    """The output's row stride is d: a store of 64 columns would overwrite the
    next head's row. Surround O with sentinels and check they survive."""
    q, k, v = _qkv(1, 130, 200, 3, 1, d, torch.bfloat16, seed=d)
    buf = torch.full((1 * 130 * 3 * d + 2 * 4096,), 7.0, dtype=torch.bfloat16, device="cuda")
    out = buf[4096:4096 + 130 * 3 * d].view(1, 130, 3, d)
    hasb.attn_fwd(q.cuda(), k.cuda(), v.cuda(), out=out)
    torch.cuda.synchronize()
    assert bool((buf[:4096] == 7.0).all()) and bool((buf[-4096:] == 7.0).all())
    o_ref, _ = oracle.attention_fwd(f64(q), f64(k), f64(v), 1.0 / math.sqrt(d), 0, 0)
    assert abs(f64(out.cpu()) - o_ref).max() < 1e-2


@pytest.mark.parametrize("d", [16, 32])
def test_small_head_dims_window_split_and_cache(d):
    q, k, v = _qkv(1, 300, 900, 4, 2, d, torch.bfloat16, seed=3 + d)
    scale = 1.0 / math.sqrt(d)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o, lse = hasb.attn_fwd_window(qc, kc, vc, window=(100, 20), scale=scale, kv_offset=500)
    torch.cuda.synchronize()
    ref = oracle.attention_fwd(f64(q), f64(k), f64(v), scale, oracle.MASK_WINDOW, 500, window=(100, 20))
    _check(o.cpu(), lse.cpu(), *ref, "bf16", what=f"window d={d}",
           p_bound=_pbound(q, k, v, scale, "bf16", oracle.MASK_WINDOW, 500, window=(100, 20)))
    o, lse, used = hasb.attn_fwd_splitkv(qc, kc, vc, n_splits=3, scale=scale)
    torch.cuda.synchronize()
    assert used == 3
    ref = oracle.attention_fwd(f64(q), f64(k), f64(v), scale, 0, 0)
    _check(o.cpu(), lse.cpu(), *ref, "bf16", what=f"split d={d}", p_bound=_pbound(q, k, v, scale, "bf16"))
    # a cache of 1200 slots of which the first 900 are valid
    S = 1200
    kcache = torch.zeros(1, S, 2, d, dtype=torch.bfloat16, device="cuda")
    vcache = torch.zeros_like(kcache)
    kcache[:, :900] = kc
    vcache[:, :900] = vc
    o, lse = hasb.attn_fwd_cache(qc, kcache, vcache, 900, scale=scale, causal=hasb.MASK_CHUNK, kv_offset=600)
    torch.cuda.synchronize()
    ref = oracle.attention_fwd(f64(q), f64(k), f64(v), scale, 2, 600)
    _check(o.cpu(), lse.cpu(), *ref, "bf16", what=f"cache d={d}", p_bound=_pbound(q, k, v, scale, "bf16", 2, 600))


# ---------------------------------------------------------------- d = 256

@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,dtype,mask,off", [
    (1, 1, 1, 1, 1, torch.bfloat16, 0, 0),
    (2, 257, 300, 4, 2, torch.bfloat16, 0, 0),        # ragged query and key tails, GQA
    (1, 300, 300, 2, 1, torch.float16, 1, 0),         # causal, MQA
    (1, 77, 500, 4, 4, torch.bfloat16, 1, 423),       # causal with an offset
    (1, 200, 700, 8, 2, torch.float16, 2, 300),       # streaming chunk
    (1, 640, 640, 2, 2, torch.bfloat16, 0, 0),        # several units per CTA order
])
def test_d256(B, Lq, Lk, Hq, Hkv, dtype, mask, off):
    d = 256
    q, k, v = _qkv(B, Lq, Lk, Hq, Hkv, d, dtype, seed=11 + Lq + Lk)
    scale = 1.0 / math.sqrt(d)
    o, lse = hasb.attn_fwd(q.cuda(), k.cuda(), v.cuda(), scale=scale, causal=mask, kv_offset=off)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_fwd(f64(q), f64(k), f64(v), scale, mask, off)
    tag = "bf16" if dtype == torch.bfloat16 else "fp16"
    _check(o.cpu(), lse.cpu(), o_ref, lse_ref, tag, what="d=256", p_bound=_pbound(q, k, v, scale, tag, mask, off))


def test_d256_large_scores_rescale_and_cache_prefix():
    """Scores that grow along the keys (each KV tile's max above the last by
    more than the lazy-rescale threshold) and a cache prefix of 900 of 1024 slots."""
    d = 256
    q, k, v = _qkv(1, 256, 900, 2, 1, d, torch.bfloat16, seed=77)
    ramp = torch.linspace(0.5, 6.0, 900).view(1, 900, 1, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    kc = torch.zeros(1, 1024, 1, d, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kc[:, :900] = k.cuda()
    vc[:, :900] = v.cuda()
    o, lse = hasb.attn_fwd_cache(q.cuda(), kc, vc, 900, scale=scale, causal=hasb.MASK_CHUNK, kv_offset=644)
    torch.cuda.synchronize()
    o_ref, lse_ref = oracle.attention_fwd(f64(q), f64(k), f64(v), scale, 2, 644)
    _check(o.cpu(), lse.cpu(), o_ref, lse_ref, "bf16", what="d=256 cache",
           p_bound=_pbound(q, k, v, scale, "bf16", 2, 644))


def test_d256_deterministic():
    q, k, v = (t.cuda() for t in _qkv(1, 300, 500, 2, 2, 256, torch.bfloat16, seed=5))
    a, la = hasb.attn_fwd(q, k, v)
    b, lb = hasb.attn_fwd(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("window,off", [((100, 20), 500), ((0, 0), 0), ((-1, 64), 200)])
def test_d256_window(window, off):
    q, k, v = _qkv(1, 300, 900, 4, 2, 256, torch.bfloat16, seed=8)
    scale = 1.0 / 16
    o, lse = hasb.attn_fwd_window(q.cuda(), k.cuda(), v.cuda(), window=window, scale=scale, kv_offset=off)
    torch.cuda.synchronize()
    ref = oracle.attention_fwd(f64(q), f64(k), f64(v), scale, oracle.MASK_WINDOW, off, window=window)
    _check(o.cpu(), lse.cpu(), *ref, "bf16", what=f"d=256 window {window}",
           p_bound=_pbound(q, k, v, scale, "bf16", oracle.MASK_WINDOW, off, window=window))


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,dtype,mask,off,n", [
    (1, 64, 3000, 4, 1, torch.bfloat16, 0, 0, 5),        # short chunk, long keys
    (1, 200, 1500, 2, 2, torch.float16, 2, 1300, 0),     # chunk mask, automatic split
    (2, 640, 640, 2, 2, torch.bfloat16, 1, 0, 3),        # causal: empty tiles and rows
    (1, 700, 700, 8, 8, torch.bfloat16, 1, 0, 6),        # causal, several units per CTA
])
def test_d256_split(B, Lq, Lk, Hq, Hkv, dtype, mask, off, n):
    q, k, v = _qkv(B, Lq, Lk, Hq, Hkv, 256, dtype, seed=21 + Lq)
    scale = 1.0 / 16
    o, lse, used = hasb.attn_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), n_splits=n, scale=scale,
                                         causal=mask, kv_offset=off)
    torch.cuda.synchronize()
    ref = oracle.attention_fwd(f64(q), f64(k), f64(v), scale, mask, off)
    tag = "bf16" if dtype == torch.bfloat16 else "fp16"
    _check(o.cpu(), lse.cpu(), *ref, tag, what=f"d=256 split {used}",
           p_bound=_pbound(q, k, v, scale, tag, mask, off))
    assert hasb.device_fault(clear=True) == 0
