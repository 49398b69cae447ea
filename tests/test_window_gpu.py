"""Sliding-window attention (attn_fwd_window) on a B200 against the FP64
oracle (mask 3, window=(left, right)). Bars as in the attention parity tests."""

from __future__ import annotations

import math

import numpy as np
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


def _case(B, Lq, Lk, Hq, Hkv, d, dtype, window, off, seed, rows=None, rounding_terms=True):
    q, k, v = inputs.make_qkv(B, Lq, Lk, Hq, Hkv, d, dtype, seed=seed)
    scale = 1.0 / math.sqrt(d)
    o, lse = hasb.attn_fwd_window(q.cuda(), k.cuda(), v.cuda(), window=window, scale=scale, kv_offset=off)
    torch.cuda.synchronize()
    f64 = lambda t: t.to(torch.float64).numpy()
    o_ref, lse_ref = oracle.attention_fwd(f64(q), f64(k), f64(v), scale, oracle.MASK_WINDOW, off,
                                          rows=rows, window=window)
    o_c, l_c = o.cpu(), lse.cpu()
    if rows is not None:
        o_c, l_c = o_c[:, rows], l_c[:, :, rows]
    tag = "bf16" if dtype == torch.bfloat16 else "fp16"
    pb = _pbound(q, k, v, scale, tag, oracle.MASK_WINDOW, off, rows=rows, window=window) if rounding_terms else None
    _check(o_c, l_c, o_ref, lse_ref, tag, what=f"window {window}", p_bound=pb)


@pytest.mark.parametrize("window", [(256, 256), (100, 0), (0, 100), (300, 37), (-1, 200), (128, -1),
                                    (0, 0), (1, 1), (1000, 1000)])
def test_windows(window):
    _case(1, 700, 700, 4, 2, 128, torch.bfloat16, window, 0, seed=1)


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,d,dtype,window,off", [
    (2, 257, 900, 4, 1, 64, torch.float16, (64, 64), 300),    # offset, ragged query tile
    (1, 1000, 1000, 2, 2, 128, torch.bfloat16, (500, 10), 0),  # tile 0 spans more KV tiles than tile 1
    (1, 130, 4000, 8, 8, 128, torch.bfloat16, (256, 256), 3800),
    (3, 64, 64, 2, 2, 64, torch.bfloat16, (5, 5), 0),         # one query tile, mostly padding
])
def test_shapes(B, Lq, Lk, Hq, Hkv, d, dtype, window, off):
    _case(B, Lq, Lk, Hq, Hkv, d, dtype, window, off, seed=7 + Lq)


def test_video_length_local_window_sampled_rows():
    """A 4096-key local window over the 20480-token video sequence (56 heads)."""
    rows = np.sort(np.random.default_rng(3).choice(20480, size=96, replace=False))
    _case(1, 20480, 20480, 56, 56, 128, torch.bfloat16, (2048, 2047), 0, seed=5, rows=rows,
          rounding_terms=False)


def test_unbounded_and_causal_windows_match_the_other_masks():
    # 64 heads: 192 row pairs, so the causal call takes the two-tile path (a
    # causal call with fewer row pairs than SMs splits each tile's keys over
    # the CTA's two slots and merges them, which rounds differently)
    q, k, v = (t.cuda() for t in inputs.make_qkv(1, 600, 900, 64, 16, 128, torch.bfloat16, seed=9))
    a, la = hasb.attn_fwd_window(q, k, v, window=(-1, -1))
    b, lb = hasb.attn_fwd(q, k, v)
    c, lc = hasb.attn_fwd_window(q, k, v, window=(-1, 0), kv_offset=300)
    d_, ld = hasb.attn_fwd(q, k, v, causal=hasb.MASK_CAUSAL, kv_offset=300)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)
    assert torch.equal(c, d_) and torch.equal(lc, ld)
