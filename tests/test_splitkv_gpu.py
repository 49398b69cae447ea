"""Key-split attention (attn_fwd_splitkv) on a B200 against the FP64 oracle:
several CTAs per query pair over disjoint key ranges, merged through the
per-range LSE. Bars as in the attention parity tests."""

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


def _case(B, Lq, Lk, Hq, Hkv, d, dtype, mask, off, n_splits, seed, rows=None):
    q, k, v = inputs.make_qkv(B, Lq, Lk, Hq, Hkv, d, dtype, seed=seed)
    scale = 1.0 / math.sqrt(d)
    o, lse, used = hasb.attn_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), n_splits=n_splits, scale=scale,
                                         causal=mask, kv_offset=off)
    torch.cuda.synchronize()
    f64 = lambda t: t.to(torch.float64).numpy()
    o_ref, lse_ref = oracle.attention_fwd(f64(q), f64(k), f64(v), scale, mask, off, rows=rows)
    o_c, l_c = o.cpu(), lse.cpu()
    if rows is not None:
        o_c, l_c = o_c[:, rows], l_c[:, :, rows]
    tag = "bf16" if dtype == torch.bfloat16 else "fp16"
    _check(o_c, l_c, o_ref, lse_ref, tag, what=f"splits {used}",
           p_bound=_pbound(q, k, v, scale, tag, mask, off, rows=rows))
    return used


@pytest.mark.parametrize("n_splits", [0, 2, 5, 56])
def test_short_chunk_long_cache(n_splits):
    used = _case(1, 256, 7140, 40, 8, 128, torch.bfloat16, inputs.MASK_CHUNK, 6884, n_splits, seed=6)
    assert used == (n_splits if n_splits else used) and used > 1


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,d,dtype,mask,off,n", [
    (2, 100, 1000, 4, 2, 64, torch.float16, 0, 0, 3),     # ragged query tile, ragged last key tile
    (1, 300, 2000, 8, 1, 128, torch.bfloat16, 2, 1500, 4),  # chunk mask: 1800 visible keys
    (1, 1, 4096, 8, 8, 128, torch.bfloat16, 0, 0, 32),    # a single query row, one tile per split
    (3, 64, 513, 2, 2, 64, torch.bfloat16, 0, 0, 0),      # automatic choice
])
def test_shapes(B, Lq, Lk, Hq, Hkv, d, dtype, mask, off, n):
    _case(B, Lq, Lk, Hq, Hkv, d, dtype, mask, off, n, seed=11 + Lq)


def test_one_split_is_attn_fwd_bitwise():
    q, k, v = (t.cuda() for t in inputs.make_qkv(1, 200, 900, 4, 2, 128, torch.bfloat16, seed=12))
    o1, l1, used = hasb.attn_fwd_splitkv(q, k, v, n_splits=1)
    o2, l2 = hasb.attn_fwd(q, k, v)
    torch.cuda.synchronize()
    assert used == 1 and torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,d,dtype,off,n", [
    (2, 2048, 2048, 8, 8, 64, torch.float16, 0, 2),       # the FP16 causal workload's shape
    (1, 1000, 1000, 2, 2, 128, torch.bfloat16, 0, 5),     # many ranges empty for the first tiles
    (1, 300, 1000, 4, 2, 128, torch.bfloat16, 700, 3),    # bottom-right causal with an offset
    (1, 16, 4096, 8, 1, 128, torch.bfloat16, 4080, 0),    # a decode-sized causal chunk, automatic split
    (1, 130, 700, 2, 2, 64, torch.bfloat16, 0, 6),        # rows whose whole range is invisible
])
def test_causal(B, Lq, Lk, Hq, Hkv, d, dtype, off, n):
    """Causal key split: empty partials (tiles or rows that see no key of a
    range) weigh nothing in the merge."""
    _case(B, Lq, Lk, Hq, Hkv, d, dtype, inputs.MASK_CAUSAL, off, n, seed=13 + Lq)


@pytest.mark.parametrize("n", [3, 4, 8, 16])
def test_causal_many_units_per_cta(n):
    """2 x 8 heads x 8 row pairs x n ranges: several units per CTA, many of
    them empty (ranges past a pair's diagonal) next to full ones; a lost
    barrier phase between them would stall the kernel until its wait limit."""
    _case(2, 2048, 2048, 8, 8, 64, torch.float16, inputs.MASK_CAUSAL, 0, n, seed=15 + n)
    assert hasb.device_fault(clear=True) == 0


def test_causal_one_split_is_attn_fwd_bitwise():
    q, k, v = (t.cuda() for t in inputs.make_qkv(1, 300, 900, 4, 2, 128, torch.bfloat16, seed=14))
    o1, l1, used = hasb.attn_fwd_splitkv(q, k, v, n_splits=1, causal=inputs.MASK_CAUSAL, kv_offset=600)
    o2, l2 = hasb.attn_fwd(q, k, v, causal=inputs.MASK_CAUSAL, kv_offset=600)
    torch.cuda.synchronize()
    assert used == 1 and torch.equal(o1, o2) and torch.equal(l1, l2)
