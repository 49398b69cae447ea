"""GPU parity of the Q/K prologue (RMSNorm then RoPE) against the FP64 oracle,
through the C ABI (``attn_qk_prologue``).

Bound: the kernel computes in float32 and rounds once to the 16-bit type, so
every output element must lie within half a unit in the last place of the
exact value (the final rounding) plus 1e-5 (float32 arithmetic on values of
order one: sums of squares, rsqrt, sincos and the rotation, each a few float32
ulps). A wrong pairing, sign, angle or normalisation axis is off by O(1).
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import head_attention_streaming_b200 as hasb
from head_attention_streaming_b200.inputs import rope_angle_table
from oracle import prologue as qp

pytestmark = pytest.mark.gpu

MANT_BITS = {torch.bfloat16: 7, torch.float16: 10}


def _ulp(x: np.ndarray, dtype) -> np.ndarray:
    mant = MANT_BITS[dtype]
    a = np.abs(x)
    tiny = 2.0 ** -14 if dtype == torch.float16 else 2.0 ** -126
    e = np.floor(np.log2(np.maximum(a, tiny)))
    return np.ldexp(1.0, (e - mant).astype(np.int64))


def _draw(shape, dtype, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (scale * torch.randn(shape, generator=g)).to(dtype)


def _check(got: torch.Tensor, x: torch.Tensor, gamma, eps, scope, angles, style):
    exact = qp.qk_prologue(x.double().numpy(), None if gamma is None else gamma.double().numpy(), eps,
                           scope, None if angles is None else angles.double().numpy(), style)
    g = got.cpu().double().numpy()
    bound = 0.5 * _ulp(exact, x.dtype) + 1e-5
    err = np.abs(g - exact)
    worst = float(np.max(err / bound))
    assert worst <= 1.0, f"max error {float(err.max()):.3e} is {worst:.2f}x the bound"
    # nearly every element is the correctly rounded exact value
    rn = torch.from_numpy(exact).to(x.dtype).double().numpy()
    assert float(np.mean(g != rn)) < 0.01


def _run(B, Lq, Lk, Hq, Hkv, d, dtype, scope, style, eps=1e-6, seed=0, with_k=True, gamma=True,
         pos0=0, scale=1.0, in_place=False):
    q = _draw((B, Lq, Hq, d), dtype, seed, scale)
    k = _draw((B, Lk, Hkv, d), dtype, seed + 1, scale) if with_k else None
    wq = d if scope == qp.NORM_HEAD else Hq * d
    wk = d if scope == qp.NORM_HEAD else Hkv * d
    gq = (1.0 + 0.1 * torch.randn(wq, generator=torch.Generator().manual_seed(seed + 2))) if gamma and scope else None
    gk = (1.0 + 0.1 * torch.randn(wk, generator=torch.Generator().manual_seed(seed + 3))) if gamma and scope else None
    aq = rope_angle_table(Lq, d, style, pos0) if style else None
    ak = rope_angle_table(Lk, d, style, pos0) if (style and with_k) else None
    dev = lambda t: None if t is None else t.cuda()
    qd, kd = dev(q), dev(k)
    out_q = qd if in_place else None
    out_k = kd if in_place else None
    oq, ok = hasb.qk_prologue(qd, kd, norm_scope=scope, eps=eps, gamma_q=dev(gq), gamma_k=dev(gk),
                              rope_style=style, angles_q=dev(aq), angles_k=dev(ak), out_q=out_q,
                              out_k=out_k)
    torch.cuda.synchronize()
    _check(oq, q, gq, eps, scope, aq, style)
    if with_k:
        _check(ok, k, gk, eps, scope, ak, style)
    if in_place:
        assert oq.data_ptr() == qd.data_ptr()


def test_dit_self_attention_prologue_full_size():
    """Q and the new K chunk of the 1785-token DiT workload: head-scope RMSNorm
    (eps 1e-6) and split-half RoPE before the cache update, as in the
    developer guide's Cosmos example; positions of the fourth chunk."""
    _run(1, 1785, 1785, 40, 40, 128, torch.bfloat16, qp.NORM_HEAD, qp.ROPE_SPLIT, pos0=5355, seed=10)


@pytest.mark.parametrize("scope", [qp.NORM_NONE, qp.NORM_HEAD, qp.NORM_INNER])
@pytest.mark.parametrize("style", [qp.ROPE_NONE, qp.ROPE_INTERLEAVED, qp.ROPE_SPLIT])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_scopes_styles_dtypes(scope, style, dtype):
    _run(2, 33, 17, 4, 2, 64, dtype, scope, style, seed=20 + 3 * scope + style)


@pytest.mark.parametrize("d", [16, 32, 128, 256])
@pytest.mark.parametrize("style", [qp.ROPE_INTERLEAVED, qp.ROPE_SPLIT])
def test_head_dims(d, style):
    _run(1, 9, 5, 3, 1, d, torch.bfloat16, qp.NORM_HEAD, style, seed=40 + d + style)


@pytest.mark.parametrize("H,d", [(1, 16), (3, 64), (5, 32), (40, 128), (7, 256)])
def test_ragged_token_widths_inner_scope(H, d):
    """Token widths that fill a partial 256-element chunk (idle lanes)."""
    _run(1, 6, 3, H, 1, d, torch.bfloat16, qp.NORM_INNER, qp.ROPE_SPLIT, seed=60 + H)


def test_query_only_interleaved_no_norm():
    _run(2, 11, 0, 8, 1, 128, torch.float16, qp.NORM_NONE, qp.ROPE_INTERLEAVED, with_k=False,
         pos0=1000, seed=70)


def test_in_place():
    _run(1, 64, 64, 8, 2, 128, torch.bfloat16, qp.NORM_HEAD, qp.ROPE_SPLIT, seed=71, in_place=True)


def test_eps_matters_for_small_inputs():
    """Features of size ~1e-3 have mean square ~1e-6, comparable to eps."""
    _run(1, 16, 16, 2, 2, 64, torch.bfloat16, qp.NORM_HEAD, qp.ROPE_NONE, eps=1e-6, scale=1e-3,
         seed=72)
    _run(1, 16, 16, 2, 2, 64, torch.float16, qp.NORM_INNER, qp.ROPE_NONE, eps=1e-6, scale=1e-3,
         seed=73, gamma=False)


def test_identity_when_nothing_requested_is_bit_exact():
    q = _draw((1, 20, 3, 64), torch.bfloat16, 80).cuda()
    k = _draw((1, 7, 3, 64), torch.bfloat16, 81).cuda()
    oq, ok = hasb.qk_prologue(q, k)
    torch.cuda.synchronize()
    assert torch.equal(oq, q) and torch.equal(ok, k)


def test_invalid_call_raises():
    q = _draw((1, 4, 2, 64), torch.bfloat16, 82).cuda()
    with pytest.raises(ValueError):
        hasb.qk_prologue(q, rope_style=qp.ROPE_SPLIT,
                         angles_q=torch.zeros(3 * 64, device="cuda"))  # wrong table size
    with pytest.raises(hasb.AttnError):
        hasb.qk_prologue(q, rope_style=qp.ROPE_SPLIT)  # RoPE without angles


def test_large_tokens_take_the_one_block_per_token_kernel():
    """A token of 64 heads x 256 features (32 KB) is too large to stage in
    shared memory: the one-block-per-token kernel serves it, same results."""
    _run(1, 20, 12, 64, 8, 256, torch.bfloat16, qp.NORM_HEAD, qp.ROPE_SPLIT, seed=77)
    _run(1, 20, 12, 64, 8, 256, torch.bfloat16, qp.NORM_INNER, qp.ROPE_INTERLEAVED, seed=78)


def test_unaligned_angle_table_takes_the_one_block_per_token_kernel():
    """An angle table that is 4- but not 16-byte aligned cannot be copied by
    cp.async: the direct kernel serves the call."""
    B, L, H, d = 1, 37, 4, 64
    q = _draw((B, L, H, d), torch.bfloat16, 81)
    ang = rope_angle_table(L, d, qp.ROPE_SPLIT, 100)
    buf = torch.zeros(L * d + 1, dtype=torch.float32, device="cuda")
    buf[1:] = ang.reshape(-1).cuda()
    ang_off = buf[1:].view(L, d)                          # data_ptr 4 bytes past a 16-byte boundary
    assert ang_off.data_ptr() % 16 != 0
    oq, _ = hasb.qk_prologue(q.cuda(), None, norm_scope=hasb.NORM_NONE, rope_style=hasb.ROPE_SPLIT,
                             angles_q=ang_off)
    torch.cuda.synchronize()
    _check(oq, q, None, 1e-6, qp.NORM_NONE, ang, qp.ROPE_SPLIT)
