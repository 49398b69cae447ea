"""Pins for the 16-bit P-rounding bound (oracle/rounding.py).

The bound says how far rounding the unnormalised probabilities to BF16 / FP16
before P V can move O (the kernel keeps the row sum in float32). It is checked
against things other than its own formula:

* a direct simulation of the rounding (torch's 16-bit casts as the rounding
  step), with the reference at the row max and lagging it by 5.5 nats;
* a hand-built worst case with one key, where the error reaches the relative
  term almost exactly: halving that term (a plausible mistake: counting the
  stored mantissa bits instead of the significant bits) fails it;
* FP16 weights below the smallest normal, where a relative-only bound fails
  and the absolute floor covers the simulation;
* the half-spacing helper against torch's round-to-nearest casts.

Source: developer guide, "Multi Head Attention Definition" (the SDPA equation
the oracle computes); skill page "optimizing-attention-flash", "Quick start"
(the tiled kernel keeps a running max and sum per row).
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import attention_fwd
from oracle.rounding import half_ulp16, p16_rounding_bound

TORCH = {"bf16": torch.bfloat16, "fp16": torch.float16}


def _round16(x, dtype):
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.float32).to(TORCH[dtype]) \
        .to(torch.float64).numpy()


def _simulate(q, k, v, scale, dtype, shift=0.0):
    """O with P = round16(exp(s - m + shift)) against the unrounded row sum; m
    the row max, so the largest P is e^shift (shift >= 0: a lagging reference)."""
    B, Lq, Hq, d = q.shape
    rep = Hq // k.shape[2]
    o = np.zeros((B, Lq, Hq, d))
    for b in range(B):
        for h in range(Hq):
            s = scale * q[b, :, h] @ k[b, :, h // rep].T
            p = np.exp(s - s.max(axis=1, keepdims=True) + shift)
            o[b, :, h] = (_round16(p, dtype) @ v[b, :, h // rep]) / p.sum(axis=1, keepdims=True)
    return o


def _inputs(seed, Lk=300, d=32, dtype="bf16"):
    g = np.random.default_rng(seed)
    q, k, v = (_round16(g.standard_normal(s), dtype) for s in ((1, 11, 2, d), (1, Lk, 1, d), (1, Lk, 1, d)))
    return q, k, v


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("seed,scale,shift", [(1, 32 ** -0.5, 0.0), (2, 32 ** -0.5, 5.5),
                                              (3, 0.6, 0.0), (4, 0.6, 5.5)])
def test_bound_covers_a_simulation(dtype, seed, scale, shift):
    q, k, v = _inputs(seed, dtype=dtype)
    o_exact, _ = attention_fwd(q, k, v, scale)
    err = np.abs(_simulate(q, k, v, scale, dtype, shift) - o_exact)
    bound = p16_rounding_bound(q, k, v, scale, dtype)
    assert np.all(err <= bound * (1 + 1e-9) + 1e-15)
    assert err.max() > 0                         # the rounding is visible
    assert err.max() > 1e-3 * bound.max()        # and the bound is not loose by many orders


@pytest.mark.parametrize("dtype,p", [("bf16", 8), ("fp16", 11)])
def test_worst_case_one_key_needs_the_full_relative_term(dtype, p):
    """One visible key: w = 1 and O = v exactly. A lagging reference that makes
    P = 1 + 2^-p - 2^-(p+12) (just below the midpoint between 1 and the next
    value) rounds P down to 1, so O moves by (P - 1) / P of v, just under
    2^-p |v|: the bound holds, a bound with 2^-(p+1) does not."""
    v = np.array([[[[3.0, -1.5, 0.25, 2.0]]]])       # [1, 1, 1, 4]
    q = np.zeros((1, 1, 1, 4))
    k = np.zeros((1, 1, 1, 4))
    P = 1.0 + 2.0 ** -p - 2.0 ** -(p + 12)
    assert _round16([P], dtype)[0] == 1.0
    o_kernel = _round16([P], dtype)[0] * v[0, 0, 0] / P   # l keeps the float P
    err = np.abs(o_kernel - v[0, 0, 0])
    bound = p16_rounding_bound(q, k, v, 1.0, dtype)[0, 0, 0]
    assert np.all(err <= bound)
    assert np.all(err > 2.0 ** -(p + 1) * np.abs(v[0, 0, 0]))


def test_fp16_subnormal_weights_need_the_absolute_term():
    """Below FP16's smallest normal (2^-14) the spacing is fixed (2^-24), so a
    small P can move by a large fraction of itself. One key at the row max
    (P = 1, exact, with v = 0) and 200 keys at P = 1.4 * 2^-24 (each rounds to
    2^-24, a 29 % change) with v = 1: a relative-only bound fails, the
    absolute floor 2^-25 w_max per key covers it."""
    n = 200
    q = np.ones((1, 1, 1, 1))
    k = np.full((1, n + 1, 1, 1), np.log(1.4 * 2.0 ** -24))
    k[0, 0, 0, 0] = 0.0
    v = np.ones((1, n + 1, 1, 1))
    v[0, 0, 0, 0] = 0.0
    o_exact, _, w = attention_fwd(q, k, v, 1.0, return_weights=True)
    err = np.abs(_simulate(q, k, v, 1.0, "fp16") - o_exact)
    rel_only = 2.0 ** -11 * np.einsum("bhrk,bkhd->brhd", w, np.abs(v))
    assert np.all(err > 10 * rel_only)
    assert np.all(err <= p16_rounding_bound(q, k, v, 1.0, "fp16"))
    # and on random scores spread over ~60 nats the bound still covers the simulation
    q, k, v = _inputs(5, d=32, dtype="fp16")
    err = np.abs(_simulate(q, k, v, 2.5, "fp16") - attention_fwd(q, k, v, 2.5)[0])
    assert np.all(err <= p16_rounding_bound(q, k, v, 2.5, "fp16") * (1 + 1e-9) + 1e-18)


def test_bound_uses_magnitudes_of_v():
    """Errors of keys with opposite-sign V need not cancel: the bound is a sum
    of |v|, so it is unchanged when V's signs flip."""
    q, k, v = _inputs(6)
    b1 = p16_rounding_bound(q, k, v, 0.3, "bf16")
    b2 = p16_rounding_bound(q, k, -v, 0.3, "bf16")
    np.testing.assert_array_equal(b1, b2)
    assert np.all(b1 > 0)


def test_masks_and_rows():
    g = np.random.default_rng(7)
    q, k, v = (g.standard_normal(s) for s in ((2, 20, 4, 16), (2, 30, 2, 16), (2, 30, 2, 16)))
    rows = [0, 7, 19]
    for mask, off in ((0, 0), (1, 10), (2, 5)):
        full = p16_rounding_bound(q, k, v, 0.4, "bf16", mask, off)
        part = p16_rounding_bound(q, k, v, 0.4, "bf16", mask, off, rows=rows)
        np.testing.assert_allclose(part, full[:, rows], rtol=1e-12, atol=0)
    # causal row 0 at offset 0 sees one key: its bound is 2^-8 |v_0|
    b = p16_rounding_bound(q, k, v, 0.4, "bf16", 1, 0)
    np.testing.assert_allclose(b[:, 0, 0], 2.0 ** -8 * np.abs(v[:, 0, 0]), rtol=1e-12)


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_half_ulp_matches_round_to_nearest(dtype):
    g = np.random.default_rng(8)
    x = np.concatenate([g.standard_normal(20000) * s for s in (1e-3, 1.0, 40.0)])
    if dtype == "fp16":
        x = np.concatenate([x, g.standard_normal(2000) * 1e-6])  # FP16 subnormals
    x = x.astype(np.float32).astype(np.float64)  # one rounding, from float32 as in the kernel
    h = half_ulp16(x, dtype)
    assert np.all(np.abs(_round16(x, dtype) - x) <= h)
    # reached at the midpoint 1 + half a spacing (ties to even round it to 1)
    one = half_ulp16([1.0], dtype)[0]
    assert one == (2.0 ** -8 if dtype == "bf16" else 2.0 ** -11)
    assert _round16([1.0 + one], dtype)[0] == 1.0
    assert half_ulp16([1.999], dtype)[0] == one and half_ulp16([2.0], dtype)[0] == 2 * one
    if dtype == "fp16":
        assert half_ulp16([1e-6], dtype)[0] == 2.0 ** -25
