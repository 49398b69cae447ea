"""Pins for the quantizer oracle and the per-token scaled FP8 attention oracle.

* The pages' printed worked examples (``tests/golden/quantize_worked_examples.json``):
  the INT8 vector, a 3x2 matrix per tensor and per slice along both axes, the
  dequantized vector, and the slice-quantized GEMM's codes, integer product
  and dequantized result.
* The inner-dimension rule: with row scales on A and column scales on B, the
  dequantized code product equals the product of the dequantized operands.
* The scaled FP8 attention: on inputs that are e4m3 values times a power of
  two per token (channel, for V) with the slice max at 448, quantization is
  lossless, so the oracle must return the exact attention of the inputs; the
  same inputs quantized along the wrong axis are not lossless (a planted
  mistake is caught).

Source: developer guide, "Quantization Toolkit" (Scale Granularity,
dequantize, Quantized GEMM, Worked Slice-Quantized GEMM).
"""

from __future__ import annotations

import json
import os

import numpy as np
import pytest

from oracle import MASK_CAUSAL, MASK_NONE, attention_fwd
from oracle import fp8
from oracle import quantize as qz

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                     "quantize_worked_examples.json")))


def test_vector_example():
    g = GOLDEN["vector"]
    codes, s = qz.quantize(np.array(g["x"]), "int8")
    assert codes.tolist() == g["codes"]
    assert s.shape == (1,) and abs(float(s[0]) - g["scale"]) < 5e-7
    np.testing.assert_allclose(qz.dequantize(codes, s), g["dequantized"], atol=5e-5)


@pytest.mark.parametrize("mode", ["tensor", "axis0", "axis1"])
def test_matrix_examples(mode):
    g = GOLDEN["matrix"]
    X = np.array(g["X"])
    if mode == "tensor":
        codes, s = qz.quantize(X, "int8", qz.TENSOR)
        assert s.shape == (1, 1)
    else:
        axis = 0 if mode == "axis0" else 1
        codes, s = qz.quantize(X, "int8", qz.SLICE, axis=axis)
        assert s.shape == ((1, 2) if axis == 0 else (3, 1))  # the reduced dimension kept with size one
    assert codes.tolist() == g[mode]["codes"]
    np.testing.assert_allclose(s.ravel(), np.ravel(g[mode]["scale"]), atol=5e-7)


def test_worked_slice_quantized_gemm():
    g = GOLDEN["gemm"]
    a, b = np.array(g["a"]), np.array(g["b"])
    qa, sa = qz.quantize(a, "int8", qz.SLICE, axis=1)
    qb, sb = qz.quantize(b, "int8", qz.SLICE, axis=0)
    assert qa.tolist() == g["qa"] and qb.tolist() == g["qb"]
    assert sa.shape == (3, 1) and sb.shape == (1, 3)
    qc = qa.astype(np.int64) @ qb.astype(np.int64)
    assert qc.tolist() == g["qc"]
    c = qz.dequantize(qc, sa, sb)
    np.testing.assert_allclose(c, g["c"], atol=5e-4)
    np.testing.assert_allclose(c, a @ b, atol=0.2)  # the page's own closeness bar


def test_inner_dimension_rule_is_exact_for_slice_scales():
    g = np.random.default_rng(1)
    A, B = g.standard_normal((7, 32)) * 3, g.standard_normal((32, 5)) * 0.1
    ca, sa = qz.quantize(A, "e4m3", qz.SLICE, axis=1)
    cb, sb = qz.quantize(B, "e4m3", qz.SLICE, axis=0)
    lhs = qz.dequantize(ca @ cb, sa, sb, precision=np.float64)
    rhs = qz.dequantize(ca, sa, precision=np.float64) @ qz.dequantize(cb, sb, precision=np.float64)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-14, atol=0)


def test_e4m3_slice_max_maps_to_448_and_zero_rows_take_the_floor():
    g = np.random.default_rng(2)
    x = g.standard_normal((6, 16)) * np.array([1e-3, 1, 10, 100, 1e4, 0])[:, None]
    codes, s = qz.quantize(x, "e4m3", qz.SLICE, axis=1)
    np.testing.assert_array_equal(np.abs(codes[:5]).max(axis=1), 448.0)
    assert s[5, 0] == qz.EPS and not codes[5].any()
    assert s.dtype == np.float32


def _exact_inputs(g, shape, axis):
    """e4m3 values whose slice max along ``axis`` is +-448, times 2^e per slice."""
    codes = fp8.e4m3(g.standard_normal(shape) * 60)
    flat = np.moveaxis(codes, axis, -1)
    flat[..., 0] = 448.0 * np.sign(flat[..., 0] + 0.5)   # one element of every slice at |448|
    codes = np.moveaxis(flat, -1, axis)
    e_shape = [1 if a == (axis % len(shape)) else shape[a] for a in range(len(shape))]
    e = g.integers(-12, 4, size=e_shape).astype(np.float64)
    return codes * 2.0 ** e


@pytest.mark.parametrize("mask,off", [(MASK_NONE, 0), (MASK_CAUSAL, 5)])
def test_scaled_fp8_attention_is_lossless_on_exact_inputs(mask, off):
    g = np.random.default_rng(3)
    q = _exact_inputs(g, (2, 9, 4, 16), -1)     # per (batch, token, head)
    k = _exact_inputs(g, (2, 14, 2, 16), -1)
    v = _exact_inputs(g, (2, 14, 2, 16), 1)     # per (batch, head, channel)
    scale = 0.02
    o, lse = fp8.attention_fp8_scaled(q, k, v, scale, mask, off)
    o_ref, lse_ref = attention_fwd(q, k, v, scale, mask, off)
    np.testing.assert_allclose(o, o_ref, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-13, atol=1e-13)
    # the scales the oracle took are the powers of two, one per token and head
    _, sq, _, sk, _, sv = fp8.quantize_attention_inputs(q, k, v)
    assert sq.shape == (2, 9, 4, 1) and sk.shape == (2, 14, 2, 1) and sv.shape == (2, 1, 2, 16)
    assert np.all(np.log2(sq) == np.round(np.log2(sq)))


def test_wrong_quantization_axis_is_caught():
    g = np.random.default_rng(4)
    q = _exact_inputs(g, (1, 9, 2, 16), -1)
    k = _exact_inputs(g, (1, 14, 2, 16), -1)
    v = _exact_inputs(g, (1, 14, 2, 16), 1)
    exact = attention_fwd(q, k, v, 0.05, MASK_NONE, 0)[0]
    # planted: Q quantized per channel (over tokens) instead of per token
    qc, sq = qz.quantize(q, "e4m3", qz.SLICE, axis=1)
    wrong = attention_fwd(qz.dequantize(qc, sq, precision=np.float64),
                          *fp8.dequantized_attention_inputs(q, k, v)[1:], 0.05, MASK_NONE, 0)[0]
    assert np.abs(wrong - exact).max() > 1e-6


def test_scaled_beats_unscaled_on_small_magnitudes():
    """Values far below 1 lose most bits in a direct e4m3 cast (subnormals) but
    not after per-token scaling: the reason for the scales."""
    g = np.random.default_rng(5)
    q = g.standard_normal((1, 16, 2, 32)) * 1e-3
    k = g.standard_normal((1, 40, 2, 32)) * 1e-3
    v = g.standard_normal((1, 40, 2, 32)) * 1e-3
    exact = attention_fwd(q, k, v, 2000.0, MASK_NONE, 0)[0]
    e_scaled = np.abs(fp8.attention_fp8_scaled(q, k, v, 2000.0)[0] - exact).max()
    e_unscaled = np.abs(fp8.attention_fp8(q, k, v, 2000.0)[0] - exact).max()
    assert e_scaled < 0.1 * e_unscaled
