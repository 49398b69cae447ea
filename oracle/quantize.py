"""CPU oracle of the quantizer: scales, quantize, dequantize.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The
product path never imports, links or calls it.

What it computes
----------------
flashdreams.accelerated developer guide, "Quantization Toolkit" ->
"Scale Granularity", "dequantize" and "Quantized GEMM". For a target type t
with largest finite value M_t (127 for int8, 448 for float8_e4m3fn) and a
scale floor eps:

* tensor granularity: one scale s = max(max |X| / M_t, eps);
* slice granularity along ``axis``: the max runs over that axis only, giving
  one scale per remaining index (axis=0 of a matrix: one per column; axis=1:
  one per row). The scale keeps every input dimension, the reduced one with
  size one.
* quantize: divide by the scale, clip to [-M_t, M_t], convert to t (int8:
  round to the nearest integer; e4m3: round to the nearest e4m3 value).
* dequantize: the codes times every given scale, with broadcasting.

The pages compute the scales in float32; so does this oracle, including the
division by the scale, because those roundings decide the integer or FP8 code.

Readings where the pages are silent:

* eps is not given; it only matters for a slice whose max |X| / M_t falls
  below it (an all-zero row, say). It is taken as 2^-126, the smallest normal
  float32, which keeps every division finite.
* int8 ties round to even (the pages' examples have no ties except 63.5, which
  gives 64 either way).
"""

from __future__ import annotations

import numpy as np

from .fp8 import e4m3

EPS = np.float32(2.0 ** -126)
M_T = {"int8": 127.0, "e4m3": 448.0}
TENSOR = "tensor"
SLICE = "slice"


def scale_of(x, dtype: str, granularity: str = TENSOR, axis: int | None = None) -> np.ndarray:
    """float32 scale(s) of x: max(max |x| / M_t, eps) over the whole tensor or
    over ``axis``, dimensions kept (the reduced ones with size one)."""
    x32 = np.asarray(x, dtype=np.float32)
    if granularity == TENSOR:
        amax = np.max(np.abs(x32), axis=None, keepdims=True)
    elif granularity == SLICE:
        amax = np.max(np.abs(x32), axis=axis, keepdims=True)
    else:
        raise ValueError(granularity)
    s = (amax / np.float32(M_T[dtype])).astype(np.float32)
    return np.maximum(s, EPS).astype(np.float32)


def quantize(x, dtype: str, granularity: str = TENSOR, axis: int | None = None):
    """(codes, scale): codes = convert(clip(x / s, -M_t, M_t)) as float64
    values (exact integers for int8, exact e4m3 values for e4m3), s float32."""
    s = scale_of(x, dtype, granularity, axis)
    y = (np.asarray(x, dtype=np.float32) / s).astype(np.float32)
    m = np.float32(M_T[dtype])
    y = np.clip(y, -m, m)
    if dtype == "int8":
        codes = np.rint(y).astype(np.float64)
    elif dtype == "e4m3":
        codes = e4m3(y)
    else:
        raise ValueError(dtype)
    return codes, s


def dequantize(codes, *scales, precision=np.float32) -> np.ndarray:
    """codes times every scale in turn, with broadcasting, in ``precision``
    (float32 as in the pages; float64 gives the exact value of the product of
    an e4m3 code and a float32 scale)."""
    out = np.asarray(codes).astype(precision)
    for s in scales:
        out = (out * np.asarray(s).astype(precision)).astype(precision)
    return out
