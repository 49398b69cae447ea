"""FP64 CPU oracle for the FP8 attention paths (unscaled and per-token scaled).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The
product path never imports, links or calls it.

What it computes
----------------
flashdreams.accelerated developer guide, "Optimized Multi Head Attention" ->
"OptimizedImplConfig" (``quantization.quantized_sdpa``): Q, K and V are cast
directly, without scales, to ``float8_e4m3fn`` (the K/V cache is kept in that
type) and the attention runs on those values; the probabilities P multiplying
V are FP8 as well. The oracle is the exact attention (``attention_fwd``) of the
e4m3 values of Q, K and V, in float64.

The scaled variant follows the quantizer's per-token rule instead (developer
guide, "Quantization Toolkit" -> "Quantized GEMM", inner-dimension rule; the
pages' SageAttention remark): Q and K are quantized with one scale per token
and head, V with one scale per channel and head (``quantize_attention_inputs``),
and the oracle is the exact attention of the dequantized values.

Readings where the pages are silent:

* The cast rounds to nearest even and saturates at +-448 (the largest finite
  e4m3 value; the type has no infinities).
* P is rounded to e4m3 before the P V product while the row sum l uses the
  unrounded P. The oracle does not model that rounding (where it happens
  depends on the running reference of the online softmax); it gives two
  per-element figures the rounding implies, for any reference at or below the
  row max (so every P <= 1, or <= 2^8 with a lagging reference: no
  saturation). With w the exact softmax weights, w_max their row maximum and
  P_j = w_j / w_max times a power of the reference gap that is <= 1:

  - ``p_rounding_bound``: a normal e4m3 value has 3 mantissa bits, so rounding
    moves it by at most 2^-4 of itself; below the smallest normal (2^-6) the
    spacing is 2^-9 and the error at most 2^-10, i.e. 2^-10 w_max in weight
    units. Hence |O_gpu - O| <= sum_j max(2^-4 w_j, 2^-10 w_max) |v_j|.
  - ``p_rounding_var``: the same errors taken as independent and uniform over
    one spacing (relative spacing at most 2^-3 for normal values, absolute
    2^-9 w_max below them) give the variance bound
    sum_j max(2^-6 w_j^2, 2^-18 w_max^2) v_j^2 / 12 of each output element.
"""

from __future__ import annotations

import numpy as np
import torch

from .attention import attention_fwd

E4M3_MAX = 448.0


def e4m3(x) -> np.ndarray:
    """Round to the nearest float8_e4m3fn value (ties to even), saturating at
    +-448, returned as float64. Uses the library cast as the rounding step."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float64)).to(torch.float32)
    t = torch.clamp(t, -E4M3_MAX, E4M3_MAX)
    return t.to(torch.float8_e4m3fn).to(torch.float64).numpy()


def attention_fp8(q, k, v, scale: float, mask: int = 0, kv_offset: int = 0, rows=None):
    """Exact attention of the e4m3-cast Q, K, V."""
    return attention_fwd(e4m3(q), e4m3(k), e4m3(v), scale, mask, kv_offset, rows=rows)


def _weights_and_v(q, k, v, scale, mask, kv_offset, rows, cast=True):
    """Yield (b, hq, w [R, Lk], v8 [Lk, d]) per (batch, head) of the cast
    inputs (or of the inputs as given, ``cast`` False: dequantized values), w
    the exact softmax weights of the rows (one head at a time, so long
    sequences need only R x Lk weights at once)."""
    if cast:
        q8, k8, v8 = e4m3(q), e4m3(k), e4m3(v)
    else:
        q8, k8, v8 = (np.asarray(t, dtype=np.float64) for t in (q, k, v))
    B, Lq, Hq, d = q8.shape
    Hkv = k8.shape[2]
    rep = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            hk = h // rep
            _, _, w = attention_fwd(q8[b:b + 1, :, h:h + 1], k8[b:b + 1, :, hk:hk + 1],
                                    v8[b:b + 1, :, hk:hk + 1], scale, mask, kv_offset, rows=rows,
                                    return_weights=True)
            yield b, h, w[0, 0], v8[b, :, hk, :]


def p_rounding_bound(q, k, v, scale: float, mask: int = 0, kv_offset: int = 0, rows=None,
                     cast: bool = True) -> np.ndarray:
    """Per-element bound [B, R, Hq, d] on |O| error from rounding P to e4m3:
    sum_j max(2^-4 w_j, 2^-10 w_max) |v_j| over the visible keys j."""
    B, Lq, Hq, d = np.shape(q)
    R = Lq if rows is None else len(rows)
    out = np.zeros((B, R, Hq, d))
    for b, h, w, v8 in _weights_and_v(q, k, v, scale, mask, kv_offset, rows, cast):
        wmax = w.max(axis=1, keepdims=True)
        per_key = np.where(w > 0, np.maximum(2.0 ** -4 * w, 2.0 ** -10 * wmax), 0.0)
        out[b, :, h, :] = per_key @ np.abs(v8)
    return out


def p_rounding_var(q, k, v, scale: float, mask: int = 0, kv_offset: int = 0, rows=None,
                   cast: bool = True) -> np.ndarray:
    """Per-element variance bound [B, R, Hq, d] of the O error from rounding P
    to e4m3, errors independent and uniform over one e4m3 spacing:
    sum_j max(2^-6 w_j^2, 2^-18 w_max^2) v_j^2 / 12 over the visible keys j."""
    B, Lq, Hq, d = np.shape(q)
    R = Lq if rows is None else len(rows)
    out = np.zeros((B, R, Hq, d))
    for b, h, w, v8 in _weights_and_v(q, k, v, scale, mask, kv_offset, rows, cast):
        wmax = w.max(axis=1, keepdims=True)
        per_key = np.where(w > 0, np.maximum(2.0 ** -6 * w * w, 2.0 ** -18 * wmax * wmax), 0.0)
        out[b, :, h, :] = per_key @ (v8 * v8) / 12.0
    return out


def quantize_attention_inputs(q, k, v, v_scaled: bool = True):
    """Per-token scaled e4m3 inputs of the scaled FP8 attention.

    developer guide, "Quantization Toolkit" -> "Quantized GEMM" (inner-dimension
    rule): the scales of each GEMM operand must be constant along the GEMM's
    reduction axis. Q K^T reduces over the head dim, so Q and K take one scale
    per (batch, token, head) (slice granularity, axis=-1: per-token
    quantization); P V reduces over the keys, so V takes one scale per (batch,
    head, channel) (slice granularity over the token axis). With ``v_scaled``
    False, V is cast directly (scale 1), as in the unscaled variant.

    Returns (q_codes, sq, k_codes, sk, v_codes, sv): codes as float64 e4m3
    values, scales float32 with the reduced axes of size one.
    """
    from .quantize import SLICE, quantize
    qc, sq = quantize(q, "e4m3", SLICE, axis=-1)
    kc, sk = quantize(k, "e4m3", SLICE, axis=-1)
    if v_scaled:
        vc, sv = quantize(v, "e4m3", SLICE, axis=1)
    else:
        vc = e4m3(v)
        sv = np.ones((np.shape(v)[0], 1, np.shape(v)[2], np.shape(v)[3]), dtype=np.float32)
    return qc, sq, kc, sk, vc, sv


def dequantized_attention_inputs(q, k, v, v_scaled: bool = True):
    """The exact (float64) dequantized Q, K, V of ``quantize_attention_inputs``:
    Q K^T of these is (s_Q s_K^T) times the code product, exactly."""
    from .quantize import dequantize
    qc, sq, kc, sk, vc, sv = quantize_attention_inputs(q, k, v, v_scaled)
    return (dequantize(qc, sq, precision=np.float64), dequantize(kc, sk, precision=np.float64),
            dequantize(vc, sv, precision=np.float64))


def attention_fp8_scaled(q, k, v, scale: float, mask: int = 0, kv_offset: int = 0, rows=None,
                         v_scaled: bool = True):
    """Exact attention of the dequantized per-token-scaled e4m3 Q, K (and the
    per-channel-scaled V)."""
    qd, kd, vd = dequantized_attention_inputs(q, k, v, v_scaled)
    return attention_fwd(qd, kd, vd, scale, mask, kv_offset, rows=rows)
