"""FP64 CPU oracle for the unscaled FP8 attention path.

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

Readings (listed in the design doc):

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


def _weights_and_v(q, k, v, scale, mask, kv_offset, rows):
    """Yield (b, hq, w [R, Lk], v8 [Lk, d]) per (batch, head) of the cast
    inputs, w the exact softmax weights of the rows (one head at a time, so
    long sequences need only R x Lk weights at once)."""
    q8, k8, v8 = e4m3(q), e4m3(k), e4m3(v)
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


def p_rounding_bound(q, k, v, scale: float, mask: int = 0, kv_offset: int = 0, rows=None) -> np.ndarray:
    """Per-element bound [B, R, Hq, d] on |O| error from rounding P to e4m3:
    sum_j max(2^-4 w_j, 2^-10 w_max) |v_j| over the visible keys j."""
    B, Lq, Hq, d = np.shape(q)
    R = Lq if rows is None else len(rows)
    out = np.zeros((B, R, Hq, d))
    for b, h, w, v8 in _weights_and_v(q, k, v, scale, mask, kv_offset, rows):
        wmax = w.max(axis=1, keepdims=True)
        per_key = np.where(w > 0, np.maximum(2.0 ** -4 * w, 2.0 ** -10 * wmax), 0.0)
        out[b, :, h, :] = per_key @ np.abs(v8)
    return out


def p_rounding_var(q, k, v, scale: float, mask: int = 0, kv_offset: int = 0, rows=None) -> np.ndarray:
    """Per-element variance bound [B, R, Hq, d] of the O error from rounding P
    to e4m3, errors independent and uniform over one e4m3 spacing:
    sum_j max(2^-6 w_j^2, 2^-18 w_max^2) v_j^2 / 12 over the visible keys j."""
    B, Lq, Hq, d = np.shape(q)
    R = Lq if rows is None else len(rows)
    out = np.zeros((B, R, Hq, d))
    for b, h, w, v8 in _weights_and_v(q, k, v, scale, mask, kv_offset, rows):
        wmax = w.max(axis=1, keepdims=True)
        per_key = np.where(w > 0, np.maximum(2.0 ** -6 * w * w, 2.0 ** -18 * wmax * wmax), 0.0)
        out[b, :, h, :] = per_key @ (v8 * v8) / 12.0
    return out
