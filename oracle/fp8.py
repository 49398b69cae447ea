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
  unrounded P. The oracle does not model that rounding; ``p_rounding_bound``
  gives the per-element bound it implies: each weight w_j carries a relative
  error of at most 2^-4 (half an e4m3 unit), so
  |O_gpu - O| <= 2^-4 sum_j w_j |v_j| (+ the 16-bit rounding of O).
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


def p_rounding_bound(q, k, v, scale: float, mask: int = 0, kv_offset: int = 0) -> np.ndarray:
    """Per-element bound [B, Lq, Hq, d] on |O| error from rounding P to e4m3:
    2^-4 * sum_j w_j |v_j| with w the exact softmax weights (tiny inputs)."""
    q8, k8, v8 = e4m3(q), e4m3(k), e4m3(v)
    _, _, w = attention_fwd(q8, k8, v8, scale, mask, kv_offset, return_weights=True)
    B, Lq, Hq, d = q8.shape
    Hkv = k8.shape[2]
    rep = Hq // Hkv
    av = np.abs(v8)
    out = np.zeros((B, Lq, Hq, d))
    for b in range(B):
        for h in range(Hq):
            out[b, :, h, :] = w[b, h] @ av[b, :, h // rep, :]
    return 2.0 ** -4 * out
