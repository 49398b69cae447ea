"""Error bounds for the 16-bit rounding steps of the BF16 / FP16 attention path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The
product path never imports, links or calls it.

What it bounds
--------------
The attention being computed is the developer guide's per-head SDPA ("Multi
Head Attention Definition", the equation for A_h): O = sum_j w_j v_j with the
exact softmax weights w_j. The oracle (``attention_fwd``) computes that in
float64. A tiled kernel of the IO-aware kind the skill page describes
("optimizing-attention-flash", "Quick start": the scores stay on chip, a
running max and sum per row) multiplies the probabilities by V on 16-bit
tensor cores, so it rounds each unnormalised probability P_j = exp(s_j - ref)
to the input's 16-bit type before that product, while the row sum l keeps the
float32 P_j. That rounding is not part of the definition; this module states
how far it can move O, so a test can tell it apart from a real error.

Reading (the pages are silent on the kernel's arithmetic): ``ref`` is a
running maximum of the row's scaled scores that lags the final row max by at
most a bounded amount, so every P_j <= 2^tau (tau = 8 in log2 units here) and
the largest P of the row is >= 1. The argument does not depend on tau.

Derivation. Round-to-nearest into a binary format with p significant bits
(BF16: p = 8, FP16: p = 11) moves a normal value x by at most 2^-p |x|
(half of one spacing, 2^(e - p + 1) for x in [2^e, 2^(e+1))). Below the
smallest normal value the spacing is fixed, so the error there is at most a
constant ``a`` (FP16: half the subnormal spacing 2^-24, i.e. 2^-25; BF16: the
float32 exponential flushes results below 2^-126 to zero, a = 2^-126). With
rounded P^_j, |P^_j - P_j| <= max(2^-p P_j, a), and

    O^ - O = sum_j (P^_j - P_j) v_j / l,    l = sum_j P_j >= max_j P_j >= 1.

Since w_j = P_j / l and w_max = max_j P_j / l >= 1 / l,

    |O^ - O| <= sum_j max(2^-p w_j, a w_max) |v_j|           (``p16_rounding_bound``)

per output element. Rescaling O and l by a common factor (a lazy rescale)
scales both sides alike, so the bound holds for a reference that moved during
the row. The final 16-bit rounding of O adds at most half a spacing of O's
format at |O| (``half_ulp16``).
"""

from __future__ import annotations

import numpy as np

from .attention import attention_fwd

# significant bits (p) and the absolute floor ``a`` of the P rounding error
FORMATS = {
    "bf16": (8, 2.0 ** -126),
    "fp16": (11, 2.0 ** -25),
}


def p16_rounding_bound(q, k, v, scale: float, dtype: str, mask: int = 0, kv_offset: int = 0,
                       rows=None, window=(-1, -1)) -> np.ndarray:
    """Per-element bound ``[B, R, Hq, d]`` on |O error| from rounding the
    probabilities to ``dtype`` ("bf16" or "fp16") before P V:
    sum_j max(2^-p w_j, a w_max) |v_j| over the visible keys j."""
    p, a = FORMATS[dtype]
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Lq, Hq, d = q.shape
    Hkv = k.shape[2]
    rep = Hq // Hkv
    R = Lq if rows is None else len(rows)
    out = np.zeros((B, R, Hq, d))
    for b in range(B):
        for h in range(Hq):
            hk = h // rep
            _, _, w = attention_fwd(q[b:b + 1, :, h:h + 1], k[b:b + 1, :, hk:hk + 1],
                                    v[b:b + 1, :, hk:hk + 1], scale, mask, kv_offset, rows=rows,
                                    return_weights=True, window=window)
            w = w[0, 0]                                     # [R, Lk], zero at invisible keys
            wmax = w.max(axis=1, keepdims=True)
            per_key = np.where(w > 0, np.maximum(2.0 ** -p * w, a * wmax), 0.0)
            out[b, :, h, :] = per_key @ np.abs(v[b, :, hk, :])
    return out


def half_ulp16(x, dtype: str) -> np.ndarray:
    """Half the spacing of the 16-bit format at |x|: the largest change that
    rounding a value of magnitude |x| to nearest can make (BF16: 8 significant
    bits, smallest normal 2^-126; FP16: 11, 2^-14, subnormal spacing below)."""
    p, _ = FORMATS[dtype]
    emin = -126 if dtype == "bf16" else -14
    e = np.floor(np.log2(np.maximum(np.abs(np.asarray(x, dtype=np.float64)), 2.0 ** emin)))
    return 2.0 ** (e - p)
