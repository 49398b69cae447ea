"""FP64 CPU oracle for the Q/K prologue: RMS normalisation, then rotary
position embedding.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The
product path never imports, links or calls it, and it shares no code with
that path: it is a plain statement of what the prologue kernel must compute.

What it computes
----------------
flashdreams.accelerated developer guide, "Optimized Multi Head Attention" ->
"Multi Head Attention Definition":

* Q/K RMS normalisation of a feature vector ``z`` of length ``m``:
  ``RMSNorm_gamma(z) = gamma * z / sqrt(mean(z**2) + eps)``. Head scope
  normalises every head on its own (``m = d``); inner scope normalises all
  heads of a token together (``m = H d``). V is never normalised.
* RoPE: pair ``r`` of a token at position ``p`` is rotated by the angle
  ``theta[p, r]``: ``(z_a, z_b) -> (z_a cos - z_b sin, z_a sin + z_b cos)``.
  Interleaved pairs are ``(2r, 2r + 1)``; split-half pairs are
  ``(r, r + d/2)``. The page applies normalisation first, then RoPE ("the
  reference below normalizes before applying RoPE").

Readings where the pages are silent:

* The angles arrive "expanded" as ``rope_freqs`` shaped ``[L, 1, 1, d]``, one
  angle per feature; pair ``r`` uses the angle stored at its first feature
  ``a_r`` (2r interleaved, r split-half). Tables built from the page's
  construction hold the same angle at ``a_r`` and ``b_r``.
* ``gamma`` is a float32 weight of length ``m`` (``d`` for head scope,
  ``H d`` for inner scope); ``None`` means all ones.
* The kernel computes in float32 from the 16-bit inputs and rounds once, after
  RoPE, to the input's 16-bit type; the oracle returns the exact float64 value.
"""

from __future__ import annotations

import numpy as np

NORM_NONE, NORM_HEAD, NORM_INNER = 0, 1, 2
ROPE_NONE, ROPE_INTERLEAVED, ROPE_SPLIT = 0, 1, 2


def rms_norm(x: np.ndarray, gamma, eps: float, scope: int) -> np.ndarray:
    """RMSNorm of ``x`` [B, L, H, d] over the head (scope 1) or the whole
    projected inner dimension H*d (scope 2); scope 0 returns ``x`` unchanged.

    Developer guide, "Multi Head Attention Definition", the RMSNorm equation.
    """
    x = np.asarray(x, dtype=np.float64)
    if scope == NORM_NONE:
        return x.copy()
    B, L, H, d = x.shape
    if scope == NORM_HEAD:
        m = d
        z = x
    elif scope == NORM_INNER:
        m = H * d
        z = x.reshape(B, L, 1, H * d)
    else:
        raise ValueError("scope must be 0, 1 or 2")
    g = np.ones(m) if gamma is None else np.asarray(gamma, dtype=np.float64).reshape(m)
    if g.shape[0] != m:
        raise ValueError("gamma length must be the normalised width")
    mean_sq = np.mean(z * z, axis=-1, keepdims=True)
    y = g * (z / np.sqrt(mean_sq + eps))
    return y.reshape(B, L, H, d)


def pairs(d: int, style: int):
    """Feature index pairs (a_r, b_r), r = 0 .. d/2 - 1, of a RoPE style."""
    if d % 2:
        raise ValueError("RoPE needs an even head dimension")
    r = np.arange(d // 2)
    if style == ROPE_INTERLEAVED:
        return 2 * r, 2 * r + 1
    if style == ROPE_SPLIT:
        return r, r + d // 2
    raise ValueError("style must be 1 (interleaved) or 2 (split-half)")


def rope(x: np.ndarray, angles, style: int) -> np.ndarray:
    """Rotate pair r of token p of ``x`` [B, L, H, d] by ``angles[p, a_r]``
    (``angles`` [L, d], the expanded per-feature table); style 0 returns ``x``.

    Developer guide, "Multi Head Attention Definition", the RoPE rotation and
    the interleaved / split-half pairings.
    """
    x = np.asarray(x, dtype=np.float64)
    if style == ROPE_NONE:
        return x.copy()
    B, L, H, d = x.shape
    ang = np.asarray(angles, dtype=np.float64).reshape(L, d)
    a, b = pairs(d, style)
    theta = ang[:, a][None, :, None, :]  # [1, L, 1, d/2]
    c, s = np.cos(theta), np.sin(theta)
    y = x.copy()
    y[..., a] = x[..., a] * c - x[..., b] * s
    y[..., b] = x[..., a] * s + x[..., b] * c
    return y


def qk_prologue(x, gamma, eps: float, scope: int, angles, style: int) -> np.ndarray:
    """RMSNorm (scope) then RoPE (style) of one of Q or K, [B, L, H, d]."""
    return rope(rms_norm(x, gamma, eps, scope), angles, style)
