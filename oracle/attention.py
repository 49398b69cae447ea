"""FP64 CPU oracle for the fused scaled-dot-product attention forward.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The
product path (the CUDA library and its Python binding) never imports, links or
calls it, and it shares no code with that path: it is a plain, slow, readable
statement of what the kernel must compute, used to check the kernel.

What it computes
----------------
flashdreams.accelerated developer guide, "Optimized Multi Head Attention" ->
"Multi Head Attention Definition", the per-head scaled dot-product attention
equation: for head h,

    A_h = softmax( Q_h K_h^T / sqrt(d) ) V_h

with the softmax taken over keys, row by row. The "optimizing-attention-flash"
skill page, "Workflow 1", Step 2, states the same thing as standard
(materialised) attention, ``softmax(q @ k^T / sqrt(d_k)) @ v``. The scale is a
parameter here (default 1/sqrt(d) in the pages; the flash-attn call on the same
page, "Workflow 2", Step 2, names it ``softmax_scale``).

Layout: token-major ``[batch, seq, heads, head_dim]`` for Q, K, V and O, as the
developer guide's definition shapes them ([B, L, H, d] for Q, [B, S, H, d] for
K and V) and as the FlashAttention-4 runtime page ("FLASH4.md", the H3 call
layout) and the skill page ("Workflow 2", Step 2) use them.

Readings where the pages are silent:

* Head mapping with fewer K/V heads (skill page, "Workflow 2", Step 3,
  multi-query attention; accelerated user guide, "Shared policy", separate
  query and K/V head counts): query head ``hq`` reads K/V head
  ``hq // (Hq // Hkv)``, i.e. consecutive groups of ``Hq // Hkv`` query heads
  share one K/V head. ``Hq % Hkv == 0`` is required.
* Masks. The visible key set of query row ``i`` is a prefix ``j < limit(i)``:
    - mode 0 (none): every key, ``limit = Lk``;
    - mode 1 (causal, skill page ``causal=True``): ``j <= kv_offset + i``,
      so ``kv_offset = Lk - Lq`` gives bottom-right alignment;
    - mode 2 (streaming chunk against a rolling block K/V cache): the query
      chunk occupies cache positions ``[kv_offset, kv_offset + Lq)`` and its
      K/V are written into the cache before it is queried (developer guide,
      "Multi Head Attention Definition" and "Generic Multi Head Attention
      Interface"; user guide, "Cache lifecycle"), and streaming self-attention
      runs the non-causal SDPA kernel over the visible cache (developer guide,
      "OptimizedMultiHeadAttention", ``sdpa_backend``). So every row of the
      chunk sees all keys up to the chunk's end: ``j < kv_offset + Lq``.
* LSE is the natural log of the sum of exp(scaled score) over visible keys,
  per (batch, query head, row), laid out ``[B, Hq, Lq]``.

Algorithm: the plain definition, two passes per row (max, then exponentials,
sum and weighted V), no online update, no tiling. Invisible keys are skipped
(not added as -inf). A library matmul forms the scores; nothing else is fused
or reordered.
"""

from __future__ import annotations

import numpy as np

MASK_NONE = 0
MASK_CAUSAL = 1
MASK_CHUNK = 2
MASK_WINDOW = 3


def kv_head(hq: int, Hq: int, Hkv: int) -> int:
    """K/V head read by query head ``hq``.

    Skill page "optimizing-attention-flash", "Workflow 2", Step 3 (multi-query
    attention: K/V carry fewer heads than Q); accelerated user guide, "Shared
    policy" (query and K/V head counts are separate). Reading: consecutive
    groups of ``Hq // Hkv`` query heads share one K/V head.
    """
    return hq // (Hq // Hkv)


def visible_limit(mask: int, i: int, Lq: int, Lk: int, kv_offset: int) -> int:
    """Number of visible keys for query row ``i``: keys ``j < limit`` are visible.

    Mode 0: all ``Lk`` keys. Mode 1 (causal, skill page "Workflow 2", Step 2,
    ``causal=True``): ``j <= kv_offset + i``. Mode 2 (streaming chunk, developer
    guide "Generic Multi Head Attention Interface": the chunk's K/V are in the
    cache before it is queried): ``j < kv_offset + Lq``.
    """
    if mask == MASK_NONE:
        return Lk
    if mask == MASK_CAUSAL:
        return min(Lk, kv_offset + i + 1)
    if mask == MASK_CHUNK:
        return min(Lk, kv_offset + Lq)
    raise ValueError(f"unknown mask mode {mask}")


def visible_range(mask: int, i: int, Lq: int, Lk: int, kv_offset: int, window=(-1, -1)):
    """Visible keys of query row ``i`` as a half-open range ``[lo, hi)``.

    Modes 0-2: ``[0, visible_limit(...))``. Mode 3 (sliding window, skill page
    "optimizing-attention-flash", "Sliding window attention": flash-attn's
    ``window_size=(left, right)``, -1 for no limit on that side): with the row's
    position ``p = kv_offset + i`` in key coordinates, keys
    ``p - left <= j <= p + right`` are visible.
    """
    if mask != MASK_WINDOW:
        return 0, visible_limit(mask, i, Lq, Lk, kv_offset)
    left, right = window
    p = kv_offset + i
    lo = 0 if left < 0 else max(0, p - left)
    hi = Lk if right < 0 else min(Lk, p + right + 1)
    return lo, hi


def attention_fwd(q, k, v, scale: float, mask: int = MASK_NONE, kv_offset: int = 0,
                  rows=None, return_weights: bool = False, window=(-1, -1)):
    """Scaled dot-product attention forward in float64.

    developer guide, "Multi Head Attention Definition" (per-head SDPA equation);
    skill page, "Workflow 1", Step 2 (standard attention).

    Args:
      q: ``[B, Lq, Hq, d]`` array (any real dtype; widened to float64).
      k, v: ``[B, Lk, Hkv, d]``.
      scale: multiplier of the dot products (1/sqrt(d) in the pages).
      mask: 0 none, 1 causal, 2 streaming chunk, 3 sliding window (see
        ``visible_limit`` and ``visible_range``).
      kv_offset: cache position of query row 0 (masks 1, 2 and 3).
      window: ``(left, right)`` of mask 3.
      rows: optional 1-D sequence of query rows to compute (all rows if None).
      return_weights: also return the softmax weights ``[B, Hq, R, Lk]`` (zero
        at invisible keys); meant for tiny inputs.

    Returns:
      ``(o, lse)``: ``o`` is ``[B, R, Hq, d]`` float64, ``lse`` is
      ``[B, Hq, R]`` float64 (natural log), R = number of rows computed. With
      ``return_weights`` a third element, the weights, follows.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, Lq, Hq, d = q.shape
    Bk, Lk, Hkv, dk = k.shape
    if v.shape != k.shape or Bk != B or dk != d:
        raise ValueError("shape mismatch between q, k, v")
    if Hq % Hkv != 0:
        raise ValueError("Hq must be a multiple of Hkv")
    rows = np.arange(Lq) if rows is None else np.asarray(rows, dtype=np.int64)
    R = rows.shape[0]

    o = np.zeros((B, R, Hq, d), dtype=np.float64)
    lse = np.zeros((B, Hq, R), dtype=np.float64)
    weights = np.zeros((B, Hq, R, Lk), dtype=np.float64) if return_weights else None

    ranges = [visible_range(mask, int(i), Lq, Lk, kv_offset, window) for i in rows]
    if any(hi <= lo for lo, hi in ranges):
        raise ValueError("every query row must see at least one key")
    for b in range(B):
        for hq in range(Hq):
            hkv = kv_head(hq, Hq, Hkv)
            K = k[b, :, hkv, :]
            V = v[b, :, hkv, :]
            Q = q[b, rows, hq, :]
            scores = scale * (Q @ K.T)  # [R, Lk]
            # rows that share one visible key range are handled together
            for lo, hi in sorted(set(ranges)):
                sel = np.array([n for n, r in enumerate(ranges) if r == (lo, hi)], dtype=np.int64)
                s = scores[sel, lo:hi]                      # visible keys only
                m = s.max(axis=1, keepdims=True)            # pass 1: row max
                e = np.exp(s - m)                           # pass 2: weights
                l = e.sum(axis=1, keepdims=True)
                o[b, sel, hq, :] = (e @ V[lo:hi]) / l
                lse[b, hq, sel] = m[:, 0] + np.log(l[:, 0])
                if return_weights:
                    weights[b, hq, sel, lo:hi] = e / l
    if return_weights:
        return o, lse, weights
    return o, lse


def flops(B: int, Lq: int, Lk: int, Hq: int, d: int, mask: int) -> float:
    """Algorithmic FLOPs of one forward: 4*B*Hq*Lq*Lk*d, halved for causal.

    Two matmuls (Q K^T and P V), each 2*Lq*Lk*d per (batch, head). The count
    is the conventional one for attention throughput; the causal half is the
    standard convention for a lower-triangular mask.
    """
    f = 4.0 * B * Hq * Lq * Lk * d
    return f / 2.0 if mask == MASK_CAUSAL else f


def visible_pairs(Lq: int, Lk: int, mask: int, kv_offset: int = 0, window=(-1, -1)) -> int:
    """Number of visible (query row, key) pairs of one (batch, head)."""
    return sum(hi - lo for lo, hi in (visible_range(mask, i, Lq, Lk, kv_offset, window)
                                      for i in range(Lq)))
