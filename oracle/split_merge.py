"""FP64 CPU oracle for combining attention over disjoint key ranges.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The
product path never imports, links or calls it.

What it computes
----------------
Attention over a key set K split into disjoint parts K_1 .. K_G: with O_g the
attention output over K_g alone and lse_g = ln sum_{j in K_g} exp(s_j), the
softmax over K is recovered exactly (developer guide, "Multi Head Attention
Definition", the softmax of the scaled scores, regrouped by parts):

    lse = ln sum_g exp(lse_g),      O = sum_g exp(lse_g - lse) O_g.

A part with no key has lse_g = -inf and weight 0. This is the combine step of
splitting the keys of one query tile across several workers (the pages'
sequence-split remark: context parallelism across GPUs).
"""

from __future__ import annotations

import numpy as np


def lse_merge(o_parts, lse_parts):
    """o_parts [G, B, L, H, d], lse_parts [G, B, H, L] -> (o [B, L, H, d], lse [B, H, L])."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = np.max(lse_parts, axis=0)                        # [B, H, L]
    w = np.exp(lse_parts - m[None])                      # [G, B, H, L], 0 for empty parts
    total = np.sum(w, axis=0)
    lse = m + np.log(total)
    wn = (w / total[None]).transpose(0, 1, 3, 2)[..., None]  # [G, B, L, H, 1]
    return np.sum(wn * o_parts, axis=0), lse
