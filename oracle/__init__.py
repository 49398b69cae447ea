"""FP64 CPU oracle for the attention forward (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package; the product path never does.
"""

from .attention import (MASK_CAUSAL, MASK_CHUNK, MASK_NONE, attention_fwd, flops,
                        kv_head, visible_limit)

__all__ = ["MASK_NONE", "MASK_CAUSAL", "MASK_CHUNK", "attention_fwd", "flops",
           "kv_head", "visible_limit"]
