"""FP64 CPU oracle for the attention forward and its Q/K prologue (test
infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
and reference legs may import this package; the product path never does.
"""

from .attention import (MASK_CAUSAL, MASK_CHUNK, MASK_NONE, MASK_WINDOW, attention_fwd, flops,
                        kv_head, visible_limit, visible_pairs, visible_range)
from .rolling_cache import stream_attention, stream_attention_after_rope, visible_tokens
from .prologue import (NORM_HEAD, NORM_INNER, NORM_NONE, ROPE_INTERLEAVED, ROPE_NONE,
                          ROPE_SPLIT, qk_prologue, rms_norm, rope)

__all__ = ["MASK_NONE", "MASK_CAUSAL", "MASK_CHUNK", "MASK_WINDOW", "attention_fwd", "flops",
           "kv_head", "visible_limit", "visible_range", "visible_pairs", "NORM_NONE", "NORM_HEAD", "NORM_INNER", "ROPE_NONE",
           "ROPE_INTERLEAVED", "ROPE_SPLIT", "qk_prologue", "rms_norm", "rope", "stream_attention",
           "stream_attention_after_rope", "visible_tokens"]
