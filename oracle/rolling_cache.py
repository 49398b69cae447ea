"""FP64 CPU oracle for streaming self-attention over a rolling block K/V cache.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module. The
product path never imports, links or calls it.

What it computes
----------------
flashdreams.accelerated developer guide, "Generic Multi Head Attention
Interface" (the streaming example) and user guide, "Accelerated building
blocks" -> "Cache lifecycle": a BlockKVCache with fixed chunk, window and sink
sizes, K/V storage ``[B, sink_size + window_size, H, d]``; per query chunk the
caller runs ``before_update(chunk_idx)``, the attention call, then
``after_update(chunk_idx)``; the current chunk's K/V are written into the
rolling cache before the chunk is queried; cached keys are evicted as the
stream advances ("test both cache fill and post-eviction steady state").

Readings where the pages are silent:

* Sizes are whole chunks: ``sink_size`` and ``window_size`` are multiples of
  the chunk length ``C``.
* Sinks are the first ``sink_size`` tokens of the stream and are never
  evicted. The window holds the most recent ``window_size`` tokens, the current
  chunk included; when a new chunk arrives and the window is full, the oldest
  window chunk is evicted. So chunk ``c`` (tokens ``c C .. c C + C - 1``) sees
  the sink tokens plus the ``window_size`` tokens ending with its own.
* Every query of the chunk sees every visible key (the chunk's own K/V are in
  the cache before it is queried, and the self-attention SDPA is non-causal),
  so the result does not depend on where the keys sit in storage.
* After-cache RoPE (``stream_attention_after_rope``): positions are
  cache-relative, the index of a key in the visible set in stream order.
"""

from __future__ import annotations

import numpy as np

from .attention import MASK_NONE, attention_fwd


def visible_tokens(chunk_idx: int, chunk: int, sink: int, window: int) -> np.ndarray:
    """Absolute token indices whose K/V chunk ``chunk_idx`` attends to."""
    if chunk < 1 or sink < 0 or window < chunk or sink % chunk or window % chunk:
        raise ValueError("sizes must be whole chunks, window >= one chunk")
    end = (chunk_idx + 1) * chunk                 # one past the chunk's last token
    win_start = max(0, end - window)
    sinks = np.arange(min(sink, win_start))       # sink tokens not already in the window
    return np.concatenate([sinks, np.arange(win_start, end)]).astype(np.int64)


def stream_attention(q_chunks, k_all, v_all, chunk: int, sink: int, window: int, scale: float):
    """Per-chunk outputs of streaming self-attention.

    q_chunks: list of [B, C, Hq, d] arrays (chunk c holds the queries of tokens
    c C .. c C + C - 1); k_all, v_all: [B, T, Hkv, d] K/V of every token of the
    stream (as written into the cache, i.e. after any before-cache RoPE).
    Returns a list of (o [B, C, Hq, d], lse [B, Hq, C]).
    """
    out = []
    for c, q in enumerate(q_chunks):
        idx = visible_tokens(c, chunk, sink, window)
        k = np.asarray(k_all)[:, idx]
        v = np.asarray(v_all)[:, idx]
        out.append(attention_fwd(q, k, v, scale, MASK_NONE, 0))
    return out


def stream_attention_after_rope(q_chunks, k_all, v_all, chunk: int, sink: int, window: int,
                                scale: float, angles, style: int, round_rotated=None):
    """Per-chunk outputs with RoPE applied after the cache update.

    developer guide, "Multi Head Attention Definition" (RoPE after the K/V
    cache update: the cache keeps unrotated keys; right before attention the
    current queries and every visible cached key are rotated with the angles of
    their current positions) and "Generic Multi Head Attention Interface" (for
    after-cache RoPE the angle table covers the query and every visible cache
    position; cached keys take cache-relative frequencies).

    Reading where the pages are silent: a visible key's current position is its
    index in the visible set in stream order (sinks first, then the window
    oldest first, the current chunk last); the chunk's queries take the
    positions of the chunk's own keys, the last ``chunk`` of them.

    q_chunks: list of [B, C, Hq, d] (already normalised, unrotated); k_all,
    v_all: [B, T, Hkv, d] as written into the cache (normalised, unrotated);
    angles: [R, d] expanded per-feature angle table of positions 0 .. R - 1.
    ``round_rotated``, if given, is applied to the rotated queries and keys
    (a path that stores them in a 16-bit type rounds there; the default keeps
    them exact). Returns a list of (o, lse) as ``stream_attention``.
    """
    out = []
    for qr, k, v in after_rope_inputs(q_chunks, k_all, v_all, chunk, sink, window, angles, style,
                                      round_rotated):
        out.append(attention_fwd(qr, k, v, scale, MASK_NONE, 0))
    return out


def after_rope_inputs(q_chunks, k_all, v_all, chunk: int, sink: int, window: int, angles, style: int,
                      round_rotated=None):
    """Per chunk, the (queries, keys, values) that ``stream_attention_after_rope``
    attends with: the chunk's queries and every visible key rotated at their
    current (cache-relative) positions, optionally rounded, and the visible
    values. Same readings and arguments as that function."""
    from .prologue import rope
    out = []
    ang = np.asarray(angles, dtype=np.float64)
    for c, q in enumerate(q_chunks):
        idx = visible_tokens(c, chunk, sink, window)
        R = len(idx)
        k = rope(np.asarray(k_all)[:, idx], ang[:R], style)
        qr = rope(np.asarray(q), ang[R - chunk:R], style)
        if round_rotated is not None:
            k, qr = round_rotated(k), round_rotated(qr)
        out.append((qr, k, np.asarray(v_all)[:, idx]))
    return out
