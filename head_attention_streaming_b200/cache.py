"""Rolling block K/V cache for streaming self-attention on B200.

The flashdreams.accelerated developer guide ("Generic Multi Head Attention
Interface", the streaming example) and user guide ("Cache lifecycle") describe
a BlockKVCache with fixed chunk, window and sink sizes and K/V storage
``[B, sink_size + window_size, H, d]``; per query chunk the caller runs
``before_update(chunk_idx)``, the attention call, ``after_update(chunk_idx)``;
the chunk's K/V are written into the cache before the chunk is queried.

Layout. The first ``sink_size`` slots hold the first chunks of the stream and
are never evicted. The remaining ``window_size`` slots are a ring of chunk
slots: chunk ``c`` past the sinks goes to ring position
``(c - sink_chunks) % window_chunks``, overwriting (evicting) the chunk
``window_chunks`` earlier. The valid slots are always a prefix of the storage
(sinks first, then the ring as it fills), and since every query of a chunk sees
every cached key, the order of keys in storage does not change the result: the
attention runs over the valid prefix directly, with no data movement.

This module holds only bookkeeping; K/V bytes move in the CUDA kernels
(``attn_stream_update`` writes the chunk, ``attn_fwd_cache`` attends).
"""

from __future__ import annotations

import torch

from . import binding


class BlockKVCache:
    """K/V storage and slot bookkeeping of one streaming self-attention layer.

    Sizes are token counts and must be whole chunks; ``window_size`` holds at
    least one chunk (the current one).
    """

    def __init__(self, batch: int, heads: int, head_dim: int, chunk_size: int, window_size: int,
                 sink_size: int = 0, dtype=torch.bfloat16, device=None):
        if chunk_size < 1 or window_size < chunk_size or sink_size < 0:
            raise ValueError("need chunk_size >= 1, window_size >= chunk_size, sink_size >= 0")
        if window_size % chunk_size or sink_size % chunk_size:
            raise ValueError("window_size and sink_size must be whole chunks")
        if dtype not in binding.DTYPE_CODES:
            raise ValueError("dtype must be bf16 or fp16")
        self.batch, self.heads, self.head_dim = batch, heads, head_dim
        self.chunk_size, self.window_size, self.sink_size = chunk_size, window_size, sink_size
        self.capacity = sink_size + window_size
        device = torch.device("cuda") if device is None else torch.device(device)
        self.k = torch.empty(batch, self.capacity, heads, head_dim, dtype=dtype, device=device)
        self.v = torch.empty_like(self.k)
        self.reset()

    # -------------------------------------------------------------- bookkeeping

    def reset(self) -> None:
        """Forget every cached chunk (the storage is reused as is)."""
        self._next = 0          # chunk index the next before_update must name
        self._pending = None    # (chunk_idx, slot) between before_update and after_update
        self._written = False

    @property
    def sink_chunks(self) -> int:
        return self.sink_size // self.chunk_size

    @property
    def window_chunks(self) -> int:
        return self.window_size // self.chunk_size

    def slot_of(self, chunk_idx: int) -> int:
        """First storage slot of chunk ``chunk_idx``."""
        if chunk_idx < self.sink_chunks:
            return chunk_idx * self.chunk_size
        ring = (chunk_idx - self.sink_chunks) % self.window_chunks
        return self.sink_size + ring * self.chunk_size

    def valid_length(self, chunk_idx: int) -> int:
        """Valid slots (a prefix of the storage) once chunk ``chunk_idx`` is written."""
        tokens = (chunk_idx + 1) * self.chunk_size
        if tokens <= self.sink_size:
            return tokens
        return self.sink_size + min(self.window_size, tokens - self.sink_size)

    def before_update(self, chunk_idx: int) -> int:
        """Reserve the slots of chunk ``chunk_idx`` (evicting the oldest window
        chunk once the ring is full); returns its first slot."""
        if self._pending is not None:
            raise RuntimeError("before_update called twice without after_update")
        if chunk_idx != self._next:
            raise RuntimeError(f"chunks must arrive in order: expected {self._next}, got {chunk_idx}")
        slot = self.slot_of(chunk_idx)
        self._pending = (chunk_idx, slot)
        self._written = False
        return slot

    def after_update(self, chunk_idx: int) -> None:
        """Commit chunk ``chunk_idx`` (written by the attention call)."""
        if self._pending is None or self._pending[0] != chunk_idx:
            raise RuntimeError("after_update must follow before_update for the same chunk")
        if not self._written:
            raise RuntimeError("the chunk's K/V were never written (no attention call)")
        self._pending = None
        self._next = chunk_idx + 1

    # ----------------------------------------------------------- one chunk step

    def cache_positions(self, chunk_idx: int) -> list[int]:
        """Cache-relative position of every valid slot once chunk ``chunk_idx``
        is written: the slot's index among the visible keys in stream order
        (sinks, then the window oldest first; the current chunk last)."""
        valid = self.valid_length(chunk_idx)
        rows = list(range(valid))
        if chunk_idx >= self.sink_chunks + self.window_chunks:
            # ring full: ring position r holds the window's ((r - r_oldest) mod W)-th chunk
            r_oldest = (chunk_idx + 1 - self.sink_chunks) % self.window_chunks
            C, W = self.chunk_size, self.window_size
            for s in range(self.sink_size, valid):
                rows[s] = self.sink_size + (s - self.sink_size - r_oldest * C) % W
        return rows

    def attend(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, scale: float | None = None,
               norm_scope: int = binding.NORM_NONE, eps: float = 1e-6, gamma_q=None, gamma_k=None,
               rope_style: int = binding.ROPE_NONE, angles_q=None, angles_k=None,
               rope_after_cache: bool = False, angles_cache=None,
               out: torch.Tensor | None = None, lse: torch.Tensor | None = None, stream=None):
        """The attention call of one streaming step, between before_update and
        after_update.

        Before-cache RoPE (default): Q/K normalisation and RoPE of the chunk,
        its K/V written into the reserved slots (one launch), then attention of
        the chunk's queries over every valid cached key (one launch);
        ``angles_q`` / ``angles_k`` are the chunk's [C, d] angle tables (its
        absolute positions).

        After-cache RoPE (``rope_after_cache=True``): the chunk's K is written
        normalised but unrotated; then the queries and every valid cached key
        are rotated with their cache-relative positions into a scratch copy of
        the K cache (one launch) and the attention runs on that copy.
        ``angles_cache`` is the [R, d] angle table of cache positions 0 .. R - 1
        (R at least the valid length); ``angles_q`` / ``angles_k`` are unused.

        q: [B, C, Hq, d]; k, v: [B, C, H, d] (C = chunk_size). Returns
        ``(out, lse)``.
        """
        if self._pending is None:
            raise RuntimeError("attend must be called between before_update and after_update")
        chunk_idx, slot = self._pending
        if k.shape != (self.batch, self.chunk_size, self.heads, self.head_dim):
            raise ValueError("k must be [batch, chunk_size, heads, head_dim]")
        valid = self.valid_length(chunk_idx)
        if not rope_after_cache:
            q_rot = binding.stream_update(k, v, self.k, self.v, slot, q=q, norm_scope=norm_scope, eps=eps,
                                          gamma_q=gamma_q, gamma_k=gamma_k, rope_style=rope_style,
                                          angles_q=angles_q, angles_k=angles_k, stream=stream)
            self._written = True
            return binding.attn_fwd_cache(q_rot, self.k, self.v, valid, scale=scale,
                                          causal=binding.MASK_NONE, out=out, lse=lse, stream=stream)
        if rope_style == binding.ROPE_NONE or angles_cache is None:
            raise ValueError("after-cache RoPE needs a rope_style and angles_cache")
        if angles_cache.dim() != 2 or angles_cache.shape[0] < valid:
            raise ValueError("angles_cache must be [R, d] with R >= the valid cache length")
        q_norm = binding.stream_update(k, v, self.k, self.v, slot, q=q, norm_scope=norm_scope, eps=eps,
                                       gamma_q=gamma_q, gamma_k=gamma_k, rope_style=binding.ROPE_NONE,
                                       stream=stream)
        self._written = True
        if getattr(self, "_k_rot", None) is None:
            self._k_rot = torch.empty_like(self.k)
            self._rows = torch.empty(self.capacity, dtype=torch.int32, device=self.k.device)
        host_rows = torch.tensor(self.cache_positions(chunk_idx), dtype=torch.int32).pin_memory()
        self._rows[:valid].copy_(host_rows, non_blocking=True)
        q_rot, _ = binding.rope_after_cache(q_norm, self.k, valid, angles_cache, rope_style=rope_style,
                                            q_row0=valid - self.chunk_size, k_rows=self._rows,
                                            q_out=q_norm, k_rot=self._k_rot, stream=stream)
        return binding.attn_fwd_cache(q_rot, self._k_rot, self.v, valid, scale=scale,
                                      causal=binding.MASK_NONE, out=out, lse=lse, stream=stream)
