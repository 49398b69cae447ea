"""Streaming self-attention through the rolling block K/V cache on a B200,
against the FP64 oracle: before_update, attend (the chunk's Q/K RMSNorm and
before-cache RoPE, its K/V written into the cache, attention over every valid
cached key), after_update, for streams that fill the cache and then evict.

Expected values: the prologue oracle on the 16-bit inputs, rounded to the
16-bit type (the cache stores 16-bit K; Q enters the attention as 16 bits),
then the rolling-cache oracle. Bars as in the attention parity tests.
"""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import head_attention_streaming_b200 as hasb
import oracle
from head_attention_streaming_b200.inputs import rope_angle_table
from oracle import prologue as qp
from oracle import rolling_cache as rc
from test_parity_gpu import _check, _pbound

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_ok):
    torch.cuda.set_device(0)
    yield
    assert hasb.device_fault(clear=True) == 0


def _round16(x: np.ndarray, dtype) -> np.ndarray:
    return torch.from_numpy(x).to(dtype).to(torch.float64).numpy()


def _stream(B, C, sink, window, Hq, Hkv, d, n_chunks, dtype, norm, style, seed, sample_rows=None):
    g = torch.Generator().manual_seed(seed)
    T = n_chunks * C
    q = torch.randn(B, T, Hq, d, generator=g).to(dtype)
    k = torch.randn(B, T, Hkv, d, generator=g).to(dtype)
    v = torch.randn(B, T, Hkv, d, generator=g).to(dtype)
    wq, wk = (d, d) if norm == qp.NORM_HEAD else (Hq * d, Hkv * d)
    gq = (1.0 + 0.1 * torch.randn(wq, generator=g)) if norm else None
    gk = (1.0 + 0.1 * torch.randn(wk, generator=g)) if norm else None
    ang = rope_angle_table(T, d, style, 0) if style else None
    scale = 1.0 / math.sqrt(d)
    eps = 1e-6
    f64 = lambda t: None if t is None else t.to(torch.float64).numpy()
    kn = _round16(qp.qk_prologue(f64(k), f64(gk), eps, norm, f64(ang), style), dtype)
    vn = f64(v)
    cache = hasb.BlockKVCache(B, Hkv, d, C, window, sink, dtype=dtype)
    dev = lambda t: None if t is None else t.cuda()
    tag = "bf16" if dtype == torch.bfloat16 else "fp16"
    for c in range(n_chunks):
        sl = slice(c * C, (c + 1) * C)
        cache.before_update(c)
        o, lse = cache.attend(dev(q[:, sl].contiguous()), dev(k[:, sl].contiguous()),
                              dev(v[:, sl].contiguous()), scale=scale, norm_scope=norm, eps=eps,
                              gamma_q=dev(gq), gamma_k=dev(gk), rope_style=style,
                              angles_q=dev(ang[sl].contiguous()) if style else None,
                              angles_k=dev(ang[sl].contiguous()) if style else None)
        torch.cuda.synchronize()
        cache.after_update(c)
        qn = _round16(qp.qk_prologue(f64(q[:, sl]), f64(gq), eps, norm,
                                     None if ang is None else f64(ang[sl]), style), dtype)
        idx = rc.visible_tokens(c, C, sink, window)
        rows = sample_rows
        o_ref, lse_ref = oracle.attention_fwd(qn, kn[:, idx], vn[:, idx], scale, oracle.MASK_NONE, 0,
                                              rows=rows)
        o_cpu, lse_cpu = o.cpu(), lse.cpu()
        if rows is not None:
            o_cpu, lse_cpu = o_cpu[:, rows], lse_cpu[:, :, rows]
        pb = _pbound(qn, kn[:, idx], vn[:, idx], scale, tag) if sample_rows is None else None
        _check(o_cpu, lse_cpu, o_ref, lse_ref, tag, what=f"chunk {c}", p_bound=pb)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_fill_then_evict_with_sink_norm_and_rope(dtype):
    """Chunk 64, one sink chunk, a three-chunk window: chunks 0-3 fill the
    cache, chunks 4-6 evict the oldest window chunk each."""
    _stream(2, 64, 64, 192, 4, 2, 128, 7, dtype, qp.NORM_HEAD, qp.ROPE_SPLIT, seed=1)


def test_sliding_window_without_sink_interleaved_inner_norm():
    _stream(1, 128, 0, 256, 4, 4, 64, 5, torch.bfloat16, qp.NORM_INNER, qp.ROPE_INTERLEAVED, seed=2)


def test_ragged_chunk_no_prologue():
    """A chunk length that is not a multiple of the 128-row tiles."""
    _stream(1, 100, 100, 300, 2, 1, 128, 6, torch.bfloat16, qp.NORM_NONE, qp.ROPE_NONE, seed=3)


def test_dit_stream_full_size_through_eviction():
    """1785-token chunks of the DiT video stream, 40 query heads over 8 K/V
    heads, a four-chunk window (7140 keys at steady state), head RMSNorm and
    split-half RoPE: five chunks, the fifth evicting the first; 64 sampled
    rows per chunk against the oracle."""
    rows = np.sort(np.random.default_rng(7).choice(1785, size=64, replace=False))
    _stream(1, 1785, 0, 7140, 40, 8, 128, 5, torch.bfloat16, qp.NORM_HEAD, qp.ROPE_SPLIT, seed=4,
            sample_rows=rows)


@pytest.mark.parametrize("style,sink,window,n_chunks,dtype", [
    (qp.ROPE_SPLIT, 128, 256, 6, torch.bfloat16),        # sink + ring, evictions from chunk 3 on
    (qp.ROPE_INTERLEAVED, 0, 384, 5, torch.float16),     # window only, evictions from chunk 3 on
])
def test_after_cache_rope_stream(style, sink, window, n_chunks, dtype):
    """RoPE after the cache update: the cache keeps normalised, unrotated K;
    each step rotates the queries and every valid cached key with their
    cache-relative positions (the oracle's reading) before attending."""
    B, C, Hq, Hkv, d = 2, 128, 4, 2, 128
    g = torch.Generator().manual_seed(50 + n_chunks)
    T = n_chunks * C
    q = torch.randn(B, T, Hq, d, generator=g).to(dtype)
    k = torch.randn(B, T, Hkv, d, generator=g).to(dtype)
    v = torch.randn(B, T, Hkv, d, generator=g).to(dtype)
    gq = 1.0 + 0.1 * torch.randn(d, generator=g)
    gk = 1.0 + 0.1 * torch.randn(d, generator=g)
    ang = rope_angle_table(sink + window, d, style, 0)       # cache positions 0 .. sink + window - 1
    scale, eps = 1.0 / math.sqrt(d), 1e-6
    f64 = lambda t: t.to(torch.float64).numpy()
    qn = _round16(qp.rms_norm(f64(q), f64(gq), eps, qp.NORM_HEAD), dtype)
    kn = _round16(qp.rms_norm(f64(k), f64(gk), eps, qp.NORM_HEAD), dtype)
    q_chunks = [qn[:, c * C:(c + 1) * C] for c in range(n_chunks)]
    r16 = lambda x: _round16(x, dtype)
    ref = rc.stream_attention_after_rope(q_chunks, kn, f64(v), C, sink, window, scale, f64(ang), style,
                                         round_rotated=r16)
    rotated = rc.after_rope_inputs(q_chunks, kn, f64(v), C, sink, window, f64(ang), style,
                                   round_rotated=r16)
    cache = hasb.BlockKVCache(B, Hkv, d, C, window, sink, dtype=dtype)
    tag = "bf16" if dtype == torch.bfloat16 else "fp16"
    for c in range(n_chunks):
        sl = slice(c * C, (c + 1) * C)
        cache.before_update(c)
        o, lse = cache.attend(q[:, sl].contiguous().cuda(), k[:, sl].contiguous().cuda(),
                              v[:, sl].contiguous().cuda(), scale=scale, norm_scope=hasb.NORM_HEAD, eps=eps,
                              gamma_q=gq.cuda(), gamma_k=gk.cuda(), rope_style=style,
                              rope_after_cache=True, angles_cache=ang.cuda())
        torch.cuda.synchronize()
        cache.after_update(c)
        _check(o.cpu(), lse.cpu(), *ref[c], tag, what=f"after-cache chunk {c}",
               p_bound=_pbound(*rotated[c], scale, tag))
    # the cache itself keeps the normalised, unrotated keys of the visible chunks
    stored = cache.k.cpu().to(torch.float64).numpy()
    last = n_chunks - 1
    for c2 in sorted(set(int(t) // C for t in rc.visible_tokens(last, C, sink, window))):
        s0 = cache.slot_of(c2)
        want = kn[:, c2 * C:(c2 + 1) * C]
        assert np.abs(stored[:, s0:s0 + C] - want).max() <= 2 ** -7 * np.abs(want).max(), c2


def test_rope_after_cache_rows_and_batch_stride():
    """attn_rope_after_cache on its own: a B = 2 cache with S > Lk (batch
    stride S), a row map that permutes the slots, slots past Lk untouched."""
    B, S, Lk, Lq, H, d = 2, 300, 250, 40, 2, 64
    g = torch.Generator().manual_seed(61)
    kc = torch.randn(B, S, H, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, Lq, 4, d, generator=g).to(torch.bfloat16)
    ang = rope_angle_table(Lk, d, qp.ROPE_SPLIT, 0)
    perm = torch.randperm(Lk, generator=g).to(torch.int32)
    k_rot = torch.full((B, S, H, d), 3.0, dtype=torch.bfloat16, device="cuda")
    q_out, _ = hasb.rope_after_cache(q.cuda(), kc.cuda(), Lk, ang.cuda(), rope_style=hasb.ROPE_SPLIT,
                                     q_row0=Lk - Lq, k_rows=perm.cuda(), k_rot=k_rot)
    torch.cuda.synchronize()
    f64 = lambda t: t.to(torch.float64).numpy()
    a = f64(ang)
    want_k = _round16(qp.rope(f64(kc[:, :Lk]), a[perm.long().numpy()], qp.ROPE_SPLIT), torch.bfloat16)
    want_q = _round16(qp.rope(f64(q), a[Lk - Lq:], qp.ROPE_SPLIT), torch.bfloat16)
    got_k = f64(k_rot.cpu())
    assert np.abs(got_k[:, :Lk] - want_k).max() <= 2 ** -7 * np.abs(want_k).max()
    assert np.all(got_k[:, Lk:] == 3.0)
    assert np.abs(f64(q_out.cpu()) - want_q).max() <= 2 ** -7 * np.abs(want_q).max()
