"""Host-side bookkeeping of the rolling block K/V cache, checked against the
oracle's visible sets (no GPU: storage on the CPU, no kernel call), and the
argument contracts of attn_stream_update / attn_fwd_cache."""

from __future__ import annotations

import pytest
import torch

import head_attention_streaming_b200 as hasb
from head_attention_streaming_b200 import BlockKVCache
from oracle import rolling_cache as rc

A = 1 << 20  # fake, 16-byte aligned device addresses: validation runs before any CUDA call


@pytest.mark.parametrize("chunk,sink,window", [(4, 0, 4), (4, 4, 12), (2, 6, 4), (8, 16, 32), (3, 0, 9)])
def test_valid_slots_hold_exactly_the_oracle_visible_tokens(chunk, sink, window):
    cache = BlockKVCache(1, 1, 16, chunk, window, sink, device="cpu")
    slot_token = {}
    for c in range(12):
        slot = cache.before_update(c)
        for i in range(chunk):
            slot_token[slot + i] = c * chunk + i
        cache._written = True  # the attention call would write the chunk here
        n = cache.valid_length(c)
        held = sorted(slot_token[s] for s in range(n))
        assert held == rc.visible_tokens(c, chunk, sink, window).tolist()
        assert n <= cache.capacity
        cache.after_update(c)


def test_lifecycle_order_is_enforced():
    cache = BlockKVCache(1, 1, 16, 4, 8, 4, device="cpu")
    with pytest.raises(RuntimeError):
        cache.before_update(1)            # chunks arrive in order
    cache.before_update(0)
    with pytest.raises(RuntimeError):
        cache.before_update(0)            # twice without after_update
    with pytest.raises(RuntimeError):
        cache.after_update(0)             # nothing written yet
    cache._written = True
    with pytest.raises(RuntimeError):
        cache.after_update(1)             # wrong chunk
    cache.after_update(0)
    cache.reset()
    assert cache.before_update(0) == 0


@pytest.mark.parametrize("bad", [dict(chunk_size=0), dict(window_size=2), dict(window_size=6),
                                 dict(sink_size=3), dict(sink_size=-4)])
def test_sizes_must_be_whole_chunks(bad):
    kw = dict(batch=1, heads=1, head_dim=16, chunk_size=4, window_size=8, sink_size=4, device="cpu")
    kw.update(bad)
    with pytest.raises(ValueError):
        BlockKVCache(**kw)


def _upd(**kw):
    a = dict(q=A, q_out=A + 0x100000, k=A + 0x200000, v=A + 0x300000, kc=A + 0x400000,
             vc=A + 0x800000, gq=None, gk=None, aq=None, ak=None, B=1, L=4, S=16, slot=8, Hq=2,
             Hkv=1, d=64, scope=1, eps=1e-6, style=0, dtype=0)
    a.update(kw)
    return hasb.lib().attn_stream_update(a["q"], a["q_out"], a["k"], a["v"], a["kc"], a["vc"], a["gq"],
                                         a["gk"], a["aq"], a["ak"], a["B"], a["L"], a["S"], a["slot"],
                                         a["Hq"], a["Hkv"], a["d"], a["scope"], a["eps"], a["style"],
                                         a["dtype"], None)


UPD_INVALID = [
    dict(k=None), dict(v=None), dict(kc=None), dict(vc=None), dict(q_out=None),
    dict(slot=-1), dict(slot=13), dict(L=17), dict(S=0), dict(B=0), dict(L=0), dict(Hkv=0), dict(Hq=0),
    dict(scope=3), dict(style=3), dict(eps=-1.0), dict(dtype=5),
    dict(style=2),                                 # RoPE without angle tables
    dict(ak=A + 0xC00000),                         # angle table without RoPE
    dict(k=A + 0x200000 + 8), dict(vc=A + 0x800000 + 2),
    dict(vc=A + 0x400000 + 0x400),                 # caches overlap each other (2 KB each)
    dict(kc=A + 0x200000),                         # cache overlaps the K input
    dict(q_out=A + 0x400000),                      # q_out overlaps a cache
]


@pytest.mark.parametrize("kw", UPD_INVALID, ids=[str(k) for k in UPD_INVALID])
def test_stream_update_invalid_arguments(kw):
    assert _upd(**kw) == hasb.ATTN_ERR_INVALID_ARG


def test_fwd_cache_rejects_a_prefix_longer_than_the_cache():
    L = hasb.lib()
    st = L.attn_fwd_cache(A, A + 0x100000, A + 0x200000, A + 0x300000, None, 1, 4, 9, 8, 2, 1, 128, 0.1,
                          0, 0, 0, None)
    assert st == hasb.ATTN_ERR_INVALID_ARG
    st = L.attn_fwd_cache(A, A + 0x100000, A + 0x200000, A + 0x300000, None, 1, 4, 4, 0, 2, 1, 128, 0.1,
                          0, 0, 0, None)
    assert st == hasb.ATTN_ERR_INVALID_ARG
