"""The chunk plan of attn_fwd_host (host logic of the C ABI, no GPU): the
chunks tile every query row of every batch exactly once, in order; there are
at most 16 of them; a chunk holds whole 256-row work units (only a batch's last
chunk may end on a ragged row count); several batches share a chunk only as
whole batches; and a call is cut only as far as every chunk keeps at least
2 MB of Q (except when the whole Q is smaller: one chunk)."""

from __future__ import annotations

import itertools

import pytest

import head_attention_streaming_b200 as hasb

MIN_BYTES = 2 << 20


def _check(B, Lq, Hq, d):
    plan = hasb.host_chunks(B, Lq, Hq, d)
    assert 1 <= len(plan) <= 16
    q_bytes = B * Lq * Hq * d * 2
    want = max(1, min(16, q_bytes // MIN_BYTES))
    seen = []
    for b0, nb, r0, n in plan:
        assert nb >= 1 and n >= 1 and 0 <= b0 and b0 + nb <= B and 0 <= r0 and r0 + n <= Lq
        if nb > 1:
            assert (r0, n) == (0, Lq)
        assert r0 % 256 == 0
        assert n % 256 == 0 or r0 + n == Lq
        seen.extend((b, r) for b in range(b0, b0 + nb) for r in range(r0, r0 + n))
    assert seen == [(b, r) for b in range(B) for r in range(Lq)]  # each row once, in order
    assert len(plan) <= want
    return plan


@pytest.mark.parametrize("B,Lq,Hq,d", list(itertools.product((1, 2, 3, 17, 64), (1, 100, 257, 1785, 5000),
                                                                (1, 8, 40), (64, 128))))
def test_plan_tiles_the_call(B, Lq, Hq, d):
    _check(B, Lq, Hq, d)


def test_known_plans():
    # the video workload: 16 chunks of 1280 rows (18.4 MB of Q each)
    assert hasb.host_chunks(1, 20480, 56, 128) == [(0, 1, 1280 * c, 1280) for c in range(16)]
    # FP16 causal [2, 2048, 8, 64]: 4.2 MB of Q, one chunk per batch
    assert hasb.host_chunks(2, 2048, 8, 64) == [(0, 1, 0, 2048), (1, 1, 0, 2048)]
    # under 2 MB of Q: one chunk
    assert hasb.host_chunks(1, 257, 8, 128) == [(0, 1, 0, 257)]
    # 64 batches, 39 MB: 16 chunks of 4 whole batches
    assert hasb.host_chunks(64, 300, 8, 128) == [(4 * c, 4, 0, 300) for c in range(16)]


def test_bad_sizes_are_refused():
    with pytest.raises(hasb.AttnError) as e:
        hasb.host_chunks(0, 10, 1, 64)
    assert e.value.status == hasb.ATTN_ERR_INVALID_ARG
