"""Pins for the key-split merge oracle: merging attention over any partition of
the keys equals attention over all keys; closed forms for two parts; empty
parts carry no weight; the merge is symmetric in its parts.

Source: developer guide, "Multi Head Attention Definition" (softmax over the
scaled scores, regrouped by disjoint key ranges).
"""

from __future__ import annotations

import math

import numpy as np
import pytest

from oracle import MASK_CHUNK, MASK_NONE, attention_fwd
from oracle.split_merge import lse_merge


def _qkv(B, Lq, Lk, Hq, Hkv, d, seed):
    g = np.random.default_rng(seed)
    return (g.standard_normal((B, Lq, Hq, d)), g.standard_normal((B, Lk, Hkv, d)),
            g.standard_normal((B, Lk, Hkv, d)))


@pytest.mark.parametrize("cuts", [[7], [1, 2, 30], [16, 32, 48], [63]])
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 1)])
def test_merge_of_a_partition_equals_full_attention(cuts, Hq, Hkv):
    B, Lq, Lk, d, scale = 2, 5, 64, 16, 0.3
    q, k, v = _qkv(B, Lq, Lk, Hq, Hkv, d, 1 + len(cuts))
    edges = [0] + cuts + [Lk]
    parts = [attention_fwd(q, k[:, a:b], v[:, a:b], scale, MASK_NONE, 0) for a, b in zip(edges, edges[1:])]
    o, lse = lse_merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    o_ref, lse_ref = attention_fwd(q, k, v, scale, MASK_NONE, 0)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_chunk_mask_split_over_the_visible_keys():
    B, Lq, Lk, d = 1, 6, 40, 8
    q, k, v = _qkv(B, Lq, Lk, 2, 2, d, 9)
    o_ref, lse_ref = attention_fwd(q, k, v, 0.4, MASK_CHUNK, 24)  # keys < 30 visible
    parts = [attention_fwd(q, k[:, a:b], v[:, a:b], 0.4, MASK_NONE, 0) for a, b in ((0, 11), (11, 30))]
    o, lse = lse_merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_two_parts_closed_form():
    # one query, one head, d = 1: parts hold a single key each
    o_parts = np.array([2.0, -1.0]).reshape(2, 1, 1, 1, 1)
    lse_parts = np.array([0.5, -0.25]).reshape(2, 1, 1, 1)
    o, lse = lse_merge(o_parts, lse_parts)
    w0 = math.exp(0.5) / (math.exp(0.5) + math.exp(-0.25))
    assert o.item() == pytest.approx(w0 * 2.0 + (1 - w0) * -1.0, abs=1e-15)
    assert lse.item() == pytest.approx(math.log(math.exp(0.5) + math.exp(-0.25)), abs=1e-15)


def test_empty_part_has_no_weight_and_order_does_not_matter():
    g = np.random.default_rng(3)
    o_parts = g.standard_normal((3, 1, 4, 2, 8))
    lse_parts = g.standard_normal((3, 1, 2, 4))
    o, lse = lse_merge(o_parts, lse_parts)
    o_e = np.concatenate([o_parts, 1e30 * np.ones((1, 1, 4, 2, 8))])  # garbage O, empty part
    lse_e = np.concatenate([lse_parts, np.full((1, 1, 2, 4), -np.inf)])
    o2, lse2 = lse_merge(o_e, lse_e)
    np.testing.assert_allclose(o2, o, rtol=1e-13)
    np.testing.assert_allclose(lse2, lse, rtol=1e-13)
    o3, lse3 = lse_merge(o_parts[::-1], lse_parts[::-1])
    np.testing.assert_allclose(o3, o, rtol=1e-13)
    np.testing.assert_allclose(lse3, lse, rtol=1e-13)
