"""Pins for the FP64 oracle: it is checked against things other than itself.

* brute force on tiny inputs (pure Python floats, additive -inf mask,
  exactly rounded sums) over every mask mode, GQA ratio and head size;
* PyTorch's float64 scaled_dot_product_attention on CPU (a library routine)
  with repeat-interleaved K/V heads and an explicit boolean mask, plus
  ``torch.logsumexp`` for the LSE;
* closed forms (zero queries or zero scale give the mean of the visible V rows;
  one key returns its V row; two keys give logistic weights; constant V);
* invariants (weights sum to one, invisible keys have no effect, key
  permutation, GQA equals MHA with replicated heads, chunk mode equals
  no mask on the truncated cache, causal row i equals a one-row chunk);
* hand-derived golden fixtures under tests/golden/;
* planted mistakes: each plausible slip in the oracle (wrong head map,
  off-by-one causal limit, dropped offset, LSE base) makes a pin fail.
"""

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import attention as oracle_mod

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, rng, scale=1.0):
    return rng.standard_normal(shape) * scale


def _brute_force(q, k, v, scale, mask, kv_offset):
    """Pure-Python attention: all scores, additive -inf mask, fsum reductions."""
    B, Lq, Hq, d = q.shape
    _, Lk, Hkv, _ = k.shape
    group = Hq // Hkv
    o = np.zeros((B, Lq, Hq, d))
    lse = np.zeros((B, Hq, Lq))
    for b in range(B):
        for h in range(Hq):
            g = h // group
            for i in range(Lq):
                if mask == 0:
                    lim = Lk
                elif mask == 1:
                    lim = min(Lk, kv_offset + i + 1)
                else:
                    lim = min(Lk, kv_offset + Lq)
                s = []
                for j in range(Lk):
                    dot = math.fsum(float(q[b, i, h, c]) * float(k[b, j, g, c]) for c in range(d))
                    s.append(scale * dot + (0.0 if j < lim else -math.inf))
                mx = max(s)
                w = [math.exp(x - mx) for x in s]
                tot = math.fsum(w)
                for c in range(d):
                    o[b, i, h, c] = math.fsum(w[j] * float(v[b, j, g, c]) for j in range(Lk)) / tot
                lse[b, h, i] = mx + math.log(tot)
    return o, lse


def _torch_sdpa(q, k, v, scale, mask, kv_offset):
    """torch float64 SDPA with explicit boolean mask and replicated K/V heads."""
    B, Lq, Hq, d = q.shape
    Lk, Hkv = k.shape[1], k.shape[2]
    group = Hq // Hkv
    tq = torch.from_numpy(q).permute(0, 2, 1, 3)                     # [B,Hq,Lq,d]
    tk = torch.from_numpy(k).repeat_interleave(group, dim=2).permute(0, 2, 1, 3)
    tv = torch.from_numpy(v).repeat_interleave(group, dim=2).permute(0, 2, 1, 3)
    if mask == 0:
        allowed = torch.ones(Lq, Lk, dtype=torch.bool)
    elif mask == 1:
        allowed = torch.ones(Lq, Lk, dtype=torch.bool).tril(diagonal=kv_offset)
    else:
        allowed = torch.zeros(Lq, Lk, dtype=torch.bool)
        allowed[:, : kv_offset + Lq] = True
    out = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=allowed,
                                                            scale=scale)
    scores = (tq @ tk.transpose(-1, -2)) * scale
    scores = scores.masked_fill(~allowed, -math.inf)
    lse = torch.logsumexp(scores, dim=-1)                          # [B,Hq,Lq]
    return out.permute(0, 2, 1, 3).numpy(), lse.numpy()


def _cases_tiny():
    cases = []
    for (Lq, Lk) in [(1, 1), (2, 3), (3, 5), (5, 5), (4, 17)]:
        for (Hq, Hkv) in [(1, 1), (4, 2), (4, 1)]:
            for mask in (0, 1, 2):
                offsets = [0] if mask == 0 else sorted({0, Lk - Lq}) if Lk >= Lq else []
                for off in offsets:
                    cases.append((Lq, Lk, Hq, Hkv, mask, off))
    return cases


@pytest.mark.parametrize("Lq,Lk,Hq,Hkv,mask,off", _cases_tiny())
def test_brute_force_tiny(Lq, Lk, Hq, Hkv, mask, off):
    rng = np.random.default_rng(1000 + Lq * 31 + Lk * 7 + Hq + mask)
    d = 8
    B = 2 if Lq < 4 else 1
    q = _rand((B, Lq, Hq, d), rng)
    k = _rand((B, Lk, Hkv, d), rng)
    v = _rand((B, Lk, Hkv, d), rng)
    scale = 0.37
    o, lse = oracle.attention_fwd(q, k, v, scale, mask, off)
    ob, lseb = _brute_force(q, k, v, scale, mask, off)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lseb, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("mask,Lq,Lk,off", [(0, 17, 129, 0), (1, 129, 129, 0), (1, 17, 129, 100),
                                            (2, 17, 129, 50), (2, 33, 129, 96)])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2), (4, 1)])
def test_torch_sdpa_float64(d, mask, Lq, Lk, off, Hq, Hkv):
    rng = np.random.default_rng(7 + d + mask * 3 + Lq + off + Hkv)
    q = _rand((2, Lq, Hq, d), rng)
    k = _rand((2, Lk, Hkv, d), rng)
    v = _rand((2, Lk, Hkv, d), rng)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attention_fwd(q, k, v, scale, mask, off)
    ot, lset = _torch_sdpa(q, k, v, scale, mask, off)
    np.testing.assert_allclose(o, ot, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lse, lset, rtol=1e-10, atol=1e-12)


def test_rows_subset_matches_full():
    rng = np.random.default_rng(3)
    q = _rand((1, 40, 2, 16), rng)
    k = _rand((1, 50, 1, 16), rng)
    v = _rand((1, 50, 1, 16), rng)
    rows = [0, 3, 17, 39]
    for mask, off in [(0, 0), (1, 10), (2, 10)]:
        o, lse = oracle.attention_fwd(q, k, v, 0.25, mask, off)
        os_, lses = oracle.attention_fwd(q, k, v, 0.25, mask, off, rows=rows)
        np.testing.assert_array_equal(os_, o[:, rows])
        np.testing.assert_array_equal(lses, lse[:, :, rows])


# ---------------------------------------------------------------- closed forms

@pytest.mark.parametrize("mask,off", [(0, 0), (1, 0), (1, 7), (2, 7)])
def test_zero_query_is_mean_of_visible_values(mask, off):
    rng = np.random.default_rng(11)
    Lq, Lk = 6, 13
    q = np.zeros((1, Lq, 2, 8))
    k = _rand((1, Lk, 2, 8), rng)
    v = _rand((1, Lk, 2, 8), rng)
    o, lse = oracle.attention_fwd(q, k, v, 0.3, mask, off)
    for i in range(Lq):
        n = Lk if mask == 0 else (off + i + 1 if mask == 1 else off + Lq)
        np.testing.assert_allclose(o[0, i], v[0, :n].mean(axis=0), rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse[0, :, i], math.log(n), rtol=1e-14)


def test_zero_scale_is_mean_of_values():
    rng = np.random.default_rng(12)
    q = _rand((1, 4, 1, 8), rng)
    k = _rand((1, 9, 1, 8), rng)
    v = _rand((1, 9, 1, 8), rng)
    o, lse = oracle.attention_fwd(q, k, v, 0.0)
    np.testing.assert_allclose(o[0, :, 0], np.broadcast_to(v[0, :, 0].mean(0), (4, 8)),
                               rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, math.log(9), rtol=1e-14)


def test_single_key_returns_its_value_row():
    rng = np.random.default_rng(13)
    q = _rand((2, 5, 3, 8), rng)
    k = _rand((2, 1, 3, 8), rng)
    v = _rand((2, 1, 3, 8), rng)
    o, lse = oracle.attention_fwd(q, k, v, 0.7)
    for b in range(2):
        for h in range(3):
            for i in range(5):
                np.testing.assert_array_equal(o[b, i, h], v[b, 0, h])
                assert lse[b, h, i] == pytest.approx(0.7 * float(q[b, i, h] @ k[b, 0, h]),
                                                     rel=1e-14, abs=1e-15)


def test_causal_row_zero_returns_first_value_row():
    rng = np.random.default_rng(14)
    q = _rand((1, 4, 2, 8), rng)
    k = _rand((1, 4, 2, 8), rng)
    v = _rand((1, 4, 2, 8), rng)
    o, _ = oracle.attention_fwd(q, k, v, 0.5, oracle.MASK_CAUSAL, 0)
    np.testing.assert_array_equal(o[0, 0], v[0, 0])


def test_two_keys_logistic():
    rng = np.random.default_rng(15)
    q = _rand((1, 3, 1, 8), rng)
    k = _rand((1, 2, 1, 8), rng)
    v = _rand((1, 2, 1, 8), rng)
    scale = 0.9
    o, lse = oracle.attention_fwd(q, k, v, scale)
    for i in range(3):
        s0 = scale * float(q[0, i, 0] @ k[0, 0, 0])
        s1 = scale * float(q[0, i, 0] @ k[0, 1, 0])
        w0 = 1.0 / (1.0 + math.exp(s1 - s0))
        np.testing.assert_allclose(o[0, i, 0], w0 * v[0, 0, 0] + (1 - w0) * v[0, 1, 0],
                                   rtol=1e-13, atol=1e-14)
        assert lse[0, 0, i] == pytest.approx(max(s0, s1) + math.log1p(math.exp(-abs(s0 - s1))),
                                             rel=1e-14)


def test_constant_values_give_constant_output():
    rng = np.random.default_rng(16)
    q = _rand((1, 7, 2, 8), rng, 3.0)
    k = _rand((1, 11, 2, 8), rng, 3.0)
    v = np.full((1, 11, 2, 8), -1.25)
    for mask, off in [(0, 0), (1, 4), (2, 4)]:
        o, _ = oracle.attention_fwd(q, k, v, 0.4, mask, off)
        np.testing.assert_allclose(o, -1.25, rtol=1e-14)


@pytest.mark.parametrize("name", ["two_key_logistic.json", "causal_zero_query_running_mean.json"])
def test_golden_fixture(name):
    with open(os.path.join(GOLDEN, name)) as f:
        fx = json.load(f)
    o, lse = oracle.attention_fwd(np.array(fx["q"]), np.array(fx["k"]), np.array(fx["v"]),
                                  fx["scale"], fx["mask"], fx["kv_offset"])
    np.testing.assert_allclose(o, np.array(fx["o"]), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(lse, np.array(fx["lse"]), rtol=1e-14, atol=1e-15)


def test_golden_fixture_numbers_follow_their_closed_forms():
    with open(os.path.join(GOLDEN, "two_key_logistic.json")) as f:
        fx = json.load(f)
    assert fx["o"][0][0][0][0] == pytest.approx(1 / (1 + math.exp(-1)), rel=1e-15)
    assert fx["lse"][0][0][0] == pytest.approx(math.log(1 + math.e), rel=1e-15)


# ------------------------------------------------------------------ invariants

@pytest.mark.parametrize("mask,off", [(0, 0), (1, 0), (1, 5), (2, 5)])
def test_weights_sum_to_one_and_vanish_on_invisible_keys(mask, off):
    rng = np.random.default_rng(21)
    Lq, Lk = 6, 12
    q = _rand((1, Lq, 2, 8), rng, 2.0)
    k = _rand((1, Lk, 1, 8), rng, 2.0)
    v = _rand((1, Lk, 1, 8), rng)
    _, _, w = oracle.attention_fwd(q, k, v, 0.5, mask, off, return_weights=True)
    for h in range(2):
        for i in range(Lq):
            assert math.fsum(w[0, h, i]) == pytest.approx(1.0, abs=1e-14)
            lim = oracle.visible_limit(mask, i, Lq, Lk, off)
            assert np.all(w[0, h, i, lim:] == 0.0)
            assert np.all(w[0, h, i, :lim] > 0.0)


@pytest.mark.parametrize("mask,off", [(1, 0), (1, 3), (2, 3)])
def test_invisible_keys_have_no_effect(mask, off):
    rng = np.random.default_rng(22)
    Lq, Lk = 5, 14
    q = _rand((1, Lq, 2, 8), rng)
    k = _rand((1, Lk, 2, 8), rng)
    v = _rand((1, Lk, 2, 8), rng)
    o, lse = oracle.attention_fwd(q, k, v, 0.5, mask, off)
    k2, v2 = k.copy(), v.copy()
    first_hidden = off + Lq          # no row sees keys from here on
    k2[:, first_hidden:] = _rand(k2[:, first_hidden:].shape, rng, 50.0)
    v2[:, first_hidden:] = 1e6
    o2, lse2 = oracle.attention_fwd(q, k2, v2, 0.5, mask, off)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    if mask == 1:
        # row by row: causal row i equals unmasked attention on keys 0..off+i
        for i in range(Lq):
            oi, li = oracle.attention_fwd(q[:, i:i + 1], k[:, : off + i + 1], v[:, : off + i + 1], 0.5)
            np.testing.assert_allclose(o[:, i], oi[:, 0], rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(lse[:, :, i], li[:, :, 0], rtol=1e-13)


def test_key_permutation_invariance():
    rng = np.random.default_rng(23)
    q = _rand((1, 6, 2, 8), rng)
    k = _rand((1, 15, 2, 8), rng)
    v = _rand((1, 15, 2, 8), rng)
    perm = rng.permutation(15)
    o, lse = oracle.attention_fwd(q, k, v, 0.6)
    o2, lse2 = oracle.attention_fwd(q, k[:, perm], v[:, perm], 0.6)
    np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, lse2, rtol=1e-13)


def test_gqa_equals_mha_with_replicated_heads():
    rng = np.random.default_rng(24)
    Hq, Hkv = 6, 2
    q = _rand((1, 5, Hq, 8), rng)
    k = _rand((1, 9, Hkv, 8), rng)
    v = _rand((1, 9, Hkv, 8), rng)
    group = Hq // Hkv
    krep = np.repeat(k, group, axis=2)      # head h -> kv head h // group
    vrep = np.repeat(v, group, axis=2)
    for mask, off in [(0, 0), (1, 4), (2, 4)]:
        o, lse = oracle.attention_fwd(q, k, v, 0.3, mask, off)
        o2, lse2 = oracle.attention_fwd(q, krep, vrep, 0.3, mask, off)
        np.testing.assert_array_equal(o, o2)
        np.testing.assert_array_equal(lse, lse2)


def test_chunk_mode_equals_no_mask_on_truncated_cache():
    rng = np.random.default_rng(25)
    Lq, Lk, off = 4, 20, 9
    q = _rand((1, Lq, 2, 8), rng)
    k = _rand((1, Lk, 1, 8), rng)
    v = _rand((1, Lk, 1, 8), rng)
    o, lse = oracle.attention_fwd(q, k, v, 0.5, oracle.MASK_CHUNK, off)
    o2, lse2 = oracle.attention_fwd(q, k[:, : off + Lq], v[:, : off + Lq], 0.5)
    np.testing.assert_allclose(o, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, lse2, rtol=1e-13)


def test_causal_row_equals_one_row_chunk():
    rng = np.random.default_rng(26)
    L = 9
    q = _rand((1, L, 2, 8), rng)
    k = _rand((1, L, 2, 8), rng)
    v = _rand((1, L, 2, 8), rng)
    o, lse = oracle.attention_fwd(q, k, v, 0.5, oracle.MASK_CAUSAL, 0)
    for i in range(L):
        oi, li = oracle.attention_fwd(q[:, i:i + 1], k, v, 0.5, oracle.MASK_CHUNK, i)
        np.testing.assert_allclose(o[:, i], oi[:, 0], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(lse[:, :, i], li[:, :, 0], rtol=1e-13)


def test_flops_convention():
    assert oracle.flops(1, 257, 257, 8, 128, 0) == 4 * 257 * 257 * 8 * 128
    assert oracle.flops(2, 2048, 2048, 8, 64, 1) == 2 * 2 * 2048 * 2048 * 8 * 64


# ------------------------------------------------------------ planted mistakes

def _pins_pass():
    """Run a compact set of pins against whatever the oracle module holds now."""
    ok = True
    rng = np.random.default_rng(99)
    q = _rand((1, 5, 4, 8), rng)
    k = _rand((1, 7, 2, 8), rng)
    v = _rand((1, 7, 2, 8), rng)
    for mask, off in [(0, 0), (1, 2), (2, 2)]:
        o, lse = oracle_mod.attention_fwd(q, k, v, 0.5, mask, off)
        ot, lset = _torch_sdpa(q, k, v, 0.5, mask, off)
        ok &= np.allclose(o, ot, rtol=1e-10, atol=1e-12) and np.allclose(lse, lset, rtol=1e-10)
    with open(os.path.join(GOLDEN, "causal_zero_query_running_mean.json")) as f:
        fx = json.load(f)
    o, lse = oracle_mod.attention_fwd(np.array(fx["q"]), np.array(fx["k"]), np.array(fx["v"]),
                                      fx["scale"], fx["mask"], fx["kv_offset"])
    ok &= np.allclose(o, np.array(fx["o"])) and np.allclose(lse, np.array(fx["lse"]))
    return bool(ok)


def test_pins_pass_on_the_unmodified_oracle():
    assert _pins_pass()


@pytest.mark.parametrize("mutation", ["head_map_modulo", "causal_strict", "causal_no_offset",
                                      "chunk_as_causal"])
def test_planted_mistake_is_caught(monkeypatch, mutation):
    orig_limit = oracle_mod.visible_limit
    if mutation == "head_map_modulo":
        monkeypatch.setattr(oracle_mod, "kv_head", lambda hq, Hq, Hkv: hq % Hkv)
    elif mutation == "causal_strict":
        monkeypatch.setattr(oracle_mod, "visible_limit",
                            lambda m, i, Lq, Lk, off: max(1, orig_limit(m, i, Lq, Lk, off) - (m == 1)))
    elif mutation == "causal_no_offset":
        monkeypatch.setattr(oracle_mod, "visible_limit",
                            lambda m, i, Lq, Lk, off: orig_limit(m, i, Lq, Lk, 0 if m == 1 else off))
    elif mutation == "chunk_as_causal":
        monkeypatch.setattr(oracle_mod, "visible_limit",
                            lambda m, i, Lq, Lk, off: orig_limit(1 if m == 2 else m, i, Lq, Lk, off))
    assert not _pins_pass()


def test_planted_lse_base_mistake_is_caught(monkeypatch):
    real_log = np.log
    monkeypatch.setattr(oracle_mod.np, "log", lambda x: real_log(x) / math.log(2.0))
    try:
        caught = not _pins_pass()
    finally:
        monkeypatch.setattr(oracle_mod.np, "log", real_log)
    assert caught
