"""Pins for the Q/K prologue oracle (RMSNorm, then RoPE) against things other
than itself: a library routine, closed forms, invariants, an independent
complex-number formulation of the rotation and a hand-derived golden fixture.
Each planted mistake at the end must be caught by at least one pin.

Source: flashdreams.accelerated developer guide, "Multi Head Attention
Definition" (RMSNorm equation; RoPE rotation, interleaved and split-half
pairings; normalisation before RoPE).
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import prologue as qp

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _angles(L, d, style, base=10000.0, pos0=0):
    """Page construction of the angle table, expanded to one angle per feature."""
    r = np.arange(d // 2)
    omega = base ** (-2.0 * r / d)
    theta = (pos0 + np.arange(L))[:, None] * omega[None, :]
    out = np.zeros((L, d))
    a, b = qp.pairs(d, style)
    out[:, a] = theta
    out[:, b] = theta
    return out


# ------------------------------------------------------------------ RMSNorm

@pytest.mark.parametrize("scope", [qp.NORM_HEAD, qp.NORM_INNER])
@pytest.mark.parametrize("d", [16, 64, 128])
def test_rmsnorm_matches_torch_rms_norm(scope, d):
    B, L, H = 2, 5, 3
    x = _rand((B, L, H, d), 1 + d + scope)
    m = d if scope == qp.NORM_HEAD else H * d
    gamma = 1.0 + 0.1 * _rand((m,), 7)
    eps = 1e-6
    got = qp.rms_norm(x, gamma, eps, scope)
    xt = torch.from_numpy(x)
    if scope == qp.NORM_HEAD:
        want = torch.nn.functional.rms_norm(xt, (d,), torch.from_numpy(gamma), eps)
    else:
        want = torch.nn.functional.rms_norm(xt.reshape(B, L, H * d), (H * d,),
                                            torch.from_numpy(gamma), eps).reshape(B, L, H, d)
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-13, atol=1e-13)


def test_rmsnorm_closed_form_three_four():
    x = np.array([3.0, 4.0]).reshape(1, 1, 1, 2)
    got = qp.rms_norm(x, None, 0.0, qp.NORM_HEAD).ravel()
    rms = math.sqrt((9.0 + 16.0) / 2.0)
    assert got[0] == pytest.approx(3.0 / rms, abs=1e-15)
    assert got[1] == pytest.approx(4.0 / rms, abs=1e-15)


@pytest.mark.parametrize("scope", [qp.NORM_HEAD, qp.NORM_INNER])
def test_rmsnorm_unit_mean_square_and_scale_invariance(scope):
    x = _rand((1, 4, 3, 32), 11)
    y = qp.rms_norm(x, None, 0.0, scope)
    groups = y if scope == qp.NORM_HEAD else y.reshape(1, 4, 1, 96)
    np.testing.assert_allclose(np.mean(groups * groups, axis=-1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(qp.rms_norm(7.5 * x, None, 0.0, scope), y, rtol=1e-12)


def test_rmsnorm_scopes_agree_with_one_head_and_zero_input_stays_zero():
    x = _rand((2, 3, 1, 64), 12)
    g = 1.0 + 0.2 * _rand((64,), 13)
    np.testing.assert_allclose(qp.rms_norm(x, g, 1e-6, qp.NORM_HEAD),
                               qp.rms_norm(x, g, 1e-6, qp.NORM_INNER), rtol=1e-14)
    z = np.zeros((1, 1, 2, 8))
    assert np.all(qp.rms_norm(z, None, 1e-6, qp.NORM_HEAD) == 0.0)


def test_rmsnorm_heads_are_independent_in_head_scope_only():
    x = _rand((1, 2, 4, 16), 14)
    x2 = x.copy()
    x2[:, :, 1, :] *= 100.0  # one head much larger
    yh, yh2 = qp.rms_norm(x, None, 1e-6, qp.NORM_HEAD), qp.rms_norm(x2, None, 1e-6, qp.NORM_HEAD)
    np.testing.assert_allclose(yh[:, :, [0, 2, 3]], yh2[:, :, [0, 2, 3]], rtol=1e-13)
    yi, yi2 = qp.rms_norm(x, None, 1e-6, qp.NORM_INNER), qp.rms_norm(x2, None, 1e-6, qp.NORM_INNER)
    assert not np.allclose(yi[:, :, 0], yi2[:, :, 0])


# --------------------------------------------------------------------- RoPE

def _rope_complex(x, angles, style):
    """Independent formulation: each pair as a complex number times e^{i theta}."""
    B, L, H, d = x.shape
    a, b = qp.pairs(d, style)
    z = x[..., a] + 1j * x[..., b]
    theta = np.asarray(angles)[:, a][None, :, None, :]
    w = z * np.exp(1j * theta)
    y = np.empty_like(x)
    y[..., a] = w.real
    y[..., b] = w.imag
    return y


@pytest.mark.parametrize("style", [qp.ROPE_INTERLEAVED, qp.ROPE_SPLIT])
@pytest.mark.parametrize("d", [16, 128])
def test_rope_matches_complex_multiplication(style, d):
    x = _rand((2, 6, 3, d), 20 + d + style)
    ang = _angles(6, d, style, pos0=1000)
    np.testing.assert_allclose(qp.rope(x, ang, style), _rope_complex(x, ang, style),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("style", [qp.ROPE_INTERLEAVED, qp.ROPE_SPLIT])
def test_rope_special_angles_and_pair_norms(style):
    d = 8
    x = _rand((1, 1, 1, d), 30)
    a, b = qp.pairs(d, style)
    zero = np.zeros((1, d))
    np.testing.assert_array_equal(qp.rope(x, zero, style), x)
    quarter = np.full((1, d), math.pi / 2)
    y = qp.rope(x, quarter, style)
    np.testing.assert_allclose(y[..., a], -x[..., b], atol=1e-15)
    np.testing.assert_allclose(y[..., b], x[..., a], atol=1e-15)
    rnd = _rand((1, d), 31) * 10.0
    rnd[:, b] = rnd[:, a]
    y = qp.rope(x, rnd, style)
    np.testing.assert_allclose(y[..., a] ** 2 + y[..., b] ** 2, x[..., a] ** 2 + x[..., b] ** 2,
                               rtol=1e-13)


@pytest.mark.parametrize("style", [qp.ROPE_INTERLEAVED, qp.ROPE_SPLIT])
def test_rope_angles_compose(style):
    x = _rand((1, 3, 2, 16), 32)
    t1, t2 = _rand((3, 16), 33), _rand((3, 16), 34)
    a, b = qp.pairs(16, style)
    for t in (t1, t2):
        t[:, b] = t[:, a]
    np.testing.assert_allclose(qp.rope(qp.rope(x, t1, style), t2, style), qp.rope(x, t1 + t2, style),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("style", [qp.ROPE_INTERLEAVED, qp.ROPE_SPLIT])
def test_rope_scores_depend_on_relative_position_only(style):
    """With theta[p, r] = p * omega_r, <rope_p(q), rope_s(k)> = <rope_{p-s}(q), k>."""
    d = 64
    q = _rand((1, 1, 1, d), 35)
    k = _rand((1, 1, 1, d), 36)
    table = _angles(40, d, style)
    for p, s in [(7, 3), (30, 30), (12, 25)]:
        lhs = float(np.sum(qp.rope(q, table[p:p + 1], style) * qp.rope(k, table[s:s + 1], style)))
        rel = ((p - s) * table[1:2])  # angle of position p - s
        rhs = float(np.sum(qp.rope(q, rel, style) * k))
        assert lhs == pytest.approx(rhs, rel=1e-11, abs=1e-11)


def test_split_half_is_interleaved_on_permuted_features():
    d = 32
    x = _rand((1, 2, 2, d), 37)
    ang_i = _angles(2, d, qp.ROPE_INTERLEAVED, pos0=5)
    # feature permutation taking split-half pairs (r, r + d/2) to (2r, 2r + 1)
    perm = np.empty(d, dtype=int)
    perm[0::2] = np.arange(d // 2)
    perm[1::2] = np.arange(d // 2) + d // 2
    ang_s = np.empty_like(ang_i)
    ang_s[:, perm] = ang_i
    y_split = qp.rope(x, ang_s, qp.ROPE_SPLIT)
    y_int = qp.rope(x[..., perm], ang_i, qp.ROPE_INTERLEAVED)
    np.testing.assert_allclose(y_split[..., perm], y_int, rtol=1e-13, atol=1e-13)


# ----------------------------------------------------------- order, golden

def test_norm_then_rope_order_matters_with_non_uniform_gamma():
    x = _rand((1, 2, 2, 16), 40)
    g = 1.0 + 0.5 * _rand((16,), 41)
    ang = _angles(2, 16, qp.ROPE_SPLIT, pos0=3)
    ours = qp.qk_prologue(x, g, 1e-6, qp.NORM_HEAD, ang, qp.ROPE_SPLIT)
    swapped = qp.rms_norm(qp.rope(x, ang, qp.ROPE_SPLIT), g, 1e-6, qp.NORM_HEAD)
    assert not np.allclose(ours, swapped)
    np.testing.assert_allclose(ours, qp.rope(qp.rms_norm(x, g, 1e-6, qp.NORM_HEAD), ang, qp.ROPE_SPLIT))


def test_golden_fixture():
    with open(os.path.join(GOLDEN, "prologue_d4_head_interleaved.json")) as f:
        g = json.load(f)
    x = np.array(g["x"], dtype=np.float64).reshape(1, 1, 1, 4)
    got = qp.qk_prologue(x, g["gamma"], g["eps"], qp.NORM_HEAD, np.array(g["angles"]).reshape(1, 4),
                         qp.ROPE_INTERLEAVED).ravel()
    np.testing.assert_allclose(got, g["expected"], rtol=0, atol=1e-15)


# ------------------------------------------------------- planted mistakes

def _planted_sign(x, angles, style):
    x = np.asarray(x, dtype=np.float64)
    B, L, H, d = x.shape
    a, b = qp.pairs(d, style)
    th = np.asarray(angles).reshape(L, d)[:, a][None, :, None, :]
    y = x.copy()
    y[..., a] = x[..., a] * np.cos(th) + x[..., b] * np.sin(th)
    y[..., b] = -x[..., a] * np.sin(th) + x[..., b] * np.cos(th)
    return y


def _planted_pairs(d, style):
    r = np.arange(d // 2)
    return 2 * r, 2 * r + 1  # interleaved for every style


def _planted_norm_axis(x, gamma, eps, scope):
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-2, keepdims=True)  # over heads instead of features
    g = 1.0 if gamma is None else np.asarray(gamma, dtype=np.float64)
    return g * x / np.sqrt(ms + eps)


def _planted_no_eps(x, gamma, eps, scope):
    return qp.__dict__["_orig_rms_norm"](x, gamma, 0.0, scope)


PINS = [test_rmsnorm_matches_torch_rms_norm, test_rope_matches_complex_multiplication,
        test_rope_special_angles_and_pair_norms, test_rope_scores_depend_on_relative_position_only,
        test_split_half_is_interleaved_on_permuted_features, test_golden_fixture,
        test_rmsnorm_closed_form_three_four]


def _caught(monkeypatch) -> bool:
    cases = [
        (test_rmsnorm_matches_torch_rms_norm, dict(scope=qp.NORM_HEAD, d=16)),
        (test_rope_matches_complex_multiplication, dict(style=qp.ROPE_SPLIT, d=16)),
        (test_rope_special_angles_and_pair_norms, dict(style=qp.ROPE_SPLIT)),
        (test_rope_scores_depend_on_relative_position_only, dict(style=qp.ROPE_SPLIT)),
        (test_split_half_is_interleaved_on_permuted_features, dict()),
        (test_golden_fixture, dict()),
    ]
    for fn, kw in cases:
        try:
            fn(**kw)
        except AssertionError:
            return True
    return False


@pytest.mark.parametrize("mistake", ["sign", "pairs", "norm_axis", "no_eps"])
def test_planted_mistakes_are_caught(monkeypatch, mistake):
    if mistake == "sign":
        monkeypatch.setattr(qp, "rope", _planted_sign)
    elif mistake == "pairs":
        monkeypatch.setattr(qp, "pairs", _planted_pairs)
    elif mistake == "norm_axis":
        monkeypatch.setattr(qp, "rms_norm", _planted_norm_axis)
    elif mistake == "no_eps":
        monkeypatch.setitem(qp.__dict__, "_orig_rms_norm", qp.rms_norm)
        monkeypatch.setattr(qp, "rms_norm", _planted_no_eps)
    assert _caught(monkeypatch), f"planted mistake '{mistake}' was not caught"
