"""Parity of the CUDA path (through the C ABI) with the FP64 oracle, on a B200.

Tolerances (the target's stated bar): O max-abs 8e-3 and mean-abs 2e-4 for
BF16, half of both for FP16; LSE abs 1e-3. Shapes other than the five
workloads add the oracle's bounds on the path's two 16-bit rounding steps (P
before P V, and O itself) to the O bars (see _check). Inputs are the seeded workloads of
head_attention_streaming_b200.inputs plus a grid of small shapes that span
several tiles, ragged tails, GQA/MQA ratios and every mask mode.
"""

import math

import numpy as np
import pytest
import torch

import head_attention_streaming_b200 as hasb
import oracle
from head_attention_streaming_b200 import inputs
from oracle.rounding import half_ulp16, p16_rounding_bound

pytestmark = pytest.mark.gpu

TOL = {"bf16": (8e-3, 2e-4), "fp16": (4e-3, 1e-4)}
LSE_TOL = 1e-3


@pytest.fixture(scope="module", autouse=True)
def _device(cuda_ok):
    torch.cuda.set_device(0)
    hasb.set_wait_timeout_ns(4_000_000_000)
    yield
    assert hasb.device_fault(clear=True) == 0


def _gpu(q, k, v, scale, mask, off):
    o, lse = hasb.attn_fwd(q.cuda(), k.cuda(), v.cuda(), scale=scale, causal=mask, kv_offset=off)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu()


def _f64(t):
    return t.to(torch.float64).numpy()


def _pbound(q, k, v, scale, dtype, mask=0, off=0, rows=None, window=(-1, -1)):
    """The oracle's bound on the O error from rounding P to the 16-bit type
    before P V (oracle.rounding.p16_rounding_bound), for the same inputs."""
    t64 = lambda t: t.to(torch.float64).numpy() if isinstance(t, torch.Tensor) else np.asarray(t)
    return p16_rounding_bound(t64(q), t64(k), t64(v), scale, dtype, mask, off, rows=rows, window=window)


def _check(o_gpu, lse_gpu, o_ref, lse_ref, dtype, what="", p_bound=None):
    """Compare with the oracle.

    The five workloads use the stated bars as they are. Other shapes (ragged
    tails, one visible key, peaked scores) can have |O| near 1, where the two
    16-bit rounding steps of the path alone exceed those absolute bars; there
    the caller passes ``p_bound``, the oracle's per-element bound on rounding
    P to 16 bits (oracle/rounding.py), and each bar grows by exactly the two
    rounding terms: elementwise
        |err| <= bar + half_ulp16(max(|O_ref|, |O|)) + p_bound,
    the final rounding of O moving it by at most half a spacing; and the mean,
    summed term by term, <= mean bar + mean(half ulp) + mean(p_bound).
    """
    max_tol, mean_tol = TOL[dtype]
    o = _f64(o_gpu)
    err = np.abs(o - o_ref)
    lerr = np.abs(lse_gpu.to(torch.float64).numpy() - lse_ref)
    assert np.isfinite(o).all(), what
    if p_bound is not None:
        h = half_ulp16(np.maximum(np.abs(o_ref), np.abs(o)), dtype)
        excess = err - (max_tol + h + p_bound)
        assert excess.max() <= 0, f"{what} O error above bar + rounding terms by {excess.max():.3g}"
        mean_bar = mean_tol + h.mean() + p_bound.mean()
        assert err.mean() <= mean_bar, f"{what} O mean-abs {err.mean():.3g} > {mean_bar:.3g}"
    else:
        assert err.max() <= max_tol, f"{what} O max-abs {err.max():.3g}"
        assert err.mean() <= mean_tol, f"{what} O mean-abs {err.mean():.3g}"
    assert lerr.max() <= LSE_TOL, f"{what} LSE max-abs {lerr.max():.3g}"


# ------------------------------------------------------------- building blocks

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_selftest_mma_tile(dtype):
    g = torch.Generator().manual_seed(11)
    q = torch.randn(128, 128, generator=g).to(dtype)
    k = torch.randn(128, 128, generator=g).to(dtype)
    v = torch.randn(128, 128, generator=g).to(dtype)
    s, o = hasb.selftest_mma(q.cuda(), k.cuda(), v.cuda())
    s, o = s.cpu().double(), o.cpu().double()
    s_ref = q.double() @ k.double().T
    assert (s - s_ref).abs().max() <= 1e-3 * s_ref.abs().max()
    p = (s.float() * 0.0625).to(dtype).double()     # the same rounding the kernel applies
    o_ref = p @ v.double()
    assert (o - o_ref).abs().max() <= 1e-4 * o_ref.abs().max() + 1e-5


def test_fma_pipe_exp2_within_its_error_bound():
    # the polynomial exponential that replaces part of the MUFU ex2 calls
    x = torch.cat([torch.linspace(-125.0, 8.0, 1_000_003), torch.tensor([0.0, 0.5, -0.5, 8.0, -125.0])])
    y = hasb.selftest_exp2(x.cuda().contiguous()).cpu().double()
    ref = torch.exp2(x.double())
    rel = ((y - ref) / ref).abs()
    assert float(rel.max()) <= 7.6e-5, float(rel.max())
    below = hasb.selftest_exp2(torch.tensor([-126.0, -400.0, float("-inf")], device="cuda")).cpu()
    assert torch.all(below >= 0) and torch.all(below < 2.0 ** -124)


def test_bounded_wait_gives_up_and_reports():
    st = hasb.selftest_wait_timeout(50_000_000)
    assert st == hasb.ATTN_ERR_TIMEOUT
    assert hasb.device_fault(clear=True) == 0      # the self-test cleared its bit
    # the context is still usable
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0


# -------------------------------------------------------------- small shapes

SMALL = [
    # B, Lq, Lk, Hq, Hkv, d, dtype, mask, kv_offset
    (1, 1, 1, 1, 1, 128, "bf16", 0, 0),
    (1, 1, 1000, 8, 1, 128, "bf16", 0, 0),
    (2, 129, 257, 4, 2, 128, "bf16", 0, 0),
    (2, 256, 256, 2, 2, 64, "bf16", 0, 0),
    (1, 300, 300, 2, 1, 64, "fp16", 1, 0),
    (2, 384, 384, 2, 2, 128, "bf16", 1, 0),
    (1, 77, 500, 4, 4, 128, "bf16", 1, 423),
    (1, 200, 700, 8, 2, 128, "bf16", 2, 300),
    (1, 513, 1000, 3, 1, 128, "fp16", 2, 487),
    (1, 130, 130, 2, 2, 64, "fp16", 2, 0),
    (3, 17, 33, 6, 3, 64, "bf16", 1, 16),
]


@pytest.mark.parametrize("B,Lq,Lk,Hq,Hkv,d,dtype,mask,off", SMALL)
def test_parity_small(B, Lq, Lk, Hq, Hkv, d, dtype, mask, off):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float16
    q, k, v = inputs.make_qkv(B, Lq, Lk, Hq, Hkv, d, tdt, seed=100 + Lq + Lk + d)
    scale = 1.0 / math.sqrt(d)
    o, lse = _gpu(q, k, v, scale, mask, off)
    o_ref, lse_ref = oracle.attention_fwd(_f64(q), _f64(k), _f64(v), scale, mask, off)
    _check(o, lse, o_ref, lse_ref, dtype, f"{B},{Lq},{Lk},{Hq},{Hkv},{d},{dtype},{mask},{off}",
           p_bound=_pbound(q, k, v, scale, dtype, mask, off))


def test_large_scores_trigger_rescaling():
    # scores spread over hundreds of log2 units: the lazy rescale must fire
    q, k, v = inputs.make_qkv(1, 256, 1024, 2, 2, 128, torch.bfloat16, seed=77)
    ramp = torch.linspace(0.1, 8.0, 1024).view(1, 1024, 1, 1)
    k = (k.float() * ramp).to(torch.bfloat16)
    o, lse = _gpu(q, k, v, 1.0 / math.sqrt(128), 0, 0)
    o_ref, lse_ref = oracle.attention_fwd(_f64(q), _f64(k), _f64(v), 1.0 / math.sqrt(128))
    _check(o, lse, o_ref, lse_ref, "bf16", "rescale",
           p_bound=_pbound(q, k, v, 1.0 / math.sqrt(128), "bf16"))


# ----------------------------------------------------------------- workloads

@pytest.mark.parametrize("name", [n for n in inputs.WORKLOAD_ORDER
                                  if inputs.WORKLOADS[n].sample_rows == 0])
def test_parity_workload(name):
    w = inputs.WORKLOADS[name]
    q, k, v = inputs.workload_inputs(w)
    o, lse = _gpu(q, k, v, w.scale, w.mask, w.kv_offset)
    o_ref, lse_ref = oracle.attention_fwd(_f64(q), _f64(k), _f64(v), w.scale, w.mask, w.kv_offset)
    _check(o, lse, o_ref, lse_ref, w.dtype, name)


@pytest.fixture(scope="module")
def video():
    w = inputs.WORKLOADS["video_20480x56x128"]
    q, k, v = inputs.workload_inputs(w)
    return w, q, k, v


def test_parity_video_sampled_rows(video):
    w, q, k, v = video
    o, lse = _gpu(q, k, v, w.scale, w.mask, w.kv_offset)
    errs, lerrs = [], []
    for h in range(w.Hq):
        rows = inputs.sample_rows(w.Lq, w.sample_rows, seed=w.seed * 1000 + h)
        o_ref, lse_ref = oracle.attention_fwd(_f64(q[:, :, h:h + 1]), _f64(k[:, :, h:h + 1]),
                                              _f64(v[:, :, h:h + 1]), w.scale, rows=rows)
        errs.append(np.abs(_f64(o[:, rows, h:h + 1]) - o_ref))
        lerrs.append(np.abs(lse[:, h:h + 1, rows].double().numpy() - lse_ref))
    err = np.concatenate([e.ravel() for e in errs])
    lerr = np.concatenate([e.ravel() for e in lerrs])
    assert err.max() <= TOL["bf16"][0], err.max()
    assert err.mean() <= TOL["bf16"][1], err.mean()
    assert lerr.max() <= LSE_TOL, lerr.max()


def test_video_zero_scale_closed_form_every_row(video):
    # scale 0: every key has weight 1/Lk, so each row is the mean of V and LSE = ln Lk
    w, q, k, v = video
    o, lse = _gpu(q, k, v, 0.0, 0, 0)
    mean_v = v.double().mean(dim=1, keepdim=True)          # [1, 1, H, d]
    err = (o.double() - mean_v).abs()
    assert err.max() <= 2e-3, float(err.max())             # bf16 rounding of |mean| < 0.05
    assert (lse.double() - math.log(w.Lk)).abs().max() <= 1e-4


@pytest.mark.parametrize("mask,off", [(1, 133), (2, 100), (1, 0)])
def test_zero_scale_masked_closed_form(mask, off):
    # scale 0 with a mask: row i is the mean of its visible V rows, LSE = ln(count);
    # exercises partial tiles where masked scores meet a zero scale
    Lq, Lk = 200, 333
    q, k, v = inputs.make_qkv(1, Lq, Lk, 2, 1, 128, torch.bfloat16, seed=21)
    o, lse = _gpu(q, k, v, 0.0, mask, off)
    vd = v.double()
    for i in range(Lq):
        n = min(Lk, off + i + 1) if mask == 1 else off + Lq
        ref = vd[0, :n, 0].mean(dim=0)
        assert (o[0, i].double() - ref).abs().max() <= 8e-3, (i, n)
        assert abs(float(lse[0, 0, i]) - math.log(n)) <= 1e-4


# ---------------------------------------------------------------- invariants

def test_deterministic_bitwise():
    w = inputs.WORKLOADS["dit_selfattn_1785x40x128_qknorm"]
    q, k, v = (t.cuda() for t in inputs.workload_inputs(w))
    o1, l1 = hasb.attn_fwd(q, k, v, scale=w.scale)
    o2, l2 = hasb.attn_fwd(q, k, v, scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("mask,off", [(2, 300), (1, 300)])
def test_invisible_keys_have_no_effect(mask, off):
    q, k, v = inputs.make_qkv(1, 200, 1000, 4, 2, 128, torch.bfloat16, seed=5)
    o1, l1 = _gpu(q, k, v, 0.088, mask, off)
    k2, v2 = k.clone(), v.clone()
    k2[:, off + 200:] = 30.0
    v2[:, off + 200:] = -1000.0
    o2, l2 = _gpu(q, k2, v2, 0.088, mask, off)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_gqa_equals_replicated_heads():
    q, k, v = inputs.make_qkv(1, 300, 400, 8, 2, 128, torch.bfloat16, seed=9)
    o1, l1 = _gpu(q, k, v, 0.09, 0, 0)
    o2, l2 = _gpu(q, k.repeat_interleave(4, dim=2).contiguous(),
                  v.repeat_interleave(4, dim=2).contiguous(), 0.09, 0, 0)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_lse_optional_and_output_buffer_reused():
    q, k, v = (t.cuda() for t in inputs.make_qkv(1, 300, 300, 2, 2, 64, torch.float16, seed=3))
    out = torch.full_like(q, float("nan"))
    o, lse = hasb.attn_fwd(q, k, v, out=out, return_lse=False)
    torch.cuda.synchronize()
    assert lse is None and o.data_ptr() == out.data_ptr() and torch.isfinite(o).all()


def test_invalid_call_on_device_raises_without_launch():
    q = torch.zeros(1, 4, 3, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 4, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(hasb.AttnError) as e:
        hasb.attn_fwd(q, k, k)                      # Hq % Hkv != 0
    assert e.value.status == hasb.ATTN_ERR_INVALID_ARG
