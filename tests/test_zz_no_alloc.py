"""attn_fwd_splitkv_static: the key-split forward for callers that cannot
allocate device memory (a framework plugin handed only its input and output
buffers, or a step loop that must not call cudaMalloc because it can
synchronize the device). Its float32 partials live in a fixed 64 MB array
inside the library instead of a caller workspace, so the call allocates
nothing. These tests call it through the C ABI and compare it with the
workspace entry point attn_fwd_splitkv (same kernels, so bitwise equal) and
with the FP64 oracle, on calls in a row, and check its size limit.

This file is collected last, so a run that stops at the first failure has
already run every other test; it passes alone in a fresh process too (the
first call, which loads the library's module and looks up the array's
address, comes before any memory reading).
"""

from __future__ import annotations

import math

import pytest
import torch

import head_attention_streaming_b200 as hasb
import oracle
from head_attention_streaming_b200 import binding, inputs

SCRATCH_BYTES = 64 << 20


def test_symbol_is_exported():
    assert hasattr(binding.lib(), "attn_fwd_splitkv_static")


def test_invalid_call_is_refused_before_any_cuda_call():
    A = 1 << 20
    used = binding.ctypes.c_int(-7)
    # a negative split count
    st = binding.lib().attn_fwd_splitkv_static(A, A + 0x100000, A + 0x200000, A + 0x300000, None, -2, 1,
                                               64, 512, 2, 1, 128, 0.1, 1, 0, 0,
                                               binding.ctypes.byref(used), None)
    assert st == hasb.ATTN_ERR_INVALID_ARG and used.value == -7


def _f64(t):
    return t.cpu().to(torch.float64).numpy()


def _against_oracle(o, lse, q, k, v, scale, mask, off):
    o_ref, lse_ref = oracle.attention_fwd(_f64(q), _f64(k), _f64(v), scale, mask, off)
    err = abs(_f64(o) - o_ref)
    assert err.max() <= 8e-3 and err.mean() <= 2e-4
    assert abs(_f64(lse) - lse_ref).max() <= 1e-3


@pytest.mark.gpu
def test_two_calls_in_a_row_match_the_workspace_path_and_allocate_nothing(cuda_ok):
    """Two static calls on different inputs, each equal bit for bit to
    attn_fwd_splitkv with the same split count (a stale partial from the first
    call would show in the second) and within the BF16 bars of the oracle. The
    outputs are preallocated, so the second call must leave device memory
    exactly as it was: neither torch's pool nor the driver's free memory moves."""
    torch.cuda.set_device(0)
    w = inputs.WORKLOADS["stream_chunk_256_vs_7140_gqa40x8"]
    runs = []
    for seed in (w.seed, w.seed + 100):
        q, k, v = (t.cuda() for t in inputs.make_qkv(w.B, w.Lq, w.Lk, w.Hq, w.Hkv, w.d, w.torch_dtype,
                                                     seed=seed))
        runs.append((q, k, v, torch.empty_like(q),
                     torch.empty(w.B, w.Hq, w.Lq, dtype=torch.float32, device="cuda")))
    torch.cuda.synchronize()
    for i, (q, k, v, o, lse) in enumerate(runs):
        if i == 1:
            free0, reserved0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_reserved()
        _, _, used = hasb.attn_fwd_splitkv_static(q, k, v, scale=w.scale, causal=w.mask, kv_offset=w.kv_offset,
                                                  out=o, lse=lse)
        torch.cuda.synchronize()
        if i == 1:
            assert torch.cuda.memory_reserved() == reserved0
            assert abs(torch.cuda.mem_get_info()[0] - free0) <= (2 << 20)
        assert used > 1
        o2, l2, used2 = hasb.attn_fwd_splitkv(q, k, v, n_splits=used, scale=w.scale, causal=w.mask,
                                              kv_offset=w.kv_offset)
        torch.cuda.synchronize()
        assert used2 == used and torch.equal(o, o2) and torch.equal(lse, l2)
        _against_oracle(o, lse, q, k, v, w.scale, w.mask, w.kv_offset)
    assert hasb.device_fault(clear=True) == 0


@pytest.mark.gpu
def test_static_scratch_causal(cuda_ok):
    """The causal key split through the static scratch equals the workspace
    path bitwise and the oracle within the bars."""
    torch.cuda.set_device(0)
    q, k, v = (t.cuda() for t in inputs.make_qkv(1, 600, 2000, 4, 2, 128, torch.bfloat16, seed=31))
    o1, l1, used = hasb.attn_fwd_splitkv_static(q, k, v, n_splits=4, causal=hasb.MASK_CAUSAL, kv_offset=1400)
    o2, l2, used2 = hasb.attn_fwd_splitkv(q, k, v, n_splits=4, causal=hasb.MASK_CAUSAL, kv_offset=1400)
    torch.cuda.synchronize()
    assert used == used2 == 4 and torch.equal(o1, o2) and torch.equal(l1, l2)
    _against_oracle(o1, l1, q, k, v, 1.0 / math.sqrt(128), 1, 1400)
    assert hasb.device_fault(clear=True) == 0


@pytest.mark.gpu
def test_automatic_count_is_lowered_to_fit_the_scratch(cuda_ok):
    """512 query rows x 40 heads over 4096 keys: the automatic choice wants more
    key ranges than 64 MB of partials hold (10.6 MB a range), so the count is
    lowered to the largest that fits (6), and the result equals the workspace
    path with that count bit for bit."""
    torch.cuda.set_device(0)
    B, Lq, Lk, Hq, Hkv, d = 1, 512, 4096, 40, 8, 128
    q, k, v = (t.cuda() for t in inputs.make_qkv(B, Lq, Lk, Hq, Hkv, d, torch.bfloat16, seed=41))
    o1, l1, used = hasb.attn_fwd_splitkv_static(q, k, v)
    torch.cuda.synchronize()
    assert hasb.splitkv_workspace_bytes(B, Lq, Hq, d, used) <= SCRATCH_BYTES
    assert hasb.splitkv_workspace_bytes(B, Lq, Hq, d, used + 1) > SCRATCH_BYTES
    assert used == 6
    o2, l2, used2 = hasb.attn_fwd_splitkv(q, k, v, n_splits=used)
    torch.cuda.synchronize()
    assert used2 == used and torch.equal(o1, o2) and torch.equal(l1, l2)
    assert hasb.device_fault(clear=True) == 0


@pytest.mark.gpu
def test_explicit_count_beyond_the_scratch_is_refused(cuda_ok):
    """One 1785-row, 40-head range needs 36.8 MB of partials, so two ranges
    (73.7 MB) exceed the 64 MB array: an explicit request for them is refused
    with ATTN_ERR_SCRATCH_LIMIT and the output is left untouched; the automatic
    count falls back to one range (attn_fwd)."""
    torch.cuda.set_device(0)
    w = inputs.WORKLOADS["stream_chunk_1785_vs_7140_gqa40x8"]
    assert hasb.splitkv_workspace_bytes(w.B, w.Lq, w.Hq, w.d, 2) > SCRATCH_BYTES
    q, k, v = (t.cuda() for t in inputs.workload_inputs(w))
    out = torch.full_like(q, 7.0)
    with pytest.raises(hasb.AttnError) as e:
        hasb.attn_fwd_splitkv_static(q, k, v, n_splits=2, scale=w.scale, causal=w.mask,
                                     kv_offset=w.kv_offset, out=out)
    assert e.value.status == hasb.ATTN_ERR_SCRATCH_LIMIT
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())
    o1, l1, used = hasb.attn_fwd_splitkv_static(q, k, v, scale=w.scale, causal=w.mask, kv_offset=w.kv_offset)
    o2, l2 = hasb.attn_fwd(q, k, v, scale=w.scale, causal=w.mask, kv_offset=w.kv_offset)
    torch.cuda.synchronize()
    assert used == 1 and torch.equal(o1, o2) and torch.equal(l1, l2)
    assert hasb.device_fault(clear=True) == 0
