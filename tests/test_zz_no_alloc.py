"""attn_fwd_splitkv_static: the key-split forward with the library's own
scratch (a file-scope device array) instead of a caller workspace; the call
allocates nothing. Checked against the FP64 oracle and against the workspace
entry point with the same split count (same kernels, bitwise equal)."""

from __future__ import annotations

import math

import pytest
import torch

import head_attention_streaming_b200 as hasb
import oracle
from head_attention_streaming_b200 import binding, inputs


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


@pytest.mark.gpu
def test_static_scratch_matches_oracle_and_workspace_path(cuda_ok):
    torch.cuda.set_device(0)
    w = inputs.WORKLOADS["stream_chunk_256_vs_7140_gqa40x8"]
    q, k, v = (t.cuda() for t in inputs.make_qkv(w.B, w.Lq, w.Lk, w.Hq, w.Hkv, w.d, w.torch_dtype,
                                                 seed=w.seed))
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    o1, l1, used = hasb.attn_fwd_splitkv_static(q, k, v, scale=w.scale, causal=w.mask,
                                                kv_offset=w.kv_offset)
    torch.cuda.synchronize()
    assert used > 1
    # nothing but the two outputs was allocated (by torch, here); the library call itself none
    out_bytes = o1.numel() * o1.element_size() + l1.numel() * 4
    assert torch.cuda.mem_get_info()[0] >= free0 - out_bytes - (4 << 20)
    o2, l2, used2 = hasb.attn_fwd_splitkv(q, k, v, n_splits=used, scale=w.scale, causal=w.mask,
                                          kv_offset=w.kv_offset)
    torch.cuda.synchronize()
    assert used2 == used and torch.equal(o1, o2) and torch.equal(l1, l2)
    f64 = lambda t: t.cpu().to(torch.float64).numpy()
    o_ref, lse_ref = oracle.attention_fwd(f64(q), f64(k), f64(v), w.scale, w.mask, w.kv_offset)
    err = abs(f64(o1) - o_ref)
    assert err.max() <= 8e-3 and err.mean() <= 2e-4
    assert abs(f64(l1) - lse_ref).max() <= 1e-3
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
    f64 = lambda t: t.cpu().to(torch.float64).numpy()
    o_ref, lse_ref = oracle.attention_fwd(f64(q), f64(k), f64(v), 1.0 / math.sqrt(128), 1, 1400)
    err = abs(f64(o1) - o_ref)
    assert err.max() <= 8e-3 and err.mean() <= 2e-4
    assert abs(f64(l1) - lse_ref).max() <= 1e-3
    assert hasb.device_fault(clear=True) == 0
