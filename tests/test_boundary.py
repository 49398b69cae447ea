"""C-ABI boundary checks that need no GPU.

The library must load on a machine without a device, export every function
include/attn.h declares, and reject every invalid argument with the right
status before making any CUDA call (so these calls are safe anywhere: nothing
is launched). The pages' strict-backend convention (FlashAttention-4 runtime
page, "FLASH4.md": a violated contract raises an error instead of changing
kernels) is what the status codes implement.
"""

import ctypes
import os
import re

import pytest

import head_attention_streaming_b200 as hasb
from head_attention_streaming_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")

A = 0x10000  # 16-byte aligned fake addresses: never dereferenced (calls fail validation first)


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|const char\*|size_t)\s+(attn_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    assert "attn_fwd" in names and "attn_status_string" in names
    assert len(names) >= 6


def test_library_loads_and_exports_every_declared_symbol():
    L = hasb.lib()
    for name in _declared_functions():
        assert hasattr(L, name), name
    assert set(_declared_functions()) == set(binding._SIGNATURES)


def test_status_strings():
    for st in range(6):
        assert hasb.status_string(st) != "unknown status"
    assert hasb.status_string(99) == "unknown status"


def _call(**kw):
    args = dict(q=A, k=A + 0x100000, v=A + 0x200000, o=A + 0x300000, lse=None, B=1, Lq=4, Lk=4,
                Hq=2, Hkv=1, d=128, scale=0.125, causal=0, kv_offset=0, dtype=0)
    args.update(kw)
    L = hasb.lib()
    return L.attn_fwd(args["q"], args["k"], args["v"], args["o"], args["lse"], args["B"], args["Lq"],
                      args["Lk"], args["Hq"], args["Hkv"], args["d"], args["scale"], args["causal"],
                      args["kv_offset"], args["dtype"], None)


INVALID = [
    dict(q=None), dict(k=None), dict(v=None), dict(o=None),
    dict(B=0), dict(Lq=0), dict(Lk=0), dict(Hq=0), dict(Hkv=0), dict(Hq=3, Hkv=2),
    dict(d=0), dict(d=96), dict(d=8), dict(d=512),
    dict(scale=float("nan")), dict(scale=float("inf")), dict(scale=-0.5),
    dict(dtype=2), dict(dtype=-1), dict(causal=3), dict(causal=-1),
    dict(kv_offset=1),                              # mask none takes no offset
    dict(causal=1, kv_offset=-1), dict(causal=1, Lq=4, Lk=4, kv_offset=1),
    dict(causal=2, Lq=3, Lk=10, kv_offset=8),       # chunk end past the cache
    dict(q=A + 8), dict(k=A + 0x100000 + 4), dict(o=A + 0x300000 + 2),
    dict(lse=A + 0x400000 + 2),
    dict(o=A),                                      # output overlaps q
    dict(o=A + 0x100000 + 64),                      # output overlaps k
    dict(B=1 << 16, Lq=1 << 16, Hq=1 << 10, Hkv=1 << 10),   # size overflow
]


@pytest.mark.parametrize("kw", INVALID, ids=[str(k) for k in INVALID])
def test_invalid_arguments_are_rejected_before_any_launch(kw):
    assert _call(**kw) == hasb.ATTN_ERR_INVALID_ARG


def test_head_dims_outside_the_pages_range_are_invalid():
    for d in (8, 48, 512):
        assert _call(d=d) == hasb.ATTN_ERR_INVALID_ARG


def test_python_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 4, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        hasb.attn_fwd(q, q, q)


def test_device_fault_null_pointer():
    assert hasb.lib().attn_device_fault(None, 0) == hasb.ATTN_ERR_INVALID_ARG


def test_selftest_timeout_rejects_out_of_range_limits():
    assert hasb.lib().attn_selftest_wait_timeout(10, None) == hasb.ATTN_ERR_INVALID_ARG
    assert hasb.lib().attn_selftest_wait_timeout(10**11, None) == hasb.ATTN_ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_LIB", None)
    monkeypatch.setattr(binding, "_SO_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="missing"):
        binding.lib()


# ----------------------------------------------------------- Q/K prologue

def _pro(**kw):
    args = dict(q=A, q_out=A + 0x100000, k=A + 0x200000, k_out=A + 0x300000, gq=None, gk=None,
                aq=A + 0x400000, ak=A + 0x500000, B=1, Lq=4, Lk=4, Hq=2, Hkv=1, d=64,
                scope=1, eps=1e-6, style=2, dtype=0)
    args.update(kw)
    return hasb.lib().attn_qk_prologue(args["q"], args["q_out"], args["k"], args["k_out"], args["gq"],
                                       args["gk"], args["aq"], args["ak"], args["B"], args["Lq"],
                                       args["Lk"], args["Hq"], args["Hkv"], args["d"], args["scope"],
                                       args["eps"], args["style"], args["dtype"], None)


PRO_INVALID = [
    dict(q=None), dict(q_out=None), dict(k_out=None), dict(k=None),   # k and k_out both or neither
    dict(B=0), dict(Lq=0), dict(Lk=0), dict(Hq=0), dict(Hkv=0),
    dict(scope=3), dict(scope=-1), dict(style=3), dict(style=-1),
    dict(eps=-1e-6), dict(eps=float("nan")), dict(eps=float("inf")), dict(dtype=2),
    dict(aq=None), dict(ak=None),                 # RoPE requested without angles
    dict(style=0),                                # angles given without RoPE
    dict(q=A + 8), dict(k_out=A + 0x300000 + 4), dict(gq=A + 0x600000 + 2), dict(aq=A + 0x400000 + 1),
    dict(q_out=A + 64),                           # partial overlap of q_out and q
    dict(k_out=A + 0x100000),                     # k_out overlaps q_out
    dict(q_out=A + 0x200000),                     # q_out overlaps k
]


@pytest.mark.parametrize("kw", PRO_INVALID, ids=[str(k) for k in PRO_INVALID])
def test_prologue_invalid_arguments_are_rejected_before_any_launch(kw):
    assert _pro(**kw) == hasb.ATTN_ERR_INVALID_ARG


@pytest.mark.parametrize("d", [8, 24, 96, 512])
def test_prologue_head_dims_outside_16_to_256_powers_of_two_are_unsupported(d):
    assert _pro(d=d) == hasb.ATTN_ERR_UNSUPPORTED


def test_prologue_python_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 4, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        hasb.qk_prologue(q)


def test_splitkv_argument_contract_before_any_cuda_call():
    L = hasb.lib()
    base = [A, A + 0x100000, A + 0x200000, A + 0x300000, None, A + 0x400000, 1 << 20]
    tail = [1, 64, 512, 2, 1, 128, 0.1]
    # a negative split count is refused; a misaligned workspace is refused; a
    # causal offset past Lk - Lq is refused like attn_fwd's
    assert L.attn_fwd_splitkv(*base, -1, *tail, 0, 0, 0, None, None) == hasb.ATTN_ERR_INVALID_ARG
    assert L.attn_fwd_splitkv(*base, 2, *tail, 1, 500, 0, None, None) == hasb.ATTN_ERR_INVALID_ARG
    bad = list(base)
    bad[5] = A + 0x400000 + 4
    assert L.attn_fwd_splitkv(*bad, 2, *tail, 0, 0, 0, None, None) == hasb.ATTN_ERR_INVALID_ARG
    assert L.attn_splitkv_workspace_bytes(1, 64, 2, 128, 4) == 4 * 1 * 2 * 64 * 129 * 4
    assert L.attn_splitkv_workspace_bytes(0, 64, 2, 128, 4) == 0


@pytest.mark.parametrize("kw", [dict(wl=-2), dict(wr=-3), dict(off=-1), dict(off=5), dict(Lq=0)])
def test_window_argument_contract(kw):
    a = dict(wl=4, wr=0, off=0, Lq=4)
    a.update(kw)
    st = hasb.lib().attn_fwd_window(A, A + 0x100000, A + 0x200000, A + 0x300000, None, 1, a["Lq"], 8, 2,
                                    1, 128, 0.1, a["wl"], a["wr"], a["off"], 0, None)
    assert st == hasb.ATTN_ERR_INVALID_ARG


def _fp8_args(**kw):
    a = dict(q=A, k=A + 0x100000, vt=A + 0x200000, o=A + 0x300000, lse=None, B=1, Lq=64, Lk=256,
             pitch=256, Hq=2, Hkv=1, d=128, scale=0.1, mask=0, off=0)
    a.update(kw)
    return [a[n] for n in ("q", "k", "vt", "o", "lse", "B", "Lq", "Lk", "pitch", "Hq", "Hkv", "d",
                           "scale", "mask", "off")] + [None]


@pytest.mark.parametrize("kw", [dict(pitch=255), dict(pitch=240), dict(q=A + 8), dict(vt=A + 4),
                                dict(Hq=3, Hkv=2), dict(mask=3), dict(mask=0, off=1),
                                dict(mask=2, off=250), dict(scale=-1.0), dict(Lk=0),
                                dict(o=A + 0x100000 + 64)])
def test_fp8_attention_argument_contract(kw):
    assert hasb.lib().attn_fwd_fp8(*_fp8_args(**kw)) == hasb.ATTN_ERR_INVALID_ARG


def test_fp8_attention_head_dim_512_is_invalid():
    assert hasb.lib().attn_fwd_fp8(*_fp8_args(d=512)) == hasb.ATTN_ERR_INVALID_ARG


def test_fp8_cast_argument_contract():
    L = hasb.lib()
    assert L.attn_fp8_cast(A, A + 0x100000, 12, 0, None) == hasb.ATTN_ERR_INVALID_ARG   # n % 8
    assert L.attn_fp8_cast(A + 8, A + 0x100000, 16, 0, None) == hasb.ATTN_ERR_INVALID_ARG  # x alignment
    assert L.attn_fp8_cast(A, A + 0x100004, 16, 0, None) == hasb.ATTN_ERR_INVALID_ARG   # y alignment
    assert L.attn_fp8_cast(A, A + 16, 16, 0, None) == hasb.ATTN_ERR_INVALID_ARG         # overlap
    assert L.attn_fp8_cast(A, A + 0x100000, 16, 2, None) == hasb.ATTN_ERR_INVALID_ARG   # dtype
    assert L.attn_fp8_cast(A, A + 0x100000, 0, 0, None) == hasb.ATTN_OK                 # empty: no launch
    vt = [A, A + 0x100000]
    assert L.attn_fp8_cast_vt(*vt, 1, 100, 1, 128, 96, 0, None) == hasb.ATTN_ERR_INVALID_ARG  # pitch < Lk
    assert L.attn_fp8_cast_vt(*vt, 1, 100, 1, 128, 120, 0, None) == hasb.ATTN_ERR_INVALID_ARG  # pitch % 16
    assert L.attn_fp8_cast_vt(*vt, 1, 100, 1, 96, 112, 0, None) == hasb.ATTN_ERR_INVALID_ARG   # d not 2^k
    assert L.attn_fp8_cast_vt(*vt, 1, 100, 1, 8, 112, 0, None) == hasb.ATTN_ERR_INVALID_ARG    # d < 16
    assert L.attn_fp8_cast_vt(A, A + 0x100, 1, 100, 1, 128, 112, 0, None) == hasb.ATTN_ERR_INVALID_ARG


def test_fp8_binding_rejects_cpu_and_wrong_types():
    import torch
    q = torch.zeros(1, 4, 2, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        hasb.fp8_cast(q)
    with pytest.raises(ValueError):
        hasb.attn_fwd_fp8(q, q, q)


def _fp8s_args(**kw):
    a = dict(q=A, k=A + 0x100000, vt=A + 0x200000, sq=A + 0x500000, sk=A + 0x600000, sv=A + 0x700000,
             o=A + 0x300000, lse=None, B=1, Lq=64, Lk=256, pitch=256, sqp=64, skp=256, Hq=2, Hkv=1,
             d=128, scale=0.1, mask=0, off=0)
    a.update(kw)
    return [a[n] for n in ("q", "k", "vt", "sq", "sk", "sv", "o", "lse", "B", "Lq", "Lk", "pitch", "sqp",
                           "skp", "Hq", "Hkv", "d", "scale", "mask", "off")] + [None]


@pytest.mark.parametrize("kw", [dict(sq=None), dict(sk=None), dict(skp=255), dict(skp=250),
                                dict(sqp=63), dict(sk=A + 0x600004), dict(sv=A + 0x700004),
                                dict(sq=A + 0x500002), dict(o=A + 0x600000)])
def test_fp8_scaled_attention_argument_contract(kw):
    assert hasb.lib().attn_fwd_fp8_scaled(*_fp8s_args(**kw)) == hasb.ATTN_ERR_INVALID_ARG


def test_fp8_scaled_attention_head_dim_512_is_invalid():
    assert hasb.lib().attn_fwd_fp8_scaled(*_fp8s_args(d=512)) == hasb.ATTN_ERR_INVALID_ARG


def test_fp8_quantize_argument_contract():
    L = hasb.lib()
    x, y, s = A, A + 0x100000, A + 0x200000
    assert L.attn_fp8_quantize_tokens(x, y, s, 1, 10, 2, 24, 10, 0, None) == hasb.ATTN_ERR_INVALID_ARG  # d
    assert L.attn_fp8_quantize_tokens(x, y, s, 1, 10, 2, 128, 9, 0, None) == hasb.ATTN_ERR_INVALID_ARG  # pitch
    assert L.attn_fp8_quantize_tokens(x, y, None, 1, 10, 2, 128, 10, 0, None) == hasb.ATTN_ERR_INVALID_ARG
    assert L.attn_fp8_quantize_tokens(x, x + 64, s, 1, 10, 2, 128, 10, 0, None) == hasb.ATTN_ERR_INVALID_ARG
    assert L.attn_fp8_quantize_tokens(x, y, s, 1, 10, 2, 128, 10, 5, None) == hasb.ATTN_ERR_INVALID_ARG  # dtype
    assert L.attn_fp8_quantize_vt(x, y, s, 1, 100, 1, 48, 112, 0, None) == hasb.ATTN_ERR_INVALID_ARG     # d
    assert L.attn_fp8_quantize_vt(x, y, None, 1, 100, 1, 128, 112, 0, None) == hasb.ATTN_ERR_INVALID_ARG
    assert L.attn_fp8_quantize_vt(x, y, s, 1, 100, 1, 128, 104, 0, None) == hasb.ATTN_ERR_INVALID_ARG    # pitch


def test_rope_after_cache_argument_contract():
    L = hasb.lib()
    args = dict(q=A, qo=A + 0x100000, kc=A + 0x200000, kr=A + 0x300000, ang=A + 0x400000, R=300, q0=260,
                rows=None, B=1, Lq=40, Lk=250, S=300, Hq=2, Hkv=1, d=64, style=2, dtype=0)

    def call(**kw):
        a = dict(args)
        a.update(kw)
        return L.attn_rope_after_cache(*[a[n] for n in ("q", "qo", "kc", "kr", "ang", "R", "q0", "rows", "B",
                                                        "Lq", "Lk", "S", "Hq", "Hkv", "d", "style",
                                                        "dtype")], None)
    assert call(style=0) == hasb.ATTN_ERR_INVALID_ARG          # RoPE is the point
    assert call(q0=261) == hasb.ATTN_ERR_INVALID_ARG           # query rows past the table
    assert call(S=200) == hasb.ATTN_ERR_INVALID_ARG            # Lk > S
    assert call(R=200) == hasb.ATTN_ERR_INVALID_ARG            # identity rows past the table
    assert call(kr=A + 0x200000 + 64) == hasb.ATTN_ERR_INVALID_ARG  # k_rot overlaps the cache
    assert call(ang=None) == hasb.ATTN_ERR_INVALID_ARG
    assert call(d=512) == hasb.ATTN_ERR_UNSUPPORTED
