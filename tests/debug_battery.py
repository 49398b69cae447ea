"""Calls every entry point of the library on small shapes and prints, per case,
a digest of the outputs' bytes and the fault and index-check words after it.

Run by tests/test_debug_gpu.py twice: in a process that loads the release
build and in one with HASB_DEBUG=1 (the index-checking build). Not a test
module itself (pytest does not collect it)."""

from __future__ import annotations

import hashlib
import json
import math
import sys

import torch

import head_attention_streaming_b200 as hasb
from head_attention_streaming_b200 import inputs


def _digest(*ts) -> str:
    h = hashlib.sha256()
    for t in ts:
        if t is not None:
            h.update(t.detach().contiguous().cpu().view(torch.uint8).numpy().tobytes())
    return h.hexdigest()[:16]


def cases():
    qkv = lambda B, Lq, Lk, Hq, Hkv, d, dt=torch.bfloat16, seed=1: [
        t.cuda() for t in inputs.make_qkv(B, Lq, Lk, Hq, Hkv, d, dt, seed=seed)]
    for d in (16, 32, 64, 128, 256):
        for mask, off in ((0, 0), (1, 77), (2, 60)):
            q, k, v = qkv(2, 200, 333, 4, 2, d, seed=d + mask)
            yield f"fwd d{d} m{mask}", lambda q=q, k=k, v=v, mask=mask, off=off: hasb.attn_fwd(
                q, k, v, causal=mask, kv_offset=off)
    q, k, v = qkv(1, 1100, 1100, 8, 2, 128, torch.float16, seed=5)          # pair split (causal, few pairs)
    yield "fwd causal pairs fp16", lambda: hasb.attn_fwd(q, k, v, causal=1)
    q, k, v = qkv(1, 600, 900, 4, 2, 128, seed=6)
    yield "window", lambda: hasb.attn_fwd_window(q, k, v, window=(100, 20), kv_offset=300)
    yield "splitkv causal", lambda: hasb.attn_fwd_splitkv(q, k, v, n_splits=3, causal=1, kv_offset=300)[:2]
    yield "splitkv static", lambda: hasb.attn_fwd_splitkv_static(q, k, v, n_splits=4)[:2]
    q2, k2, v2 = qkv(1, 300, 700, 4, 2, 256, seed=7)
    yield "splitkv d256", lambda: hasb.attn_fwd_splitkv(q2, k2, v2, n_splits=3)[:2]
    q8, k8, vt8 = hasb.fp8_cast(q), hasb.fp8_cast(k), hasb.fp8_cast_vt(v)
    yield "fp8 casts", lambda: (q8, k8, vt8)
    yield "fp8", lambda: hasb.attn_fwd_fp8(q8, k8, vt8, causal=1, kv_offset=300)
    sq8, sq = hasb.fp8_quantize_tokens(q)
    sk8, sk = hasb.fp8_quantize_tokens(k)
    sv8, sv = hasb.fp8_quantize_vt(v)
    yield "fp8 quantizers", lambda: (sq8, sq, sk8, sk, sv8, sv)
    yield "fp8 scaled", lambda: hasb.attn_fwd_fp8_scaled(sq8, sq, sk8, sk, sv8, sv)
    g = torch.Generator().manual_seed(3)
    ang = inputs.rope_angle_table(200, 128, hasb.ROPE_SPLIT, 50).cuda()
    qp, kp = qkv(2, 200, 200, 4, 2, 128, seed=8)[:2]
    gq = (1 + 0.1 * torch.randn(128, generator=g)).cuda()
    yield "prologue head split", lambda: hasb.qk_prologue(qp, kp, norm_scope=hasb.NORM_HEAD, gamma_q=gq,
                                                          gamma_k=gq, rope_style=hasb.ROPE_SPLIT,
                                                          angles_q=ang, angles_k=ang)
    angi = inputs.rope_angle_table(200, 128, hasb.ROPE_INTERLEAVED, 0).cuda()
    yield "prologue inner interleaved", lambda: hasb.qk_prologue(qp, kp, norm_scope=hasb.NORM_INNER,
                                                                 rope_style=hasb.ROPE_INTERLEAVED,
                                                                 angles_q=angi, angles_k=angi)
    C = 64
    cache = hasb.BlockKVCache(1, 2, 128, C, 2 * C, C)
    qs, ks, vs = qkv(1, 3 * C, 3 * C, 4, 2, 128, seed=9)
    angc = inputs.rope_angle_table(3 * C, 128, hasb.ROPE_SPLIT, 0).cuda()

    def stream():
        outs = []
        for c in range(3):
            sl = slice(c * C, (c + 1) * C)
            cache.before_update(c)
            outs += list(cache.attend(qs[:, sl].contiguous(), ks[:, sl].contiguous(), vs[:, sl].contiguous(),
                                      norm_scope=hasb.NORM_HEAD, rope_style=hasb.ROPE_SPLIT,
                                      angles_q=angc[sl].contiguous(), angles_k=angc[sl].contiguous()))
            cache.after_update(c)
        return outs
    yield "stream cache", stream
    qh, kh, vh = (t.cpu().pin_memory() for t in qkv(1, 700, 900, 4, 2, 128, seed=10))

    def host():
        oh = torch.empty_like(qh).pin_memory()
        lh = torch.empty(1, 4, 700).pin_memory()
        bufs = [torch.empty_like(qh, device="cuda"), torch.empty_like(kh, device="cuda"),
                torch.empty_like(vh, device="cuda"), torch.empty_like(qh, device="cuda"),
                torch.empty(1, 4, 700, device="cuda")]
        hasb.attn_fwd_host(qh, kh, vh, oh, lh, *bufs, causal=1, kv_offset=200)
        torch.cuda.synchronize()
        return oh, lh
    yield "host path", host


def main():
    torch.cuda.set_device(0)
    hasb.set_wait_timeout_ns(2_000_000_000)
    out = {"debug": hasb.is_debug_build(), "cases": []}
    for name, fn in cases():
        res = fn()
        torch.cuda.synchronize()
        ts = res if isinstance(res, (tuple, list)) else (res,)
        out["cases"].append({"name": name, "digest": _digest(*ts), "fault": hasb.device_fault(clear=True),
                             "site": hasb.debug_fault_site(clear=True)})
    print(json.dumps(out))


if __name__ == "__main__":
    sys.exit(main())
