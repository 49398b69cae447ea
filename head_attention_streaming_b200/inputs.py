"""Seeded synthetic inputs and the named workloads.

This module is shared by the tests, the benchmark and the smoke check. It holds
no attention arithmetic: it draws Q, K, V and describes the workload shapes.
The CUDA path and the FP64 oracle both consume what it returns.

Recipe: one CPU ``torch.Generator`` seeded per workload draws Q, then K, then V
as i.i.d. N(0, 1) float32 tensors, which are rounded to the 16-bit storage
dtype (round to nearest even). The DiT self-attention workload first applies a
head-scoped Q/K RMSNorm with unit weight and eps 1e-6 in float32 (the
flashdreams developer guide, "Multi Head Attention Definition", RMSNorm
equation with m = d; ``qk_norm_eps=1e-6`` in its Cosmos example); V is never
normalised.
"""

from __future__ import annotations

import dataclasses
import math

import torch

MASK_NONE = 0
MASK_CAUSAL = 1
MASK_CHUNK = 2


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Lq: int
    Lk: int
    Hq: int
    Hkv: int
    d: int
    dtype: str            # "bf16" | "fp16"
    mask: int             # 0 none, 1 causal, 2 streaming chunk
    kv_offset: int
    scale: float
    seed: int
    qk_rmsnorm: bool = False
    sample_rows: int = 0  # >0: oracle checks this many seeded rows per head

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16

    def flops(self) -> float:
        """4*B*Hq*Lq*Lk*d, halved for the causal mask."""
        f = 4.0 * self.B * self.Hq * self.Lq * self.Lk * self.d
        return f / 2.0 if self.mask == MASK_CAUSAL else f


# The five synthetic workloads. Shapes come from the pages:
#  * [1,257,8,128] and [1,20480,56,128] BF16: the FlashAttention-4 runtime page,
#    "GB10 Validation" table;
#  * [2,2048,8,64] FP16 causal, scale 1/8: the skill page's timing snippet
#    ("Workflow 1", Step 3) with flash-attn's causal flag;
#  * L=1785, 40 heads x 128 (width 5120): the LightX2V DreamZero QKV GEMM shape
#    [1785, 5120]; Q/K RMSNorm from the developer guide's definition;
#  * the streaming chunk: 4 cached chunks of 1785 tokens, 8 K/V heads for 40
#    query heads, chunk at cache offset 3*1785.
WORKLOADS = {
    w.name: w for w in [
        Workload("bf16_257x8x128", 1, 257, 257, 8, 8, 128, "bf16", MASK_NONE, 0,
                 1.0 / math.sqrt(128), seed=1),
        Workload("fp16_causal_2x2048x8x64", 2, 2048, 2048, 8, 8, 64, "fp16", MASK_CAUSAL, 0,
                 1.0 / 8.0, seed=2),
        Workload("dit_selfattn_1785x40x128_qknorm", 1, 1785, 1785, 40, 40, 128, "bf16",
                 MASK_NONE, 0, 1.0 / math.sqrt(128), seed=3, qk_rmsnorm=True),
        Workload("stream_chunk_1785_vs_7140_gqa40x8", 1, 1785, 7140, 40, 8, 128, "bf16",
                 MASK_CHUNK, 5355, 1.0 / math.sqrt(128), seed=4),
        Workload("video_20480x56x128", 1, 20480, 20480, 56, 56, 128, "bf16", MASK_NONE, 0,
                 1.0 / math.sqrt(128), seed=5, sample_rows=256),
        # a short streaming chunk (256 tokens) against the same 7140-key cache:
        # one 256-row query pair per head, 40 work units for 148 SMs unless the
        # keys are split (attn_fwd_splitkv)
        Workload("stream_chunk_256_vs_7140_gqa40x8", 1, 256, 7140, 40, 8, 128, "bf16",
                 MASK_CHUNK, 6884, 1.0 / math.sqrt(128), seed=6),
    ]
}

# Order used by the tests and the benchmark (small case first).
WORKLOAD_ORDER = list(WORKLOADS)
BENCH_WORKLOAD = "video_20480x56x128"


def _rmsnorm_heads(x: torch.Tensor, eps: float = 1e-6) -> torch.Tensor:
    """Head-scoped RMSNorm with unit weight: x / sqrt(mean(x^2 over d) + eps)."""
    return x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + eps)


def make_qkv(B: int, Lq: int, Lk: int, Hq: int, Hkv: int, d: int, dtype=torch.bfloat16,
             seed: int = 0, qk_rmsnorm: bool = False):
    """Draw Q [B,Lq,Hq,d], K and V [B,Lk,Hkv,d] on the CPU in ``dtype``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    q = torch.randn((B, Lq, Hq, d), generator=g, dtype=torch.float32)
    k = torch.randn((B, Lk, Hkv, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Lk, Hkv, d), generator=g, dtype=torch.float32)
    if qk_rmsnorm:
        q = _rmsnorm_heads(q)
        k = _rmsnorm_heads(k)
    return q.to(dtype), k.to(dtype), v.to(dtype)


def workload_inputs(w: Workload):
    """CPU inputs of a named workload."""
    return make_qkv(w.B, w.Lq, w.Lk, w.Hq, w.Hkv, w.d, w.torch_dtype, w.seed, w.qk_rmsnorm)


def sample_rows(Lq: int, n: int, seed: int):
    """``n`` distinct query rows drawn without replacement (seeded), sorted.

    Used where the oracle checks a sample of rows per head of a long sequence.
    """
    if n >= Lq:
        return torch.arange(Lq)
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) + 1000)
    return torch.randperm(Lq, generator=g)[:n].sort().values


def rope_angle_table(L: int, d: int, style: int, pos0: int = 0, base: float = 10000.0) -> torch.Tensor:
    """The caller-side ``rope_freqs`` input: float32 [L, d] rotation angles for
    sequence positions ``pos0 .. pos0 + L - 1``, built as the developer guide
    ("Multi Head Attention Definition") describes the model doing it: pair r
    of a head gets ``theta = p * base**(-2 r / d)``, and the table is
    "expanded" to one angle per feature, the pair's angle stored at both of its
    features ((2r, 2r + 1) for style 1, interleaved; (r, r + d/2) for style 2,
    split-half). The prologue reads it; it computes no angles itself.
    """
    r = torch.arange(d // 2, dtype=torch.float64)
    omega = base ** (-2.0 * r / d)
    theta = (pos0 + torch.arange(L, dtype=torch.float64))[:, None] * omega[None, :]
    table = torch.empty(L, d, dtype=torch.float64)
    if style == 1:
        table[:, 0::2] = theta
        table[:, 1::2] = theta
    elif style == 2:
        table[:, : d // 2] = theta
        table[:, d // 2:] = theta
    else:
        raise ValueError("style must be 1 (interleaved) or 2 (split-half)")
    return table.to(torch.float32)
