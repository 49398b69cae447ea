"""bench.py's roofline `traffic` field: the DRAM bytes per launch come from a
committed ncu summary, and only for the launch that summary measured (the video
workload's plain 16-bit kernel, while the kernel sources still hash to the
recorded digest). Every other workload or launch variant reports null."""

from __future__ import annotations

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_other_workloads_and_variants_get_no_traffic():
    for name in ("bf16_257x8x128", "fp16_causal_2x2048x8x64", "dit_selfattn_1785x40x128_qknorm",
                 "stream_chunk_1785_vs_7140_gqa40x8", "video_20480x56x128@1x8192x8192x32x32x128"):
        assert bench.attn_traffic(name) == (None, "no ncu summary of this workload / variant")
    assert bench.attn_traffic(bench.PROFILED_WORKLOAD, split_used=4)[0] is None
    assert bench.attn_traffic(bench.PROFILED_WORKLOAD, window=(2048, 2047))[0] is None


def test_profiled_workload_uses_the_summary_only_while_the_sources_match():
    traffic, src = bench.attn_traffic(bench.PROFILED_WORKLOAD)
    expect, esrc = bench.profiled_traffic()
    assert (traffic, src) == (expect, esrc)
    if src == "ncu":
        # per launch, near the 1.179 GB of algorithmic bytes of one video launch
        assert 1.0e9 < traffic < 1.4e9
    else:
        assert traffic is None and src == "kernel changed since the ncu capture"


def test_digest_ignores_comments_but_not_code(tmp_path):
    a, b, c = tmp_path / "a.cu", tmp_path / "b.cu", tmp_path / "c.cu"
    a.write_text("int f(int x) {\n  return x + 1;\n}\n")
    b.write_text("// the successor\nint f(int x) {  /* one more\n than x */\n\n  return x + 1;  // plus one\n}\n")
    c.write_text("int f(int x) {\n  return x + 2;\n}\n")
    h = lambda p: bench.kernel_source_hash([str(p)])
    assert h(a) == h(b)
    assert h(a) != h(c)
