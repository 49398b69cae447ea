"""Fused scaled-dot-product attention forward for NVIDIA B200 (sm_100a).

The computation runs in ``libattn_sm100.so`` (C ABI in ``include/attn.h``);
``binding`` marshals torch tensors into it. The library is loaded on first use,
so importing ``head_attention_streaming_b200.inputs`` needs no GPU.
"""

from .binding import (ATTN_ERR_CUDA, ATTN_ERR_INVALID_ARG, ATTN_ERR_SCRATCH_LIMIT, ATTN_ERR_TIMEOUT,
                      ATTN_ERR_UNSUPPORTED,
                      ATTN_OK, MASK_CAUSAL, MASK_CHUNK, MASK_NONE, NORM_HEAD, NORM_INNER,
                      NORM_NONE, ROPE_INTERLEAVED, ROPE_NONE, ROPE_SPLIT, AttnError, attn_fwd,
                      attn_fwd_cache, attn_fwd_host, attn_fwd_splitkv, attn_fwd_splitkv_static,
                      attn_fwd_window, attn_fwd_fp8, attn_fwd_fp8_scaled, fp8_cast, fp8_cast_vt,
                      fp8_quantize_tokens, fp8_quantize_vt, qk_prologue, rope_after_cache,
                      splitkv_workspace_bytes, stream_update,
                      debug_fault_site, device_fault, host_chunks, is_debug_build, lib, library_path, selftest_exp2,
                      selftest_mma,
                      selftest_wait_timeout,
                      set_wait_timeout_ns, status_string)

__all__ = ["attn_fwd", "attn_fwd_host", "AttnError", "lib", "library_path", "status_string", "device_fault",
           "debug_fault_site", "host_chunks", "is_debug_build",
           "set_wait_timeout_ns", "selftest_mma", "selftest_exp2", "selftest_wait_timeout", "ATTN_OK",
           "ATTN_ERR_INVALID_ARG", "ATTN_ERR_UNSUPPORTED", "ATTN_ERR_CUDA", "ATTN_ERR_TIMEOUT",
           "ATTN_ERR_SCRATCH_LIMIT",
           "MASK_NONE", "MASK_CAUSAL", "MASK_CHUNK", "qk_prologue", "NORM_NONE", "NORM_HEAD",
           "NORM_INNER", "ROPE_NONE", "ROPE_INTERLEAVED", "ROPE_SPLIT", "attn_fwd_cache", "stream_update",
           "attn_fwd_splitkv", "splitkv_workspace_bytes", "attn_fwd_splitkv_static", "attn_fwd_window",
           "attn_fwd_fp8", "fp8_cast", "fp8_cast_vt", "attn_fwd_fp8_scaled", "fp8_quantize_tokens",
           "fp8_quantize_vt", "rope_after_cache", "BlockKVCache"]

from .cache import BlockKVCache  # noqa: E402
