"""Exact attention forward for B200 (sm_100a): one fused tcgen05/TMA kernel
behind a C ABI (include/attn_fwd.h), with this thin Python binding.

    o, lse = attn_fwd(q, k, v, causal=True)

computes O = softmax(scale*QK^T [+causal mask]) V and the per-row natural-log
log-sum-exp, for bf16 [B, H, N, d] CUDA tensors with d in {64, 128};
attn_decode does the same for one new query row per head against N cached
keys (split-K/V).
"""
from ._lib import (AttnError, attn_bwd, attn_decode, attn_fwd, attn_fwd_fp8, attn_fwd_host,
                   attn_standard, bwd_workspace_bytes, decode_workspace_bytes, device_status,
                   fp8_workspace_bytes, fwd_schedule, header_functions, host_workspace_bytes,
                   load_library, standard_workspace_bytes, status_str, version)

__all__ = ["AttnError", "attn_bwd", "attn_decode", "attn_fwd", "attn_fwd_fp8", "attn_fwd_host",
           "attn_standard", "bwd_workspace_bytes", "fp8_workspace_bytes",
           "decode_workspace_bytes", "device_status", "fwd_schedule", "header_functions",
           "host_workspace_bytes", "load_library", "standard_workspace_bytes", "status_str",
           "version"]
