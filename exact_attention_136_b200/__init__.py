"""Exact attention forward and backward for NVIDIA B200 (sm_100a).

    from exact_attention_136_b200 import forward, backward
    out, lse = forward(q, k, v, causal=True)      # [batch, seqlen, heads, headdim]
    dq, dk, dv = backward(q, k, v, out, lse, dout, causal=True)
    out = flash_attn_func(q, k, v, causal=True)  # the pages' call, with autograd

The computation runs in libfa_b200.so (hand-written sm_100a CUDA, C ABI in
include/fa.h); this package only marshals arguments.
"""

from .api import (auto_splits, backward, backward_varlen, device_status, forward, forward_fp8, forward_host,
                  forward_varlen, set_wait_limit_ns, wait_probe)
from .interface import flash_attn_func, flash_attn_varlen_func

__all__ = ["forward", "forward_fp8", "forward_host", "forward_varlen", "backward", "backward_varlen",
           "flash_attn_func", "flash_attn_varlen_func", "auto_splits", "device_status", "set_wait_limit_ns", "wait_probe"]
