"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module holds no attention arithmetic.  It draws Q, K, V i.i.d. N(0, 1)
in fp32 on the CPU ``torch.Generator`` (the pages draw their inputs with
``torch.randn``: Flash Attention | Hermes Skill, Quick start and Workflow 1,
Steps 3-4), rounds them to the storage dtype (round-to-nearest-even), and for
FP8 quantises each tensor to e4m3 with one fp32 scale per tensor
(scale = amax / 448, values clamped to the finite e4m3 range).

Both sides receive the same rounded values: the CUDA path gets the storage
tensors, the oracle gets them upcast to float64 (FP8: dequantised as
``x8 * scale`` in float64).
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

E4M3_MAX = 448.0

_DTYPES = {
    "fp16": torch.float16,
    "bf16": torch.bfloat16,
    "e4m3": torch.float8_e4m3fn,
}


def torch_dtype(name: str) -> torch.dtype:
    return _DTYPES[name]


@dataclass
class QKV:
    """Storage tensors (CPU) plus per-tensor descales (1.0 unless FP8)."""

    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    q_descale: float = 1.0
    k_descale: float = 1.0
    v_descale: float = 1.0

    def as_float64(self):
        """The exact values the method sees, as float64 tensors (FP8: dequantised)."""
        return (self.q.to(torch.float64) * self.q_descale,
                self.k.to(torch.float64) * self.k_descale,
                self.v.to(torch.float64) * self.v_descale)


def randn(shape, seed: int) -> torch.Tensor:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def quantize_e4m3(x: torch.Tensor):
    """Per-tensor e4m3 quantisation: returns (x8, scale) with x ~= x8 * scale."""
    amax = float(x.abs().max())
    scale = amax / E4M3_MAX if amax > 0 else 1.0
    scale = float(torch.tensor(scale, dtype=torch.float32))  # an fp32 value
    x8 = (x / scale).clamp_(-E4M3_MAX, E4M3_MAX).to(torch.float8_e4m3fn)
    return x8, scale


def make_qkv(B: int, n_q: int, n_k: int, H: int, D: int, dtype: str,
             seeds=(1001, 1002, 1003), h_kv: int = None) -> QKV:
    """Q [B, n_q, H, D], K and V [B, n_k, h_kv, D] (h_kv defaults to H) drawn
    N(0, 1) from the given seeds."""
    h_kv = H if h_kv is None else h_kv
    q = randn((B, n_q, H, D), seeds[0])
    k = randn((B, n_k, h_kv, D), seeds[1])
    v = randn((B, n_k, h_kv, D), seeds[2])
    if dtype == "e4m3":
        q8, sq = quantize_e4m3(q)
        k8, sk = quantize_e4m3(k)
        v8, sv = quantize_e4m3(v)
        return QKV(q8, k8, v8, sq, sk, sv)
    t = _DTYPES[dtype]
    return QKV(q.to(t), k.to(t), v.to(t))
