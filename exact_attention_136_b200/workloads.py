"""Named workloads, FLOP accounting and row sampling (host logic only).

The shapes are the pages' own (Flash Attention | Hermes Skill, Workflow 1
Step 3 benchmark B2 H8 N2048 D64 fp16 and Step 4 accuracy check B1 H8 N512
D64 fp16 with scale 1/8; Workflow 2 Step 4 B4 N4096 H32 D64) plus the
long-context causal, sliding-window and FP8 cases this library is measured
on.  Every workload uses the ``[batch, seqlen, heads, headdim]`` layout.
"""

from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

BLOCK = 128  # FLOP accounting granularity (query rows x keys), fixed


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    n_q: int
    n_k: int
    H: int
    D: int
    dtype: str          # "fp16" | "bf16" | "e4m3"
    causal: bool
    window_left: int    # -1 = unlimited
    scale: float
    index: int          # seed offset: seeds are 1001/1002/1003 + 100 * index
    desc: str
    kv_heads: int = 0   # K/V heads (0 = H); fewer for multi-/grouped-query attention
    splits: int = 1     # key-range slices (fa_fwd_splitkv) for few query rows against many keys
    mask: str = ""      # "" none; "bool30": boolean [1, 1, N_q, N_k] mask, 30 % of pairs masked out

    @property
    def h_kv(self):
        return self.kv_heads if self.kv_heads > 0 else self.H

    @property
    def seeds(self):
        return (1001 + 100 * self.index, 1002 + 100 * self.index, 1003 + 100 * self.index)


WORKLOADS = {
    "pr1_b1h8n512d64_fp16": Workload(
        "pr1_b1h8n512d64_fp16", 1, 512, 512, 8, 64, "fp16", False, -1, 1.0 / 8.0, 0,
        "non-causal B1 H8 N512 D64 fp16, scale 1/8 (the pages' accuracy check)"),
    "b2h8n2048d64_fp16": Workload(
        "b2h8n2048d64_fp16", 2, 2048, 2048, 8, 64, "fp16", False, -1, 1.0 / 8.0, 1,
        "non-causal B2 H8 N2048 D64 fp16, scale 1/8 (the pages' benchmark shape)"),
    "causal_b4h32n8192d128_bf16": Workload(
        "causal_b4h32n8192d128_bf16", 4, 8192, 8192, 32, 128, "bf16", True, -1,
        1.0 / math.sqrt(128.0), 2,
        "causal B4 H32 N8192 D128 bf16, scale 1/sqrt(128)"),
    "swa4096_b1h32n32768d128_bf16": Workload(
        "swa4096_b1h32n32768d128_bf16", 1, 32768, 32768, 32, 128, "bf16", True, 4096,
        1.0 / math.sqrt(128.0), 3,
        "causal sliding window i-4096 <= j <= i, B1 H32 N32768 D128 bf16"),
    "fp8_causal_b2h16n16384d128": Workload(
        "fp8_causal_b2h16n16384d128", 2, 16384, 16384, 16, 128, "e4m3", True, -1,
        1.0 / math.sqrt(128.0), 4,
        "FP8 e4m3 causal B2 H16 N16384 D128, per-tensor scales, bf16 output"),
    "b4h32n4096d64_fp16": Workload(
        "b4h32n4096d64_fp16", 4, 4096, 4096, 32, 64, "fp16", False, -1, 1.0 / 8.0, 5,
        "non-causal B4 N4096 H32 D64 fp16 (the pages' flash-attn timing shape)"),
    "gqa_causal_b4h32kv8n8192d128_bf16": Workload(
        "gqa_causal_b4h32kv8n8192d128_bf16", 4, 8192, 8192, 32, 128, "bf16", True, -1,
        1.0 / math.sqrt(128.0), 6,
        "grouped-query causal B4 H32 (8 K/V heads) N8192 D128 bf16, scale 1/sqrt(128)", 8),
    "splitkv_b1h32kv8q128k65536d128_bf16": Workload(
        "splitkv_b1h32kv8q128k65536d128_bf16", 1, 128, 65536, 32, 128, "bf16", False, -1,
        1.0 / math.sqrt(128.0), 7,
        "128 query rows against 65536 keys (decode-like: 32 work units for 148 SMs unsplit), "
        "B1 H32 (8 K/V heads) D128 bf16, key range in 4 slices", 8, 4),
    "mask_b2h16n4096d128_bf16": Workload(
        "mask_b2h16n4096d128_bf16", 2, 4096, 4096, 16, 128, "bf16", False, -1,
        1.0 / math.sqrt(128.0), 8,
        "non-causal B2 H16 N4096 D128 bf16 with a boolean attn_mask [1, 1, N, N] (30 % masked out)",
        0, 1, "bool30"),
}

# order used by tests; the headline bench workload is the causal bf16 D128 case
ORDER = list(WORKLOADS)
HEADLINE = "causal_b4h32n8192d128_bf16"


def _visible_range(i, n_k, causal, window_left):
    """Inclusive key range [lo, hi] visible to query i (hi < lo when empty)."""
    lo = 0 if window_left < 0 else max(0, i - window_left)
    hi = n_k - 1 if not causal else min(i, n_k - 1)
    return lo, hi


def block_fraction(n_q, n_k, causal, window_left, block=BLOCK):
    """Fraction of block x block (query, key) tiles holding >= 1 visible pair."""
    nqb = -(-n_q // block)
    nkb = -(-n_k // block)
    count = 0
    for qb in range(nqb):
        i0 = qb * block
        i1 = min(n_q, i0 + block) - 1
        lo, _ = _visible_range(i0, n_k, causal, window_left)
        _, hi = _visible_range(i1, n_k, causal, window_left)
        if hi >= lo:
            count += (hi // block) - (lo // block) + 1
    return count / float(nqb * nkb)


def element_fraction(n_q, n_k, causal, window_left):
    """Fraction of (query, key) pairs that are visible."""
    total = 0
    for i in range(n_q):
        lo, hi = _visible_range(i, n_k, causal, window_left)
        total += max(0, hi - lo + 1)
    return total / float(n_q * n_k)


def make_mask(w: Workload):
    """The workload's attention mask as a CPU torch tensor (None when it has none); seeded like
    the inputs (seed 1004 + 100 * index)."""
    if not w.mask:
        return None
    import torch
    g = torch.Generator().manual_seed(1004 + 100 * w.index)
    if w.mask == "bool30":
        return torch.rand((1, 1, w.n_q, w.n_k), generator=g) >= 0.3
    raise ValueError(f"unknown mask {w.mask!r}")


def flops(w: Workload) -> float:
    """Counted FLOP of one forward: 4 * B * H * N_q * N_k * D times the block fraction."""
    return 4.0 * w.B * w.H * w.n_q * w.n_k * w.D * block_fraction(w.n_q, w.n_k, w.causal, w.window_left)


def sample_rows(w: Workload, count: int = 512, seed: int = 7) -> np.ndarray:
    """Sorted query rows for sampled parity and oracle timing on long sequences.

    Always includes rows 0, 1, 127, 128, N-1 and, for windows, the window-edge
    rows w-1, w, w+1; the rest are drawn without replacement from seed 7.
    """
    n = w.n_q
    must = {0, 1, 127, 128, n - 1}
    if w.window_left >= 0:
        must |= {w.window_left - 1, w.window_left, w.window_left + 1}
    must = {r for r in must if 0 <= r < n}
    if count >= n:
        return np.arange(n, dtype=np.int64)
    rng = np.random.default_rng(seed)
    pool = np.setdiff1d(np.arange(n), np.fromiter(must, dtype=np.int64))
    extra = rng.choice(pool, size=max(0, count - len(must)), replace=False)
    return np.sort(np.concatenate([np.fromiter(must, dtype=np.int64), extra]).astype(np.int64))
