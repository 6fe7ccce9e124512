"""Test helper: run the fp64 oracle on the exact values a CUDA call saw.

Upcasts one (batch, head) slice at a time, so long sequences only ever hold
one head's Q, K and V in float64.
"""

import numpy as np
import torch

from oracle import attention_ref

TOL_O = {"fp16": 4e-3, "bf16": 1.6e-2, "e4m3": 6e-2}
TOL_LSE = 1e-3


def _f64(t: torch.Tensor, descale: float) -> np.ndarray:
    return (t.to(torch.float64) * descale).numpy()


def oracle(qkv, scale, causal, window_left, rows=None, mask=None):
    """(O [B, R, H, D], LSE [B, H, R]) in float64 for the given QKV bundle (mask: numpy,
    [B or 1, H or 1, N_q, N_k], bool or real)."""
    B, n_q, H, D = qkv.q.shape
    R = n_q if rows is None else len(rows)
    if qkv.k.shape[2] != H or mask is not None:
        # grouped K/V heads: the oracle maps query heads to K/V heads itself
        # (one batch at a time, all heads)
        O = np.zeros((B, R, H, D))
        L = np.zeros((B, H, R))
        for b in range(B):
            mb = None if mask is None else mask[b:b + 1] if mask.shape[0] > 1 else mask
            o, l = attention_ref(_f64(qkv.q[b:b + 1], qkv.q_descale), _f64(qkv.k[b:b + 1], qkv.k_descale),
                                 _f64(qkv.v[b:b + 1], qkv.v_descale), scale, causal, window_left, rows=rows,
                                 mask=mb)
            O[b], L[b] = o[0], l[0]
        return O, L
    O = np.zeros((B, R, H, D))
    L = np.zeros((B, H, R))
    for b in range(B):
        for h in range(H):
            q = _f64(qkv.q[b:b + 1, :, h:h + 1], qkv.q_descale)
            k = _f64(qkv.k[b:b + 1, :, h:h + 1], qkv.k_descale)
            v = _f64(qkv.v[b:b + 1, :, h:h + 1], qkv.v_descale)
            o, l = attention_ref(q, k, v, scale, causal, window_left, rows=rows)
            O[b, :, h] = o[0, :, 0]
            L[b, h] = l[0, 0]
    return O, L


def compare(out, lse, ref_o, ref_l, rows=None):
    """Max |dO| and max |dLSE| (the -inf pattern of LSE must match exactly)."""
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.float().cpu().numpy().astype(np.float64) if lse is not None else None
    if rows is not None:
        o = o[:, np.asarray(rows)]
        l = l[:, :, np.asarray(rows)] if l is not None else None
    assert np.all(np.isfinite(o)), "non-finite output"
    d_o = float(np.max(np.abs(o - ref_o))) if o.size else 0.0
    d_l = 0.0
    if l is not None and l.size:
        inf_ref = ~np.isfinite(ref_l)
        assert np.array_equal(inf_ref, ~np.isfinite(l)), "LSE -inf pattern differs"
        if (~inf_ref).any():
            d_l = float(np.max(np.abs(l[~inf_ref] - ref_l[~inf_ref])))
    return d_o, d_l
