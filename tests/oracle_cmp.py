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


def oracle(qkv, scale, causal, window_left, rows=None, mask=None, window_right=-1):
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
                                 mask=mb, window_right=window_right)
            O[b], L[b] = o[0], l[0]
        return O, L
    O = np.zeros((B, R, H, D))
    L = np.zeros((B, H, R))
    for b in range(B):
        for h in range(H):
            q = _f64(qkv.q[b:b + 1, :, h:h + 1], qkv.q_descale)
            k = _f64(qkv.k[b:b + 1, :, h:h + 1], qkv.k_descale)
            v = _f64(qkv.v[b:b + 1, :, h:h + 1], qkv.v_descale)
            o, l = attention_ref(q, k, v, scale, causal, window_left, rows=rows, window_right=window_right)
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


def backward_bounds(q, k, v, do, o_used, lse_used, scale, causal, window_left, unit_roundoff, dropout_p=0.0,
                    seed=0, offset=0, window_right=-1):
    """Per-element bounds (dq, dk, dv; shaped like q, k, v) on how far a
    backward computed the way the CUDA path does can be from the exact
    gradients, all arrays float64 numpy.

    The path recomputes P = exp(scale q.k - LSE) in fp32 from the forward's
    LSE (relative error e1 <= |LSE_used - LSE| + 1e-6), takes the row term
    from the forward's rounded output, Dt_i = sum_d dO_id O_used_id (error
    eD_i <= sum_d |dO_id| |O_used_id - O_id| + 1e-6 sum_d |dO_id O_id|),
    rounds P to the 16-bit input type for dV = P^T dO and dS = P (dP - Dt)
    for dK = scale dS^T Q and dQ = scale dS K (relative u each), and
    accumulates in fp32.  To first order:
        |d dV_kd| <= (u + e1) sum_i P_ik |dO_id|
        |d dS_ik| <= (u + e1)(1 + u) |dS_ik| + (1 + u) P_ik eD_i
        |d dK_kd| <= scale sum_i |d dS_ik| |Q_id|,  |d dQ_id| <= scale sum_k |d dS_ik| |K_kd|
    each plus 1e-5 of the matching sum of absolute products (fp32 sums).
    With fewer K/V heads than query heads (query head h reads K/V head
    h // (H / H_kv)) the dK and dV bounds add up over each group's heads.
    With dropout (keep bits Z) the same steps apply to the dropped forward:
    P in dV becomes Z P / (1 - p) and dP becomes Z dP / (1 - p).
    """
    from oracle import dropout_keep
    from oracle import attention_ref
    u = float(unit_roundoff)
    B, n_q, H, D = q.shape
    n_k, h_kv = k.shape[1], k.shape[2]
    group = H // h_kv
    bq, bk, bv = np.zeros(q.shape), np.zeros(k.shape), np.zeros(v.shape)
    o_ref, l_ref, probs = attention_ref(q, k, v, scale, causal, window_left, return_probs=True, dropout_p=dropout_p,
                                        seed=seed, offset=offset, window_right=window_right)
    for b in range(B):
        for h in range(H):
            hk = h // group
            p = probs[b, h]
            g = do[b, :, h, :]
            vv = v[b, :, hk, :]
            qq = q[b, :, h, :]
            kk = k[b, :, hk, :]
            dp = g @ vv.T
            pd = p
            if dropout_p > 0.0:
                z = dropout_keep(seed, offset, b, h, H, np.arange(n_q), n_k, dropout_p) / (1.0 - dropout_p)
                pd = z * p
                dp = z * dp
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            l_diff = np.where(np.isfinite(l_ref[b, h]), np.abs(lse_used[b, h] - l_ref[b, h]), 0.0)
            e1 = (1.01 * l_diff + 1e-6)[:, None]                       # per query row
            e_d = (np.abs(g) * np.abs(o_used[b, :, h, :] - o_ref[b, :, h, :])).sum(axis=1) + \
                1e-6 * np.abs(g * o_ref[b, :, h, :]).sum(axis=1)
            bv[b, :, hk, :] += ((u + e1) * pd).T @ np.abs(g) + 1e-5 * pd.T @ np.abs(g)
            d_ds = (u + e1) * (1 + u) * np.abs(ds) + (1 + u) * p * e_d[:, None]
            bk[b, :, hk, :] += scale * (d_ds.T @ np.abs(qq) + 1e-5 * np.abs(ds).T @ np.abs(qq))
            bq[b, :, h, :] = scale * (d_ds @ np.abs(kk) + 1e-5 * np.abs(ds) @ np.abs(kk))
    return bq, bk, bv
