"""Plain fp64 CPU oracle for exact scaled-dot-product attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path (the CUDA library
``libfa_b200.so`` and the Python binding in ``exact_attention_136_b200``)
imports, calls or links this module, and this module imports nothing from the
product package.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.

What it computes
----------------
"Standard attention" as the Flash Attention skill pages write it out
(Flash Attention | Hermes Skill, Workflow 1, Step 2 "Replace standard
attention"; the same step on the Russian mirror "Flash Attention - Fast
Memory-Efficient Attention"): the softmax over keys of the scaled
query-key dot products, multiplied by the values.  The explainer page
(FlashAttention, aiunderstanding.org, "Overview"/"Deep dive") states that
the tiled method reaches exactly the same attention, so the plain definition
written out here *is* the oracle:

    S_ij   = scale * sum_d Q[b,i,h,d] * K[b,j,h,d]          (all (i, j))
    S_ij   = -inf  where key j is not visible to query i
    m_i    = max_j S_ij
    l_i    = sum_j exp(S_ij - m_i)
    P_ij   = exp(S_ij - m_i) / l_i
    O_i    = sum_j P_ij V[b,j,h,:]
    LSE_i  = m_i + ln(l_i)            (natural log of sum_j exp(S_ij))

Rows that see no key at all get O_i = 0 and LSE_i = -inf.

Visibility (the "mask" of the pages' ``causal=True`` and ``window_size``
arguments; Flash Attention | Hermes Skill, Workflow 2, Steps 2-3):
    causal:                key j visible to query i only if j <= i
    window_left = w >= 0:  key j visible to query i only if j >= i - w
    window_right = w >= 0: key j visible to query i only if j <= i + w
    -1:                    no bound on that side (the pages' ``(-1, -1)``)
The pages' sliding-window example passes ``window_size=(256, 256)``, i.e. up
to 256 keys on each side of the query; with ``causal=True`` beside it
the keys after the query stay hidden (causal wins, as in the flash-attn
call the pages show), and without ``causal`` the right window admits keys up
to ``w`` positions after the query.
Indices are absolute (top-left aligned) also when N_q != N_k; this is the
plainest reading, since the pages only show N_q == N_k.

Attention mask (the ``attn_mask`` argument of the pages' SDPA call, Flash
Attention | Hermes Skill, Workflow 1, Step 2).  The pages pass ``mask`` to
``scaled_dot_product_attention`` without defining it; the reading here is
that call's convention: a boolean mask keeps key j for query i where it is
True, a floating-point mask is added to the scaled scores, S_ij =
scale * q_i.k_j + mask_ij, before the softmax.  It broadcasts over batch and
heads like ``[B or 1, H or 1, N_q, N_k]`` and applies together with causal
and window visibility.

Multi-query / grouped-query attention (Flash Attention | Hermes Skill,
Workflow 2, Step 3 "Enable advanced features": K and V may have fewer heads
than Q, "shared K/V across heads").  The pages do not say which query heads
share a K/V head; the reading here is contiguous groups: with H query heads
and H_kv key/value heads (H a multiple of H_kv), query head h uses key/value
head h // (H / H_kv).  H_kv = 1 is multi-query attention, H_kv = H the
ordinary case.

Dropout (the ``dropout_p`` argument of the pages' flash_attn_func, Flash
Attention | Hermes Skill, Workflow 2, Step 2; the pages define neither the
operation nor its random numbers).  The reading here is the usual one for
attention dropout: after the softmax, each probability P_ij is kept with
probability 1 - p and then divided by 1 - p, or set to 0, independently:

    O_i = sum_j (Z_ij / (1 - p)) P_ij V[b,j,h,:],   Z_ij in {0, 1}

with P and LSE exactly as above (the softmax normaliser counts every visible
key; dropout does not change LSE).  The keep bits Z come from the
counter-based generator in ``philox.py`` keyed by (seed, offset) and indexed
by (batch, query head, row, key), so any implementation can reproduce them.

Layouts follow the pages' flash_attn_func layout ``[batch, seqlen, nheads,
headdim]`` for Q, K, V and O (Workflow 2, Step 2), and ``[batch, heads,
N_q]`` for LSE (the pages print no LSE layout; this is our reading).

Everything is float64.  Inputs are the exact dtype-rounded (or dequantised
FP8) values, upcast.  Matrix products use numpy's BLAS matmul, which is the
only library primitive used; there is no tiling, fusion or online softmax.
"""

from __future__ import annotations

import math
from typing import Iterable

import numpy as np

from .philox import dropout_keep

__all__ = [
    "visibility",
    "attention_ref",
    "attention_bruteforce",
    "attention_backward_ref",
]


def visibility(rows: Iterable[int], n_k: int, causal: bool, window_left: int, window_right: int = -1) -> np.ndarray:
    """Boolean [len(rows), n_k] table: True where key j is visible to query i.

    Follows the pages' flash_attn_func arguments (Flash Attention | Hermes
    Skill, Workflow 2, Step 2 ``causal=True`` and Step 3 ``window_size=(left,
    right)``): causal hides keys after the query, a left window of ``w`` hides
    keys more than ``w`` positions before it, a right window of ``w`` keys
    more than ``w`` positions after it, ``-1`` means unlimited.
    """
    i = np.asarray(list(rows) if not isinstance(rows, np.ndarray) else rows, dtype=np.int64)[:, None]
    j = np.arange(n_k, dtype=np.int64)[None, :]
    vis = np.ones((i.shape[0], n_k), dtype=bool)
    if causal:
        vis &= j <= i
    if window_left >= 0:
        vis &= j >= i - window_left
    if window_right >= 0:
        vis &= j <= i + window_right
    return vis


def attention_ref(q, k, v, scale: float, causal: bool = False, window_left: int = -1,
                  rows=None, return_probs: bool = False, mask=None, dropout_p: float = 0.0,
                  seed: int = 0, offset: int = 0, window_right: int = -1):
    """Exact attention forward in float64 (definition in the module docstring).

    q: [B, N_q, H, D]; k, v: [B, N_k, H_kv, D] with H a multiple of H_kv
       (query head h reads key/value head h // (H / H_kv)); any real dtype,
       upcast to fp64.
    rows: optional 1-D array of query indices; only those rows are computed
          (used for long sequences where the full N_q x N_k matrix is large).
    mask: optional boolean (True = attend) or real array broadcastable to
          [B, H, N_q, N_k]; a real mask is added to the scaled scores.
    dropout_p, seed, offset: dropout of the probabilities (0 = none), keep
          bits from philox.dropout_keep.
    Returns (O [B, R, H, D], LSE [B, H, R]) with R = len(rows) (or N_q), and
    with ``return_probs`` also the softmax P [B, H, R, N_k] (before dropout).
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if q.ndim != 4 or k.ndim != 4 or v.ndim != 4:
        raise ValueError("q, k, v must be [batch, seqlen, heads, headdim]")
    B, n_q, H, D = q.shape
    n_k, h_kv = k.shape[1], k.shape[2]
    if k.shape != (B, n_k, h_kv, D) or v.shape != (B, n_k, h_kv, D):
        raise ValueError("k and v must be [B, N_k, H_kv, D] matching q")
    if h_kv < 1 or H % h_kv != 0:
        raise ValueError("the number of query heads must be a multiple of the key/value heads")
    group = H // h_kv
    rows = np.arange(n_q, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    R = rows.shape[0]
    vis0 = visibility(rows, n_k, causal, window_left, window_right)
    if mask is not None:
        mask = np.asarray(mask)
        if mask.ndim != 4 or mask.shape[2] != n_q or mask.shape[3] != n_k or mask.shape[0] not in (1, B) \
                or mask.shape[1] not in (1, H):
            raise ValueError("mask must be [B or 1, H or 1, N_q, N_k]")
        is_bool = mask.dtype == np.bool_

    out = np.zeros((B, R, H, D), dtype=np.float64)
    lse = np.full((B, H, R), -np.inf, dtype=np.float64)
    probs = np.zeros((B, H, R, n_k), dtype=np.float64) if return_probs else None
    for b in range(B):
        for h in range(H):
            hk = h // group   # key/value head shared by this query head's group
            vis = vis0
            add = None
            if mask is not None:
                m_bh = mask[b if mask.shape[0] > 1 else 0, h if mask.shape[1] > 1 else 0][rows]
                if is_bool:
                    vis = vis0 & m_bh
                else:
                    add = m_bh.astype(np.float64)
                    vis = vis0 & (add > -np.inf)
            seen = vis.any(axis=1)
            # scores of every selected query against every key
            s = scale * (q[b, rows, h, :] @ k[b, :, hk, :].T)
            if add is not None:
                s = s + np.where(vis, add, 0.0)
            s = np.where(vis, s, -np.inf)
            m = np.where(seen, s.max(axis=1, initial=-np.inf), 0.0)
            e = np.where(vis, np.exp(s - m[:, None]), 0.0)
            l = e.sum(axis=1)
            p = e / np.where(seen, l, 1.0)[:, None]
            if dropout_p > 0.0:
                keep = dropout_keep(seed, offset, b, h, H, rows, n_k, dropout_p)
                out[b, :, h, :] = (np.where(keep, p, 0.0) / (1.0 - dropout_p)) @ v[b, :, hk, :]
            else:
                out[b, :, h, :] = p @ v[b, :, hk, :]
            lse[b, h, :] = np.where(seen, m + np.log(np.where(seen, l, 1.0)), -np.inf)
            if return_probs:
                probs[b, h] = p
    if return_probs:
        return out, lse, probs
    return out, lse


def attention_bruteforce(q, k, v, scale: float, causal: bool = False, window_left: int = -1, mask=None,
                         dropout_p: float = 0.0, seed: int = 0, offset: int = 0, window_right: int = -1):
    """Pure-Python triple loop over (query, key, dim), for tiny shapes only.

    Written independently of ``attention_ref``: nested lists, ``math.exp``, no
    max subtraction, and the visibility rule spelled out inline.  Used only to
    pin ``attention_ref``.  Returns (O, LSE) as nested Python lists shaped like
    ``attention_ref``'s outputs.  K and V may have fewer heads than Q (query
    head h then reads head h * H_kv // H, the same contiguous groups).  mask:
    optional nested [B or 1][H or 1][N_q][N_k] of booleans (keep where True)
    or numbers (added to the scaled score).  dropout_p > 0: each weight is
    kept where philox.dropout_keep says so and then divided by 1 - dropout_p.
    """
    B = len(q)
    n_q = len(q[0])
    H = len(q[0][0])
    D = len(q[0][0][0])
    n_k = len(k[0])
    h_kv = len(k[0][0])
    O = [[[[0.0] * D for _ in range(H)] for _ in range(n_q)] for _ in range(B)]
    L = [[[float("-inf")] * n_q for _ in range(H)] for _ in range(B)]
    for b in range(B):
        for h in range(H):
            g = h * h_kv // H
            kept = dropout_keep(seed, offset, b, h, H, range(n_q), n_k, dropout_p) if dropout_p > 0 else None
            for i in range(n_q):
                weights = []
                for j in range(n_k):
                    if causal and j > i:
                        continue
                    if window_left != -1 and i - j > window_left:
                        continue
                    if window_right != -1 and j - i > window_right:
                        continue
                    bias = 0.0
                    if mask is not None:
                        mval = mask[b if len(mask) > 1 else 0][h if len(mask[0]) > 1 else 0][i][j]
                        if isinstance(mval, bool):
                            if not mval:
                                continue
                        else:
                            if mval == float("-inf"):
                                continue
                            bias = float(mval)
                    dot = 0.0
                    for d in range(D):
                        dot += float(q[b][i][h][d]) * float(k[b][j][g][d])
                    weights.append((j, math.exp(scale * dot + bias)))
                total = sum(w for _, w in weights)
                if not weights:
                    continue
                L[b][h][i] = math.log(total)
                for d in range(D):
                    acc = 0.0
                    for j, w in weights:
                        if kept is not None:
                            if not kept[i][j]:
                                continue
                            w = w / (1.0 - dropout_p)
                        acc += w * float(v[b][j][g][d])
                    O[b][i][h][d] = acc / total
    return O, L


def attention_backward_ref(q, k, v, do, scale: float, causal: bool = False, window_left: int = -1,
                           dropout_p: float = 0.0, seed: int = 0, offset: int = 0, window_right: int = -1):
    """Gradients of the exact attention forward, in float64.

    The pages name the backward pass only by its method: the speed and memory
    savings come from tiling and recomputation, i.e. the attention matrix is
    recomputed from the inputs instead of stored (Flash Attention | Hermes
    Skill, "Quick start"; the same on the Russian mirror "Flash Attention -
    Fast Memory-Efficient Attention"), and FlashAttention-3 runs FP16/BF16
    forward and backward (same pages, "Workflow 3: H100 FP8 optimization
    (FlashAttention-3)").  What it computes is fixed by the forward:
    for an upstream gradient dO of O, the vector-Jacobian products

        dV = P^T dO
        dP = dO V^T
        dS_ij = P_ij (dP_ij - sum_j' P_ij' dP_ij')      (softmax Jacobian)
        dQ = scale * dS K
        dK = scale * dS^T Q

    with P, S, visibility and the K/V head of each query head exactly as in
    ``attention_ref``; a K/V head shared by a group of query heads gets the sum
    of their dK and dV.  Invisible (i, j) pairs have P_ij = 0 and contribute
    nothing, and a row with no visible key contributes nothing at all.  With
    dropout (keep bits Z, probability p) the forward uses Pd = Z P / (1 - p),
    so dV = Pd^T dO, dP = Z (dO V^T) / (1 - p), and dS, dQ, dK follow as above
    (sum_j' P_ij' dP_ij' is still sum_d dO_id O_id).

    q, do: [B, N_q, H, D]; k, v: [B, N_k, H_kv, D].  Returns (dQ, dK, dV)
    shaped like q, k, v.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    B, n_q, H, D = q.shape
    n_k, h_kv = k.shape[1], k.shape[2]
    if do.shape != q.shape:
        raise ValueError("do must be shaped like q")
    _, _, probs = attention_ref(q, k, v, scale, causal, window_left, return_probs=True, window_right=window_right)
    rows = np.arange(n_q, dtype=np.int64)
    group = H // h_kv
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            hk = h // group
            p = probs[b, h]                       # [N_q, N_k], zero where invisible
            g = do[b, :, h, :]                    # [N_q, D]
            dp = g @ v[b, :, hk, :].T             # [N_q, N_k]
            if dropout_p > 0.0:
                z = dropout_keep(seed, offset, b, h, H, rows, n_k, dropout_p) / (1.0 - dropout_p)
                dv[b, :, hk, :] += (z * p).T @ g
                dp = z * dp
            else:
                dv[b, :, hk, :] += p.T @ g
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            dq[b, :, h, :] = scale * (ds @ k[b, :, hk, :])
            dk[b, :, hk, :] += scale * (ds.T @ q[b, :, h, :])
    return dq, dk, dv
