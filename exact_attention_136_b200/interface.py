"""The pages' call, ``flash_attn_func``, over this library, with autograd.

Flash Attention | Hermes Skill, Workflow 2, Step 2 calls
``flash_attn_func(q, k, v, dropout_p=0.0, causal=...)`` on
``[batch, seqlen, nheads, headdim]`` tensors, and Step 3 adds
``window_size=(left, right)`` and K/V with fewer heads; the default softmax
scale is 1/sqrt(headdim) (the page's "auto-scale").  This module gives that
call, backed by ``forward`` and ``backward`` (argument marshalling only: the
computation is libfa_b200.so's), so code written against the pages' call can
switch to this library and train through it.

Readings (the pages leave these open):
- ``window_size=(left, right)``: key j is visible to query i only if
  i - left <= j <= i + right, -1 meaning no bound on that side
  (fa_fwd_window).  With ``causal=True`` the right window is zero whatever
  ``right`` says (the page pairs causal=True with a two-sided window, which
  contradict each other; causal wins).
- ``dropout_p``: the usual attention dropout, each softmax probability kept
  with probability 1 - p and scaled by 1 / (1 - p) (fa_fwd_dropout).  The
  pages name no random generator; each call draws a 64-bit seed from
  torch's default generator (so ``torch.manual_seed`` makes runs
  repeatable) and the backward redraws the same keep bits from it.
- The backward takes fp16 / bf16 inputs; K/V may have fewer heads than Q.
"""

from __future__ import annotations

from typing import Optional, Tuple

import torch

from .api import backward, backward_varlen, forward, forward_varlen


def _window(causal: bool, window_size: Tuple[int, int]) -> Tuple[int, int]:
    """(left, right) as forward / backward take them; right -1 under causal."""
    left, right = (int(window_size[0]), int(window_size[1]))
    if left < -1 or right < -1:
        raise ValueError("window_size entries are -1 (unlimited) or >= 0")
    return (left, -1) if causal else (left, right)


class _FlashAttn(torch.autograd.Function):
    """O = attention(q, k, v); the backward recomputes from O and the LSE."""

    @staticmethod
    def forward(ctx, q, k, v, scale, causal, window_left, window_right, dropout_p, seed):
        if dropout_p:
            out, lse = forward(q, k, v, scale, causal, window_left, dropout_p=dropout_p, seed=seed,
                               window_right=window_right)
        else:
            out, lse = forward(q, k, v, scale, causal, window_left, window_right=window_right)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.scale, ctx.causal, ctx.window_left, ctx.window_right = scale, causal, window_left, window_right
        ctx.dropout_p, ctx.seed = dropout_p, seed
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, dlse):
        if dlse is not None and bool(torch.any(dlse != 0)):
            raise NotImplementedError("gradients through the returned LSE are not supported")
        q, k, v, out, lse = ctx.saved_tensors
        if ctx.dropout_p:
            dq, dk, dv = backward(q, k, v, out, lse, dout.contiguous(), ctx.scale, ctx.causal, ctx.window_left,
                                  dropout_p=ctx.dropout_p, seed=ctx.seed, window_right=ctx.window_right)
        else:
            dq, dk, dv = backward(q, k, v, out, lse, dout.contiguous(), ctx.scale, ctx.causal, ctx.window_left,
                                  window_right=ctx.window_right)
        return dq, dk, dv, None, None, None, None, None, None


def flash_attn_func(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, dropout_p: float = 0.0,
                    softmax_scale: Optional[float] = None, causal: bool = False,
                    window_size: Tuple[int, int] = (-1, -1), return_lse: bool = False):
    """The pages' flash_attn_func on [batch, seqlen, nheads, headdim] tensors.

    Returns O (and LSE [batch, nheads, seqlen_q], natural log, with
    return_lse).  Differentiable in q, k, v (fp16 / bf16).  dropout_p > 0
    drops attention probabilities (a fresh seed from torch's default
    generator per call).
    """
    dropout_p = float(dropout_p)
    if not (0.0 <= dropout_p < 1.0):
        raise ValueError("dropout_p must be in [0, 1)")
    wl, wr = _window(bool(causal), window_size)
    scale = float(softmax_scale) if softmax_scale is not None else q.shape[-1] ** -0.5
    seed = int(torch.randint(0, 2 ** 62, (1,)).item()) if dropout_p > 0.0 else 0
    needs_grad = torch.is_grad_enabled() and any(t.requires_grad for t in (q, k, v))
    if needs_grad:
        out, lse = _FlashAttn.apply(q, k, v, scale, bool(causal), wl, wr, dropout_p, seed)
    elif dropout_p > 0.0:
        out, lse = forward(q, k, v, scale, bool(causal), wl, dropout_p=dropout_p, seed=seed, window_right=wr)
    else:
        out, lse = forward(q, k, v, scale, bool(causal), wl, window_right=wr)
    return (out, lse) if return_lse else out


class _FlashAttnPacked(torch.autograd.Function):
    """O = attention over a packed batch; the backward recomputes from O and the LSE."""

    @staticmethod
    def forward(ctx, q, k, v, cu_q, cu_k, max_q, max_k, scale, causal, window_left, window_right, dropout_p, seed):
        kw = dict(window_right=window_right, dropout_p=dropout_p, seed=seed if dropout_p else None)
        out, lse = forward_varlen(q, k, v, cu_q, cu_k, max_q, max_k, scale, causal, window_left, **kw)
        ctx.save_for_backward(q, k, v, out, lse, cu_q, cu_k)
        ctx.args = (max_q, max_k, scale, causal, window_left, kw)
        ctx.mark_non_differentiable(lse)
        return out, lse

    @staticmethod
    def backward(ctx, dout, dlse):
        if dlse is not None and bool(torch.any(dlse != 0)):
            raise NotImplementedError("gradients through the returned LSE are not supported")
        q, k, v, out, lse, cu_q, cu_k = ctx.saved_tensors
        max_q, max_k, scale, causal, window_left, kw = ctx.args
        dq, dk, dv = backward_varlen(q, k, v, out, lse, dout.contiguous(), cu_q, cu_k, max_q, max_k, scale, causal,
                                     window_left, **kw)
        return (dq, dk, dv) + (None,) * 10


def flash_attn_varlen_func(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens_q: torch.Tensor,
                           cu_seqlens_k: torch.Tensor, max_seqlen_q: int, max_seqlen_k: int, dropout_p: float = 0.0,
                           softmax_scale: Optional[float] = None, causal: bool = False,
                           window_size: Tuple[int, int] = (-1, -1), return_lse: bool = False):
    """flash_attn_func's options over a packed batch: q [total_q, nheads, headdim], k, v [total_k,
    nheads_kv, headdim], sequence b at rows cu_seqlens_q[b] .. cu_seqlens_q[b+1] (int32 CUDA tensors;
    max_seqlen_q / max_seqlen_k bound every sequence).  Returns O [total_q, nheads, headdim] (and LSE
    [nheads, total_q] with return_lse); differentiable in q, k, v (fp16 / bf16)."""
    dropout_p = float(dropout_p)
    if not (0.0 <= dropout_p < 1.0):
        raise ValueError("dropout_p must be in [0, 1)")
    wl, wr = _window(bool(causal), window_size)
    scale = float(softmax_scale) if softmax_scale is not None else q.shape[-1] ** -0.5
    seed = int(torch.randint(0, 2 ** 62, (1,)).item()) if dropout_p > 0.0 else 0
    needs_grad = torch.is_grad_enabled() and any(t.requires_grad for t in (q, k, v))
    if needs_grad:
        out, lse = _FlashAttnPacked.apply(q, k, v, cu_seqlens_q, cu_seqlens_k, int(max_seqlen_q), int(max_seqlen_k),
                                          scale, bool(causal), wl, wr, dropout_p, seed)
    else:
        out, lse = forward_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, int(max_seqlen_q), int(max_seqlen_k), scale,
                                  bool(causal), wl, window_right=wr, dropout_p=dropout_p,
                                  seed=seed if dropout_p else None)
    return (out, lse) if return_lse else out
