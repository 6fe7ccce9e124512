"""Python entry points over the C ABI (argument marshalling only).

Tensors use the pages' flash_attn_func layout [batch, seqlen, nheads,
headdim] (Flash Attention | Hermes Skill, Workflow 2, Step 2).  PyTorch only
allocates outputs and supplies the current CUDA stream; every step of the
computation runs in libfa_b200.so.
"""

from __future__ import annotations

import ctypes
import math
from typing import Optional, Tuple

import torch

from . import _lib

_DT = {torch.float16: _lib.FA_FP16, torch.bfloat16: _lib.FA_BF16, torch.float8_e4m3fn: _lib.FA_E4M3}


def _check_inputs(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor):
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (no CPU path)")
        if t.dim() != 4:
            raise ValueError(f"{name} must be [batch, seqlen, heads, headdim]")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in _DT:
        raise ValueError("q, k, v must share one dtype: float16, bfloat16 or float8_e4m3fn")
    B, n_q, H, D = q.shape
    h_kv = k.shape[2]
    if k.shape[0] != B or k.shape[3] != D or v.shape != k.shape:
        raise ValueError("k and v must be [B, N_k, H_kv, D] with q's B and D")
    if h_kv < 1 or H % h_kv != 0:
        raise ValueError("q's head count must be a multiple of k's and v's (grouped-query attention)")
    if not (q.device == k.device == v.device):
        raise ValueError("q, k, v must be on one device")
    return B, n_q, k.shape[1], H, h_kv, D


def _outputs(q, B, n_q, H, D, out, lse, want_lse):
    out_dtype = torch.float16 if q.dtype == torch.float16 else torch.bfloat16
    if out is None:
        out = torch.empty((B, n_q, H, D), dtype=out_dtype, device=q.device)
    elif out.shape != (B, n_q, H, D) or out.dtype != out_dtype or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous {out_dtype} tensor of shape {(B, n_q, H, D)}")
    if lse is None and want_lse:
        lse = torch.empty((B, H, n_q), dtype=torch.float32, device=q.device)
    elif lse is not None and (lse.shape != (B, H, n_q) or lse.dtype != torch.float32
                              or not lse.is_contiguous()):
        raise ValueError(f"lse must be a contiguous float32 tensor of shape {(B, H, n_q)}")
    return out, lse


def _mask_args(attn_mask: torch.Tensor, q: torch.Tensor, B: int, H: int, n_q: int, n_k: int):
    """attn_mask ([N_q, N_k] or [B or 1, H or 1, N_q, N_k]; bool = attend where True, float = added to
    the scaled scores) as the library takes it: bytes or the output's 16-bit type, rows starting on
    16-byte boundaries, broadcast dimensions with stride 0.  Like SDPA, a float mask must have the
    inputs' type (the output's 16-bit type for FP8 inputs); no other float type is narrowed
    silently.  A mask already in that form is passed as it is; otherwise it is copied into a
    padded buffer.  Returns (buffer, kind, stride_b, stride_h, stride_q)."""
    m = attn_mask
    if m.dim() == 2:
        m = m[None, None]
    if (m.dim() != 4 or m.shape[2] != n_q or m.shape[3] != n_k or m.shape[0] not in (1, B)
            or m.shape[1] not in (1, H)):
        raise ValueError("attn_mask must be [N_q, N_k] or [B or 1, H or 1, N_q, N_k]")
    out_dt = torch.float16 if q.dtype == torch.float16 else torch.bfloat16
    if m.dtype == torch.bool:
        kind, dt = _lib.FA_MASK_BOOL, torch.uint8
    elif m.dtype == out_dt:
        kind, dt = _lib.FA_MASK_ADD, out_dt
    else:
        raise ValueError(f"attn_mask must be bool or {out_dt} (the inputs' type), not {m.dtype}")
    es = 1 if dt == torch.uint8 else 2
    direct = m.view(torch.uint8) if m.dtype == torch.bool else m
    # broadcast dimensions read with stride 0
    strides = [direct.stride(i) if direct.shape[i] > 1 else 0 for i in range(4)]
    if n_q == 1:
        strides[2] = n_k
    # passed as it is when its rows are whole 16-byte chunks on 16-byte boundaries
    if (direct.device == q.device and (n_k * es) % 16 == 0 and direct.stride(3) == 1
            and direct.data_ptr() % 16 == 0 and all((st * es) % 16 == 0 for st in strides[:3])
            and strides[2] >= n_k):
        return direct, kind, strides[0], strides[1], strides[2]
    per = 16 // es
    n_pad = -(-n_k // per) * per
    buf = torch.zeros((m.shape[0], m.shape[1], n_q, n_pad), dtype=dt, device=q.device)
    buf[..., :n_k] = m.to(device=q.device).view(torch.uint8) if m.dtype == torch.bool else m.to(device=q.device)
    sb = buf.stride(0) if m.shape[0] > 1 else 0
    sh = buf.stride(1) if m.shape[1] > 1 else 0
    return buf, kind, sb, sh, buf.stride(2)


def _masked(q, k, v, out, lse, B, n_q, n_k, H, h_kv, D, scale, causal, window_left, dt, descales, attn_mask, s):
    # a padded copy of the mask is made on the launching stream (allocated
    # there too), so the kernel reads it after the copy and its memory is not
    # handed out again before the kernel has run
    with torch.cuda.stream(s):
        buf, kind, sb, sh, sq = _mask_args(attn_mask, q, B, H, n_q, n_k)
    rc = _lib.lib().fa_fwd_mask(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                lse.data_ptr() if lse is not None else None, B, n_q, n_k, H, h_kv, D, scale,
                                int(bool(causal)), int(window_left), dt, float(descales[0]), float(descales[1]),
                                float(descales[2]), buf.data_ptr(), kind, sb, sh, sq, s.cuda_stream)
    _lib.check(rc, "fa_fwd_mask")


def auto_splits(B: int, n_q: int, n_k: int, H: int, device=None) -> int:
    """Key-range slices that fill the GPU: one per SM for every work unit
    (256 query rows of one (batch, head)) short of the SM count, at most one
    per 128-key block; 1 when the units already cover the SMs."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    units = B * H * max(1, -(-n_q // 256))
    if units >= sms:
        return 1
    return max(1, min(-(-n_k // 128), -(-sms // units)))


def _splitkv(q, k, v, out, lse, B, n_q, n_k, H, h_kv, D, scale, causal, window_left, dt, descales,
             num_splits, s):
    """fa_fwd_splitkv with a workspace from PyTorch's allocator."""
    nbytes = _lib.lib().fa_fwd_splitkv_workspace_bytes(B, n_q, n_k, H, D, num_splits)
    # allocated on the launching stream: not handed out again before the kernels have used it
    with torch.cuda.stream(s):
        ws = torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=q.device)
    rc = _lib.lib().fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                   lse.data_ptr() if lse is not None else None, B, n_q, n_k, H, h_kv, D, scale,
                                   int(bool(causal)), int(window_left), dt, float(descales[0]),
                                   float(descales[1]), float(descales[2]), int(num_splits),
                                   ws.data_ptr() if nbytes else None, int(nbytes), s.cuda_stream)
    _lib.check(rc, "fa_fwd_splitkv")


def forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: Optional[float] = None,
            causal: bool = False, window_left: int = -1, out: Optional[torch.Tensor] = None,
            lse: Optional[torch.Tensor] = None, return_lse: bool = True,
            stream: Optional[torch.cuda.Stream] = None, num_splits: int = 1,
            attn_mask: Optional[torch.Tensor] = None, dropout_p: float = 0.0, seed: Optional[int] = None,
            offset: int = 0, window_right: int = -1) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Exact attention forward; returns (out, lse).

    scale=None means 1/sqrt(headdim), the pages' auto scale (Workflow 2,
    Step 2).  window_left=-1 means no window.  window_right >= 0 keeps only
    keys at most that many positions after the query (the right entry of the
    pages' window_size, Workflow 2, Step 3; fa_fwd_window), not combined with
    attn_mask, num_splits or dropout.  For float8_e4m3fn inputs all
    descales are 1; use forward_fp8 to pass per-tensor scales.  k and v may
    have fewer heads than q (multi-query / grouped-query attention, Workflow
    2, Step 3): query head h then reads head h // (H / H_kv).  num_splits > 1
    splits the key range into that many slices run in parallel and merged
    (for few query rows against many keys); 0 picks it with auto_splits.
    attn_mask: the pages' SDPA mask (Workflow 1, Step 2) -- bool (attend where
    True) or float (added to the scaled scores), [N_q, N_k] or
    [B or 1, H or 1, N_q, N_k]; not combined with num_splits.
    dropout_p > 0: dropout of the attention probabilities (fa_fwd_dropout;
    fp16 / bf16, not combined with attn_mask or num_splits), with the keep
    bits drawn from the 64-bit seed (required) and the 32-bit offset; the
    backward needs the same seed and offset.
    """
    B, n_q, n_k, H, h_kv, D = _check_inputs(q, k, v)
    _check_right_window(window_right, attn_mask, num_splits)
    if dropout_p:
        return _dropout_forward(q, k, v, scale, causal, window_left, out, lse, return_lse, stream, num_splits,
                                attn_mask, dropout_p, seed, offset, window_right)
    if num_splits == 0:
        # (a right window takes the one-launch path: no key-range slices)
        num_splits = 1 if window_right != -1 else auto_splits(B, n_q, n_k, H, q.device)
    if q.dtype == torch.float8_e4m3fn:
        return forward_fp8(q, k, v, 1.0, 1.0, 1.0, scale, causal, window_left, out, lse, return_lse, stream,
                           num_splits, attn_mask, window_right)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    out, lse = _outputs(q, B, n_q, H, D, out, lse, return_lse)
    with torch.cuda.device(q.device):
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        lse_p = lse.data_ptr() if lse is not None else None
        if attn_mask is not None:
            if num_splits > 1:
                raise ValueError("attn_mask is not combined with num_splits")
            _masked(q, k, v, out, lse, B, n_q, n_k, H, h_kv, D, scale, causal, window_left, _DT[q.dtype],
                    (1.0, 1.0, 1.0), attn_mask, s)
            return out, lse
        if num_splits > 1:
            _splitkv(q, k, v, out, lse, B, n_q, n_k, H, h_kv, D, scale, causal, window_left, _DT[q.dtype],
                     (1.0, 1.0, 1.0), num_splits, s)
            return out, lse
        if window_right != -1:
            rc = _lib.lib().fa_fwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_p, B, n_q,
                                          n_k, H, h_kv, D, scale, int(bool(causal)), int(window_left),
                                          int(window_right), _DT[q.dtype], 1.0, 1.0, 1.0, s.cuda_stream)
            _lib.check(rc, "fa_fwd_window")
            return out, lse
        if h_kv == H:
            rc = _lib.lib().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_p, B, n_q, n_k, H,
                                   D, scale, int(bool(causal)), int(window_left), _DT[q.dtype], s.cuda_stream)
        else:
            rc = _lib.lib().fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse_p, B, n_q,
                                       n_k, H, h_kv, D, scale, int(bool(causal)), int(window_left), _DT[q.dtype],
                                       1.0, 1.0, 1.0, s.cuda_stream)
    _lib.check(rc, "fa_fwd" if h_kv == H else "fa_fwd_gqa")
    return out, lse


def _check_right_window(window_right, attn_mask=None, num_splits=1):
    if window_right == -1:
        return
    if window_right < -1:
        raise ValueError("window_right must be -1 (no bound) or >= 0")
    if attn_mask is not None or num_splits not in (0, 1):
        raise ValueError("window_right is not combined with attn_mask or num_splits "
                         "(a boolean attn_mask expresses any window)")


def _fwd_ex(q, k, v, out, lse, B, n_q, n_k, H, h_kv, D, scale, causal, window_left, window_right, dt, descales,
            stream, packed=None, dropout=(0.0, 0, 0)):
    """fa_fwd_ex: every combinable option in one call.  packed = (cu_q, cu_k, total_q, total_k) or None;
    dropout = (p, seed, offset)."""
    a = _lib.FwdArgs()
    a.q, a.k, a.v, a.out = q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr()
    a.lse = lse.data_ptr() if lse is not None else None
    a.B, a.N_q, a.N_k, a.H, a.H_kv, a.D = B, n_q, n_k, H, h_kv, D
    a.scale, a.causal, a.window_left, a.window_right = scale, int(bool(causal)), int(window_left), int(window_right)
    a.dtype = dt
    a.q_descale, a.k_descale, a.v_descale = (float(x) for x in descales)
    if packed is not None:
        a.cu_seqlens_q, a.cu_seqlens_k = packed[0].data_ptr(), packed[1].data_ptr()
        a.total_q, a.total_k = packed[2], packed[3]
    a.dropout_p, a.seed, a.offset = float(dropout[0]), int(dropout[1]) & ((1 << 64) - 1), int(dropout[2]) & 0xFFFFFFFF
    _lib.check(_lib.lib().fa_fwd_ex(ctypes.byref(a), stream.cuda_stream), "fa_fwd_ex")


def _bwd_ex(q, k, v, out, dout, lse, dq, dk, dv, B, n_q, n_k, H, h_kv, D, scale, causal, window_left,
            window_right, dt, ws, nbytes, stream, packed=None, dropout=(0.0, 0, 0)):
    """fa_bwd_ex: the backward of _fwd_ex with the same options."""
    a = _lib.BwdArgs()
    a.q, a.k, a.v, a.out, a.dout, a.lse = (t.data_ptr() for t in (q, k, v, out, dout, lse))
    a.dq, a.dk, a.dv = dq.data_ptr(), dk.data_ptr(), dv.data_ptr()
    a.B, a.N_q, a.N_k, a.H, a.H_kv, a.D = B, n_q, n_k, H, h_kv, D
    a.scale, a.causal, a.window_left, a.window_right = scale, int(bool(causal)), int(window_left), int(window_right)
    a.dtype = dt
    if packed is not None:
        a.cu_seqlens_q, a.cu_seqlens_k = packed[0].data_ptr(), packed[1].data_ptr()
        a.total_q, a.total_k = packed[2], packed[3]
    a.dropout_p, a.seed, a.offset = float(dropout[0]), int(dropout[1]) & ((1 << 64) - 1), int(dropout[2]) & 0xFFFFFFFF
    a.workspace, a.workspace_bytes = ws.data_ptr(), nbytes
    _lib.check(_lib.lib().fa_bwd_ex(ctypes.byref(a), stream.cuda_stream), "fa_bwd_ex")


def _dropout_forward(q, k, v, scale, causal, window_left, out, lse, return_lse, stream, num_splits, attn_mask,
                     dropout_p, seed, offset, window_right=-1):
    B, n_q, n_k, H, h_kv, D = _check_inputs(q, k, v)
    if not (0.0 <= dropout_p < 1.0):
        raise ValueError("dropout_p must be in [0, 1)")
    if q.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("dropout takes fp16 or bf16 inputs")
    if attn_mask is not None or num_splits not in (0, 1):
        raise ValueError("dropout is not combined with attn_mask or num_splits")
    if seed is None:
        raise ValueError("dropout needs an explicit seed (and offset) so the backward can redraw the mask")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    out, lse = _outputs(q, B, n_q, H, D, out, lse, return_lse)
    with torch.cuda.device(q.device):
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        if window_right != -1:
            _fwd_ex(q, k, v, out, lse, B, n_q, n_k, H, h_kv, D, scale, causal, window_left, window_right,
                    _DT[q.dtype], (1.0, 1.0, 1.0), s, dropout=(dropout_p, seed, offset))
            return out, lse
        rc = _lib.lib().fa_fwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                       lse.data_ptr() if lse is not None else None, B, n_q, n_k, H, h_kv, D, scale,
                                       int(bool(causal)), int(window_left), _DT[q.dtype], float(dropout_p),
                                       int(seed) & ((1 << 64) - 1), int(offset) & 0xFFFFFFFF, s.cuda_stream)
    _lib.check(rc, "fa_fwd_dropout")
    return out, lse


def forward_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens_q: torch.Tensor,
                   cu_seqlens_k: torch.Tensor, max_seqlen_q: int, max_seqlen_k: int, scale: Optional[float] = None,
                   causal: bool = False, window_left: int = -1, descales=(1.0, 1.0, 1.0),
                   stream: Optional[torch.cuda.Stream] = None, window_right: int = -1, dropout_p: float = 0.0,
                   seed: Optional[int] = None, offset: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """Attention over a packed batch of sequences (fa_fwd_varlen): q [total_q,
    H, D], k, v [total_k, H_kv, D]; sequence b owns rows cu_seqlens_q[b] ..
    cu_seqlens_q[b+1] and keys cu_seqlens_k[b] .. cu_seqlens_k[b+1] (int32 CUDA
    tensors of B + 1 entries).  Returns (out [total_q, H, D], lse [H, total_q]).
    window_right and dropout (p, seed, offset; sequence b draws as batch b
    would) go through fa_fwd_ex."""
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or t.dim() != 3 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor [total, heads, headdim]")
    if not (q.dtype == k.dtype == v.dtype) or q.dtype not in _DT:
        raise ValueError("q, k, v must share one dtype: float16, bfloat16 or float8_e4m3fn")
    for name, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if not t.is_cuda or t.dtype != torch.int32 or t.dim() != 1 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous int32 CUDA tensor")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold B + 1 >= 2 entries")
    total_q, H, D = q.shape
    total_k, h_kv = k.shape[0], k.shape[1]
    if v.shape != k.shape or k.shape[2] != D or h_kv < 1 or H % h_kv != 0:
        raise ValueError("k and v must be [total_k, H_kv, D] with H a multiple of H_kv")
    B = cu_seqlens_q.numel() - 1
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    out_dtype = torch.float16 if q.dtype == torch.float16 else torch.bfloat16
    out = torch.empty((total_q, H, D), dtype=out_dtype, device=q.device)
    lse = torch.empty((H, total_q), dtype=torch.float32, device=q.device)
    _check_right_window(window_right)
    if dropout_p and seed is None:
        raise ValueError("dropout needs an explicit seed (and offset) so the backward can redraw the mask")
    with torch.cuda.device(q.device):
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        if window_right != -1 or dropout_p:
            _fwd_ex(q, k, v, out, lse, B, int(max_seqlen_q), int(max_seqlen_k), H, h_kv, D, scale, causal,
                    window_left, window_right, _DT[q.dtype], descales, s,
                    packed=(cu_seqlens_q, cu_seqlens_k, total_q, total_k),
                    dropout=(dropout_p, seed or 0, offset))
            return out, lse
        rc = _lib.lib().fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                      cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, int(max_seqlen_q),
                                      int(max_seqlen_k), total_q, total_k, H, h_kv, D, scale, int(bool(causal)),
                                      int(window_left), _DT[q.dtype], float(descales[0]), float(descales[1]),
                                      float(descales[2]), s.cuda_stream)
    _lib.check(rc, "fa_fwd_varlen")
    return out, lse


def backward_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, lse: torch.Tensor,
                    dout: torch.Tensor, cu_seqlens_q: torch.Tensor, cu_seqlens_k: torch.Tensor, max_seqlen_q: int,
                    max_seqlen_k: int, scale: Optional[float] = None, causal: bool = False, window_left: int = -1,
                    stream: Optional[torch.cuda.Stream] = None, window_right: int = -1, dropout_p: float = 0.0,
                    seed: Optional[int] = None, offset: int = 0) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Gradients (dq [total_q, H, D], dk, dv [total_k, H_kv, D]) of forward_varlen over the same packed
    batch (fa_bwd_varlen), from its out and lse [H, total_q] (fp16 / bf16).  max_seqlen_q / max_seqlen_k
    must bound every sequence's length.  window_right and dropout as given to the forward (fa_bwd_ex)."""
    for name, t in (("q", q), ("k", k), ("v", v), ("out", out), ("dout", dout)):
        if not t.is_cuda or t.dim() != 3 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor [total, heads, headdim]")
    if q.dtype not in (torch.float16, torch.bfloat16) or not (q.dtype == k.dtype == v.dtype):
        raise ValueError("backward_varlen takes fp16 or bf16 q, k, v of one dtype")
    for name, t in (("out", out), ("dout", dout)):
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device:
            raise ValueError(f"{name} must be a tensor like q")
    for name, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k)):
        if not t.is_cuda or t.dtype != torch.int32 or t.dim() != 1 or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous int32 CUDA tensor")
    if cu_seqlens_q.numel() != cu_seqlens_k.numel() or cu_seqlens_q.numel() < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must both hold B + 1 >= 2 entries")
    total_q, H, D = q.shape
    total_k, h_kv = k.shape[0], k.shape[1]
    if v.shape != k.shape or k.shape[2] != D or h_kv < 1 or H % h_kv != 0:
        raise ValueError("k and v must be [total_k, H_kv, D] with H a multiple of H_kv")
    if lse.shape != (H, total_q) or lse.dtype != torch.float32 or lse.device != q.device or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [H, total_q] tensor on q's device")
    B = cu_seqlens_q.numel() - 1
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    with torch.cuda.device(q.device):
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        nbytes = int(_lib.lib().fa_bwd_workspace_bytes(1, total_q, H, D))
        with torch.cuda.stream(s):
            ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
        _check_right_window(window_right)
        if dropout_p and seed is None:
            raise ValueError("a dropout backward needs the forward's seed (and offset)")
        if window_right != -1 or dropout_p:
            _bwd_ex(q, k, v, out, dout, lse, dq, dk, dv, B, int(max_seqlen_q), int(max_seqlen_k), H, h_kv, D, scale,
                    causal, window_left, window_right, _DT[q.dtype], ws, nbytes, s,
                    packed=(cu_seqlens_q, cu_seqlens_k, total_q, total_k), dropout=(dropout_p, seed or 0, offset))
            if s != torch.cuda.current_stream(q.device):
                for t in (dq, dk, dv):
                    t.record_stream(s)
            return dq, dk, dv
        rc = _lib.lib().fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(),
                                      lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                      cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), B, int(max_seqlen_q),
                                      int(max_seqlen_k), total_q, total_k, H, h_kv, D, scale, int(bool(causal)),
                                      int(window_left), _DT[q.dtype], ws.data_ptr(), nbytes, s.cuda_stream)
        if s != torch.cuda.current_stream(q.device):
            for t in (dq, dk, dv):
                t.record_stream(s)
    _lib.check(rc, "fa_bwd_varlen")
    return dq, dk, dv


def forward_fp8(q8: torch.Tensor, k8: torch.Tensor, v8: torch.Tensor, q_descale: float, k_descale: float,
                v_descale: float, scale: Optional[float] = None, causal: bool = False,
                window_left: int = -1, out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                return_lse: bool = True, stream: Optional[torch.cuda.Stream] = None, num_splits: int = 1,
                attn_mask: Optional[torch.Tensor] = None, window_right: int = -1):
    """FP8 e4m3 forward with per-tensor descales; out is bfloat16."""
    B, n_q, n_k, H, h_kv, D = _check_inputs(q8, k8, v8)
    _check_right_window(window_right, attn_mask, num_splits)
    if num_splits == 0:
        num_splits = 1 if window_right != -1 else auto_splits(B, n_q, n_k, H, q8.device)
    if q8.dtype != torch.float8_e4m3fn:
        raise ValueError("forward_fp8 takes float8_e4m3fn tensors")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    out, lse = _outputs(q8, B, n_q, H, D, out, lse, return_lse)
    with torch.cuda.device(q8.device):
        s = stream if stream is not None else torch.cuda.current_stream(q8.device)
        lse_p = lse.data_ptr() if lse is not None else None
        if attn_mask is not None:
            if num_splits > 1:
                raise ValueError("attn_mask is not combined with num_splits")
            _masked(q8, k8, v8, out, lse, B, n_q, n_k, H, h_kv, D, scale, causal, window_left, _lib.FA_E4M3,
                    (q_descale, k_descale, v_descale), attn_mask, s)
            return out, lse
        if num_splits > 1:
            _splitkv(q8, k8, v8, out, lse, B, n_q, n_k, H, h_kv, D, scale, causal, window_left, _lib.FA_E4M3,
                     (q_descale, k_descale, v_descale), num_splits, s)
            return out, lse
        if window_right != -1:
            rc = _lib.lib().fa_fwd_window(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), out.data_ptr(), lse_p, B, n_q,
                                          n_k, H, h_kv, D, scale, int(bool(causal)), int(window_left),
                                          int(window_right), _lib.FA_E4M3, float(q_descale), float(k_descale),
                                          float(v_descale), s.cuda_stream)
            _lib.check(rc, "fa_fwd_window")
            return out, lse
        if h_kv == H:
            rc = _lib.lib().fa_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), out.data_ptr(), lse_p, B, n_q,
                                       n_k, H, D, scale, int(bool(causal)), int(window_left), float(q_descale),
                                       float(k_descale), float(v_descale), s.cuda_stream)
        else:
            rc = _lib.lib().fa_fwd_gqa(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), out.data_ptr(), lse_p, B, n_q,
                                       n_k, H, h_kv, D, scale, int(bool(causal)), int(window_left), _lib.FA_E4M3,
                                       float(q_descale), float(k_descale), float(v_descale), s.cuda_stream)
    _lib.check(rc, "fa_fwd_fp8" if h_kv == H else "fa_fwd_gqa")
    return out, lse


def backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor, lse: torch.Tensor,
             dout: torch.Tensor, scale: Optional[float] = None, causal: bool = False, window_left: int = -1,
             stream: Optional[torch.cuda.Stream] = None, dropout_p: float = 0.0, seed: Optional[int] = None,
             offset: int = 0, window_right: int = -1) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Gradients (dq, dk, dv) of forward(q, k, v, scale, causal, window_left,
    window_right=...) for the upstream gradient dout, from the forward's out
    and lse (fp16 / bf16).  k and v may have fewer heads than q (grouped-query attention):
    dk and dv of a K/V head then sum over the query heads that read it.
    dropout_p, seed, offset: those of a dropout forward (fa_bwd_dropout redraws
    its keep bits).  The fp32 workspace the library needs is taken from
    torch's allocator for the call."""
    B, n_q, n_k, H, h_kv, D = _check_inputs(q, k, v)
    if q.dtype not in (torch.float16, torch.bfloat16):
        raise ValueError("backward takes fp16 or bf16 inputs")
    _check_right_window(window_right)
    for name, t in (("out", out), ("dout", dout)):
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous tensor like q")
    if lse.shape != (B, H, n_q) or lse.dtype != torch.float32 or lse.device != q.device or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 [B, H, N_q] tensor on q's device")
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    with torch.cuda.device(q.device):
        s = stream if stream is not None else torch.cuda.current_stream(q.device)
        nbytes = int(_lib.lib().fa_bwd_workspace_bytes(B, n_q, H, D))
        with torch.cuda.stream(s):
            ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device)
        if dropout_p and window_right != -1:
            if seed is None:
                raise ValueError("a dropout backward needs the forward's seed (and offset)")
            _bwd_ex(q, k, v, out, dout, lse, dq, dk, dv, B, n_q, n_k, H, h_kv, D, scale, causal, window_left,
                    window_right, _DT[q.dtype], ws, nbytes, s, dropout=(dropout_p, seed, offset))
            rc = _lib.FA_OK
        elif dropout_p:
            if seed is None:
                raise ValueError("a dropout backward needs the forward's seed (and offset)")
            rc = _lib.lib().fa_bwd_dropout(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(),
                                           lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, n_q, n_k, H,
                                           h_kv, D, scale, int(bool(causal)), int(window_left), _DT[q.dtype],
                                           float(dropout_p), int(seed) & ((1 << 64) - 1), int(offset) & 0xFFFFFFFF,
                                           ws.data_ptr(), nbytes, s.cuda_stream)
        elif window_right != -1:
            rc = _lib.lib().fa_bwd_window(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(),
                                          lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, n_q, n_k, H,
                                          h_kv, D, scale, int(bool(causal)), int(window_left), int(window_right),
                                          _DT[q.dtype], ws.data_ptr(), nbytes, s.cuda_stream)
        elif h_kv == H:
            rc = _lib.lib().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(),
                                   lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, n_q, n_k, H, D,
                                   scale, int(bool(causal)), int(window_left), _DT[q.dtype], ws.data_ptr(), nbytes,
                                   s.cuda_stream)
        else:
            rc = _lib.lib().fa_bwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), dout.data_ptr(),
                                       lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, n_q, n_k, H,
                                       h_kv, D, scale, int(bool(causal)), int(window_left), _DT[q.dtype],
                                       ws.data_ptr(), nbytes, s.cuda_stream)
        # the outputs come from the current stream's pool: keep them reserved
        # until the launching stream's kernels have written them
        if s != torch.cuda.current_stream(q.device):
            for t in (dq, dk, dv):
                t.record_stream(s)
    _lib.check(rc, "fa_bwd_dropout" if dropout_p else "fa_bwd_window" if window_right != -1
               else ("fa_bwd" if h_kv == H else "fa_bwd_gqa"))
    return dq, dk, dv


def forward_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, staging, scale: float, causal: bool = False,
                 window_left: int = -1, descales=(1.0, 1.0, 1.0), out: Optional[torch.Tensor] = None,
                 lse: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
                 synchronize: bool = True):
    """Forward on HOST tensors through fa_fwd_host.

    q, k, v are CPU tensors (pinned for asynchronous copies); `staging` is a
    dict of device tensors "q", "k", "v", "out", "lse" that the call copies
    through.  Returns the host (out, lse).  synchronize=False enqueues the
    copies and the forward on the stream and returns at once
    (fa_fwd_host_async): out and lse are valid after the stream completes,
    and calls on other streams with their own staging run concurrently.
    """
    B, n_q, H, D = q.shape
    n_k = k.shape[1]
    dt = _DT[q.dtype]
    out_dtype = torch.float16 if q.dtype == torch.float16 else torch.bfloat16
    if out is None:
        out = torch.empty((B, n_q, H, D), dtype=out_dtype, pin_memory=True)
    if lse is None:
        lse = torch.empty((B, H, n_q), dtype=torch.float32, pin_memory=True)
    dev = staging["q"].device
    with torch.cuda.device(dev):
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        fn = _lib.lib().fa_fwd_host if synchronize else _lib.lib().fa_fwd_host_async
        rc = fn(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                staging["q"].data_ptr(), staging["k"].data_ptr(), staging["v"].data_ptr(),
                staging["out"].data_ptr(), staging["lse"].data_ptr(), B, n_q, n_k, H, D,
                float(scale), int(bool(causal)), int(window_left), dt,
                float(descales[0]), float(descales[1]), float(descales[2]), s.cuda_stream)
    _lib.check(rc, "fa_fwd_host" if synchronize else "fa_fwd_host_async")
    return out, lse


def device_status(stream: Optional[torch.cuda.Stream] = None, device=None) -> Tuple[int, int]:
    """(status, flags) of the device status word; synchronises the stream and clears the word."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        flags = ctypes.c_int(0)
        rc = _lib.lib().fa_device_status(s.cuda_stream, ctypes.byref(flags))
    return rc, flags.value


def set_wait_limit_ns(limit_ns: int) -> None:
    _lib.lib().fa_set_wait_limit_ns(int(limit_ns))


def wait_probe(limit_ns: int, stream: Optional[torch.cuda.Stream] = None, device=None) -> None:
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(dev):
        s = stream if stream is not None else torch.cuda.current_stream(dev)
        _lib.check(_lib.lib().fa_wait_probe(int(limit_ns), s.cuda_stream), "fa_wait_probe")
