"""flash_attn_func (the pages' call) on the CPU: its argument handling and
autograd plumbing, with the library's forward / backward replaced by the
fp64 oracle (the GPU entry points themselves are covered by the GPU tests)."""

import math

import numpy as np
import pytest
import torch

import exact_attention_136_b200.interface as itf
from oracle import attention_backward_ref, attention_ref


@pytest.fixture
def oracle_backend(monkeypatch):
    calls = []

    def fwd(q, k, v, scale, causal, window_left, dropout_p=0.0, seed=None, offset=0, window_right=-1):
        calls.append(("fwd", scale, causal, window_left) + ((dropout_p, seed, offset) if dropout_p else ())
                     + ((window_right,) if window_right != -1 else ()))
        o, l = attention_ref(q.detach().numpy(), k.detach().numpy(), v.detach().numpy(), scale, causal, window_left,
                             dropout_p=dropout_p, seed=seed or 0, offset=offset, window_right=window_right)
        return torch.from_numpy(o), torch.from_numpy(l)

    def bwd(q, k, v, out, lse, dout, scale, causal, window_left, dropout_p=0.0, seed=None, offset=0, window_right=-1):
        calls.append(("bwd", scale, causal, window_left) + ((dropout_p, seed, offset) if dropout_p else ())
                     + ((window_right,) if window_right != -1 else ()))
        g = attention_backward_ref(q.detach().numpy(), k.detach().numpy(), v.detach().numpy(), dout.numpy(), scale,
                                   causal, window_left, dropout_p=dropout_p, seed=seed or 0, offset=offset,
                                   window_right=window_right)
        return tuple(torch.from_numpy(x) for x in g)

    monkeypatch.setattr(itf, "forward", fwd)
    monkeypatch.setattr(itf, "backward", bwd)
    return calls


def _plain_attention(q, k, v, scale, causal, wl, wr=-1):
    """Softmax attention with torch ops, [B, N, H, D] (torch autograd differentiates it)."""
    s = torch.einsum("bihd,bjhd->bhij", q, k) * scale
    n_q, n_k = q.shape[1], k.shape[1]
    i = torch.arange(n_q)[:, None]
    j = torch.arange(n_k)[None, :]
    vis = torch.ones(n_q, n_k, dtype=torch.bool)
    if causal:
        vis &= j <= i
    if wl >= 0:
        vis &= j >= i - wl
    if wr >= 0:
        vis &= j <= i + wr
    s = s.masked_fill(~vis, float("-inf"))
    return torch.einsum("bhij,bjhd->bihd", torch.softmax(s, dim=-1), v)


@pytest.mark.parametrize("causal, window", [(False, (-1, -1)), (True, (-1, -1)), (True, (3, 3)), (False, (2, -1)),
                                           (False, (2, 3)), (False, (-1, 1))])
def test_gradients_match_torch_autograd(oracle_backend, causal, window):
    g = torch.Generator().manual_seed(7)
    q, k, v = (torch.randn(1, 9, 2, 4, generator=g, dtype=torch.float64, requires_grad=True) for _ in range(3))
    do = torch.randn(1, 9, 2, 4, generator=g, dtype=torch.float64)
    out = itf.flash_attn_func(q, k, v, causal=causal, window_size=window)
    out.backward(do)
    wl, wr = window[0], (-1 if causal else window[1])
    q2, k2, v2 = (t.detach().clone().requires_grad_() for t in (q, k, v))
    ref = _plain_attention(q2, k2, v2, 0.5, causal, wl, wr)   # default scale 1/sqrt(4)
    ref.backward(do)
    assert torch.allclose(out, ref, atol=1e-12)
    for a, b in ((q.grad, q2.grad), (k.grad, k2.grad), (v.grad, v2.grad)):
        assert torch.allclose(a, b, atol=1e-12)
    # scale, causal and window reach the library unchanged, forward then backward
    extra = (wr,) if wr != -1 else ()
    assert oracle_backend == [("fwd", 0.5, causal, wl) + extra, ("bwd", 0.5, causal, wl) + extra]


def test_no_grad_path_and_lse(oracle_backend):
    q, k, v = (torch.randn(1, 5, 1, 8, dtype=torch.float64) for _ in range(3))
    out, lse = itf.flash_attn_func(q, k, v, softmax_scale=0.3, causal=True, return_lse=True)
    o, l = attention_ref(q.numpy(), k.numpy(), v.numpy(), 0.3, True, -1)
    assert np.allclose(out.numpy(), o) and np.allclose(lse.numpy(), l)
    assert oracle_backend == [("fwd", 0.3, True, -1)]   # no autograd record without requires_grad


def test_rejected_arguments(oracle_backend):
    q = torch.zeros(1, 4, 1, 8, dtype=torch.float64)
    for bad_p in (-0.1, 1.0):
        with pytest.raises(ValueError):
            itf.flash_attn_func(q, q, q, dropout_p=bad_p)
    with pytest.raises(ValueError):
        itf.flash_attn_func(q, q, q, window_size=(-2, -1))
    assert oracle_backend == []


def test_causal_two_sided_window_reads_as_left_window(oracle_backend):
    # the pages pair causal=True with window_size=(256, 256); causal wins on the right
    q = torch.zeros(1, 4, 1, 8, dtype=torch.float64)
    itf.flash_attn_func(q, q, q, causal=True, window_size=(256, 256))
    assert oracle_backend == [("fwd", 8 ** -0.5, True, 256)]


def test_dropout_gradients_and_seed_plumbing(oracle_backend):
    """dropout_p > 0: the forward and the backward get the same seed (drawn
    from torch's default generator), and the gradients are torch autograd's
    of softmax * Z / (1 - p) @ V with the oracle's keep bits Z."""
    from oracle import dropout_keep
    g = torch.Generator().manual_seed(9)
    B, n, H, D, p = 1, 10, 2, 4, 0.3
    q, k, v = (torch.randn(B, n, H, D, generator=g, dtype=torch.float64, requires_grad=True) for _ in range(3))
    do = torch.randn(B, n, H, D, generator=g, dtype=torch.float64)
    torch.manual_seed(1234)
    out = itf.flash_attn_func(q, k, v, dropout_p=p, causal=True)
    out.backward(do)
    (_, _, _, _, p_f, seed_f, off_f), (_, _, _, _, p_b, seed_b, off_b) = oracle_backend
    assert (p_f, seed_f, off_f) == (p_b, seed_b, off_b) == (p, seed_f, 0)
    # the same torch seed gives the same dropout seed
    torch.manual_seed(1234)
    again = itf.flash_attn_func(q.detach(), k.detach(), v.detach(), dropout_p=p, causal=True)
    assert oracle_backend[-1][5] == seed_f and torch.equal(again, out.detach())
    q2, k2, v2 = (t.detach().clone().requires_grad_() for t in (q, k, v))
    s = torch.einsum("bihd,bjhd->bhij", q2, k2) * D ** -0.5
    s = s.masked_fill(~torch.tril(torch.ones(n, n, dtype=torch.bool)), float("-inf"))
    z = torch.stack([torch.from_numpy(dropout_keep(seed_f, 0, 0, h, H, np.arange(n), n, p)) for h in range(H)])[None]
    ref = torch.einsum("bhij,bjhd->bihd", torch.softmax(s, dim=-1) * z / (1 - p), v2)
    ref.backward(do)
    assert torch.allclose(out, ref, atol=1e-12)
    for a, b in ((q.grad, q2.grad), (k.grad, k2.grad), (v.grad, v2.grad)):
        assert torch.allclose(a, b, atol=1e-12)


def test_dropout_with_two_sided_window_reaches_both_calls(oracle_backend):
    """dropout_p with a non-causal window_size=(left, right): the forward and the backward get the same
    seed and both window entries."""
    g = torch.Generator().manual_seed(13)
    q, k, v = (torch.randn(1, 12, 2, 4, generator=g, dtype=torch.float64, requires_grad=True) for _ in range(3))
    itf.flash_attn_func(q, k, v, dropout_p=0.2, window_size=(3, 2)).sum().backward()
    (f, bw) = oracle_backend
    assert f[0] == "fwd" and bw[0] == "bwd"
    assert f[1:] == bw[1:] and f[3] == 3 and f[4] == 0.2 and f[6] == 0 and f[7] == 2
    assert all(t.grad is not None and torch.isfinite(t.grad).all() for t in (q, k, v))


@pytest.fixture
def packed_backend(monkeypatch):
    """forward_varlen / backward_varlen replaced by the oracle run on each sequence (CPU tensors)."""
    calls = []

    def seqs(cu):
        c = cu.tolist()
        return [(c[i], c[i + 1]) for i in range(len(c) - 1)]

    def fwd(q, k, v, cu_q, cu_k, max_q, max_k, scale, causal, wl, window_right=-1, dropout_p=0.0, seed=None,
            offset=0):
        calls.append(("fwd", max_q, max_k, scale, causal, wl, window_right, dropout_p))
        out = torch.zeros(q.shape, dtype=torch.float64)
        lse = torch.zeros((q.shape[1], q.shape[0]), dtype=torch.float64)
        for (q0, q1), (k0, k1) in zip(seqs(cu_q), seqs(cu_k)):
            o, l = attention_ref(q[None, q0:q1].detach().numpy(), k[None, k0:k1].detach().numpy(),
                                 v[None, k0:k1].detach().numpy(), scale, causal, wl, window_right=window_right)
            out[q0:q1], lse[:, q0:q1] = torch.from_numpy(o[0]), torch.from_numpy(l[0])
        return out, lse

    def bwd(q, k, v, out, lse, dout, cu_q, cu_k, max_q, max_k, scale, causal, wl, window_right=-1, dropout_p=0.0,
            seed=None, offset=0):
        calls.append(("bwd", max_q, max_k, scale, causal, wl, window_right, dropout_p))
        grads = [torch.zeros(t.shape, dtype=torch.float64) for t in (q, k, v)]
        for (q0, q1), (k0, k1) in zip(seqs(cu_q), seqs(cu_k)):
            g = attention_backward_ref(q[None, q0:q1].detach().numpy(), k[None, k0:k1].detach().numpy(),
                                       v[None, k0:k1].detach().numpy(), dout[None, q0:q1].numpy(), scale, causal, wl,
                                       window_right=window_right)
            grads[0][q0:q1] = torch.from_numpy(g[0][0])
            grads[1][k0:k1] = torch.from_numpy(g[1][0])
            grads[2][k0:k1] = torch.from_numpy(g[2][0])
        return tuple(grads)

    monkeypatch.setattr(itf, "forward_varlen", fwd)
    monkeypatch.setattr(itf, "backward_varlen", bwd)
    return calls


@pytest.mark.parametrize("causal, window", [(True, (-1, -1)), (False, (2, 3))])
def test_packed_call_gradients_match_torch_autograd(packed_backend, causal, window):
    """flash_attn_varlen_func: gradients of the packed call equal torch autograd's of plain attention run
    on each sequence alone, and the options reach the packed forward and backward unchanged."""
    g = torch.Generator().manual_seed(21)
    lens = [5, 1, 8]
    total = sum(lens)
    q, k, v = (torch.randn(total, 2, 4, generator=g, dtype=torch.float64, requires_grad=True) for _ in range(3))
    do = torch.randn(total, 2, 4, generator=g, dtype=torch.float64)
    cu = torch.tensor([0, 5, 6, 14], dtype=torch.int32)
    out = itf.flash_attn_varlen_func(q, k, v, cu, cu, 8, 8, causal=causal, window_size=window)
    out.backward(do)
    wl, wr = window[0], (-1 if causal else window[1])
    q2, k2, v2 = (t.detach().clone().requires_grad_() for t in (q, k, v))
    refs = []
    for a, b in ((0, 5), (5, 6), (6, 14)):
        refs.append(_plain_attention(q2[None, a:b], k2[None, a:b], v2[None, a:b], 0.5, causal, wl, wr)[0])
    torch.cat(refs).backward(do)
    assert torch.allclose(out, torch.cat(refs), atol=1e-12)
    for a_, b_ in ((q.grad, q2.grad), (k.grad, k2.grad), (v.grad, v2.grad)):
        assert torch.allclose(a_, b_, atol=1e-12)
    assert packed_backend == [("fwd", 8, 8, 0.5, causal, wl, wr, 0.0), ("bwd", 8, 8, 0.5, causal, wl, wr, 0.0)]
