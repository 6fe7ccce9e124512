"""Packed variable-length batches (fa_fwd_varlen) against the fp64 oracle
run on each sequence alone, and against the padded-batch forward."""

import math

import numpy as np
import pytest
import torch

from exact_attention_136_b200 import _lib, device_status, forward, forward_varlen, inputs
from oracle import attention_ref
from tests.oracle_cmp import TOL_LSE, TOL_O

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    _lib.lib()


def _packed(lens_q, lens_k, H, h_kv, D, dt, seed):
    tq, tk = int(sum(lens_q)), int(sum(lens_k))
    qkv = inputs.make_qkv(1, max(tq, 1), max(tk, 1), H, D, dt, seeds=(seed, seed + 1, seed + 2), h_kv=h_kv)
    q, k, v = qkv.q[0, :tq], qkv.k[0, :tk], qkv.v[0, :tk]
    cu_q = torch.tensor(np.concatenate([[0], np.cumsum(lens_q)]), dtype=torch.int32)
    cu_k = torch.tensor(np.concatenate([[0], np.cumsum(lens_k)]), dtype=torch.int32)
    return qkv, q, k, v, cu_q, cu_k


CASES = [
    # lens_q, lens_k, H, H_kv, D, dtype, causal, window_left
    ([1, 300, 128, 517, 64], [1, 300, 128, 517, 64], 2, 2, 128, "bf16", True, -1),
    ([700, 5, 256, 1000], [700, 5, 256, 1000], 4, 2, 64, "fp16", False, -1),
    ([129, 0, 333, 1], [200, 17, 0, 90], 2, 1, 128, "fp16", False, -1),
    ([600, 255, 1024], [600, 255, 1024], 2, 2, 128, "bf16", True, 100),
    ([384, 77, 1500], [384, 77, 1500], 2, 2, 128, "e4m3", True, -1),
]


@pytest.mark.parametrize("lens_q,lens_k,H,h_kv,D,dt,causal,wl", CASES)
def test_varlen_matches_oracle_per_sequence(lens_q, lens_k, H, h_kv, D, dt, causal, wl):
    qkv, q, k, v, cu_q, cu_k = _packed(lens_q, lens_k, H, h_kv, D, dt, 300 + sum(lens_q))
    scale = 1.0 / math.sqrt(D)
    out, lse = forward_varlen(q.contiguous().to(DEV), k.contiguous().to(DEV), v.contiguous().to(DEV), cu_q.to(DEV),
                              cu_k.to(DEV), max(lens_q), max(lens_k), scale, causal, wl,
                              descales=(qkv.q_descale, qkv.k_descale, qkv.v_descale))
    torch.cuda.synchronize()
    assert device_status()[0] == 0
    o, l = out.float().cpu().numpy(), lse.cpu().numpy()
    assert np.all(np.isfinite(o)), "rows left unwritten"
    f64 = lambda t, d: (t.to(torch.float64) * d).numpy()
    for b in range(len(lens_q)):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        if q1 == q0:
            continue
        ref_o, ref_l = attention_ref(f64(q[None, q0:q1], qkv.q_descale), f64(k[None, k0:k1], qkv.k_descale),
                                     f64(v[None, k0:k1], qkv.v_descale), scale, causal, wl)
        d_o = float(np.max(np.abs(o[q0:q1] - ref_o[0])))
        assert d_o <= TOL_O[dt], f"sequence {b}: max|dO| {d_o:.3e}"
        got_l, want_l = l[:, q0:q1], ref_l[0]
        assert np.array_equal(np.isfinite(got_l), np.isfinite(want_l)), f"sequence {b}: -inf pattern"
        fin = np.isfinite(want_l)
        if fin.any():
            assert float(np.max(np.abs(got_l[fin] - want_l[fin]))) <= TOL_LSE, f"sequence {b}: LSE"


def test_equal_lengths_reproduce_the_padded_batch():
    B, n, H, D = 3, 513, 2, 128
    qkv = inputs.make_qkv(B, n, n, H, D, "bf16", seeds=(11, 12, 13))
    q, k, v = qkv.q.to(DEV), qkv.k.to(DEV), qkv.v.to(DEV)
    ref_o, ref_l = forward(q, k, v, 0.09, True)
    cu = torch.arange(0, (B + 1) * n, n, dtype=torch.int32, device=DEV)
    out, lse = forward_varlen(q.reshape(B * n, H, D), k.reshape(B * n, H, D), v.reshape(B * n, H, D), cu, cu, n, n,
                              0.09, True)
    torch.cuda.synchronize()
    assert torch.equal(out.reshape(B, n, H, D), ref_o)
    # LSE: [H, total] against [B, H, N]
    assert torch.equal(lse.reshape(H, B, n).permute(1, 0, 2), ref_l)


def test_no_keys_at_all():
    lens = [3, 0, 5]
    cu_q = torch.tensor([0, 3, 3, 8], dtype=torch.int32, device=DEV)
    cu_k = torch.zeros(4, dtype=torch.int32, device=DEV)
    q = torch.randn(8, 2, 64, device=DEV).to(torch.float16)
    k = torch.zeros(1, 2, 64, device=DEV, dtype=torch.float16)[:0]
    out, lse = forward_varlen(q, k, k, cu_q, cu_k, max(lens), 0, 0.125, False)
    torch.cuda.synchronize()
    assert bool((out == 0).all()) and bool(torch.isinf(lse).all() and (lse < 0).all())


U = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}

BWD_CASES = [
    # lens_q, lens_k, H, H_kv, D, dtype, causal, window_left
    ([1, 300, 128, 517, 64], [1, 300, 128, 517, 64], 2, 2, 128, "bf16", True, -1),
    ([700, 5, 256, 1000], [700, 5, 256, 1000], 4, 2, 64, "fp16", False, -1),
    ([129, 0, 333, 1], [200, 17, 0, 90], 2, 1, 128, "fp16", False, -1),
    ([600, 255, 1024], [600, 255, 1024], 2, 2, 128, "bf16", True, 100),
]


@pytest.mark.parametrize("lens_q,lens_k,H,h_kv,D,dt,causal,wl", BWD_CASES)
def test_varlen_backward_matches_oracle_per_sequence(lens_q, lens_k, H, h_kv, D, dt, causal, wl):
    """fa_bwd_varlen: every sequence's dQ, dK, dV against the oracle's exact
    gradients of that sequence alone, under the per-element bounds of the
    padded backward's tests; a sequence without keys gets dQ = 0, keys
    without queries dK = dV = 0."""
    from exact_attention_136_b200 import backward_varlen
    from oracle import attention_backward_ref
    from tests.oracle_cmp import backward_bounds
    qkv, q, k, v, cu_q, cu_k = _packed(lens_q, lens_k, H, h_kv, D, dt, 700 + sum(lens_q))
    tq = int(sum(lens_q))
    do = inputs.make_qkv(1, max(tq, 1), 1, H, D, dt, seeds=(901, 902, 903)).q[0, :tq]
    scale = 1.0 / math.sqrt(D)
    qd, kd, vd, dod, cq, ck = (t.contiguous().to(DEV) for t in (q, k, v, do, cu_q, cu_k))
    out, lse = forward_varlen(qd, kd, vd, cq, ck, max(lens_q), max(lens_k), scale, causal, wl)
    dq, dk, dv = backward_varlen(qd, kd, vd, out, lse, dod, cq, ck, max(lens_q), max(lens_k), scale, causal, wl)
    torch.cuda.synchronize()
    assert device_status()[0] == 0
    f64 = lambda t: t.detach().double().cpu().numpy()
    gq, gk, gv, o_all, l_all = f64(dq), f64(dk), f64(dv), f64(out), f64(lse)
    for name, g in (("dq", gq), ("dk", gk), ("dv", gv)):
        assert np.all(np.isfinite(g)), f"{name}: rows left unwritten"
    for b in range(len(lens_q)):
        q0, q1 = int(cu_q[b]), int(cu_q[b + 1])
        k0, k1 = int(cu_k[b]), int(cu_k[b + 1])
        if q1 == q0 or k1 == k0:
            # nothing to attend: zero gradients
            assert not gq[q0:q1].any() and not gk[k0:k1].any() and not gv[k0:k1].any(), f"sequence {b}"
            continue
        args = [f64(t)[None] for t in (q[q0:q1], k[k0:k1], v[k0:k1], do[q0:q1])]
        ref = attention_backward_ref(*args, scale, causal, wl)
        bounds = backward_bounds(*args, o_all[None, q0:q1], l_all[None, :, q0:q1], scale, causal, wl, U[dt])
        for name, got, want, bnd in zip(("dq", "dk", "dv"), (gq[q0:q1], gk[k0:k1], gv[k0:k1]), ref, bounds):
            err = np.abs(got - want[0])
            worst = float(np.max(err / (bnd[0] + U[dt] * np.abs(want[0]) + 1e-6)))
            assert worst <= 1.0, f"sequence {b} {name}: error exceeds its bound by x{worst:.3f}"


def test_varlen_backward_equal_lengths_reproduce_the_padded_batch():
    """Equal lengths: the packed backward takes the padded backward's steps in the same order (bit for bit)."""
    from exact_attention_136_b200 import backward, backward_varlen
    B, n, H, h_kv, D = 3, 513, 4, 2, 128
    qkv = inputs.make_qkv(B, n, n, H, D, "bf16", seeds=(21, 22, 23), h_kv=h_kv)
    q, k, v = qkv.q.to(DEV), qkv.k.to(DEV), qkv.v.to(DEV)
    do = inputs.make_qkv(B, n, n, H, D, "bf16", seeds=(24, 25, 26)).q.to(DEV)
    out, lse = forward(q, k, v, 0.09, True)
    ref = backward(q, k, v, out, lse, do, 0.09, True)
    cu = torch.arange(0, (B + 1) * n, n, dtype=torch.int32, device=DEV)
    flat = lambda t: t.reshape(B * n, t.shape[2], D)
    # the packed LSE is [H, total_q]: batch b's rows follow batch b-1's
    lse_p = lse.permute(1, 0, 2).reshape(H, B * n).contiguous()
    got = backward_varlen(flat(q), flat(k), flat(v), flat(out), lse_p, flat(do), cu, cu, n, n, 0.09, True)
    torch.cuda.synchronize()
    for g, r in zip(got, ref):
        assert torch.equal(g, flat(r))


def test_varlen_backward_rejects_bad_sizes():
    from exact_attention_136_b200 import backward_varlen
    t = torch.zeros((256, 2, 64), device=DEV, dtype=torch.float16)
    lse = torch.zeros((2, 256), device=DEV)
    cu = torch.tensor([0, 128, 256], dtype=torch.int32, device=DEV)
    with pytest.raises(_lib.FAError):
        backward_varlen(t, t, t, t, lse, t, cu, cu, 0, 128)       # rows but max_seqlen_q 0
    with pytest.raises(_lib.FAError):
        backward_varlen(t, t, t, t, lse, t, cu, cu, 128, 300)     # longer than the packed keys


def test_packed_call_with_autograd_equals_the_direct_calls():
    """flash_attn_varlen_func (autograd over the packed batch) gives the outputs and gradients of
    forward_varlen / backward_varlen bit for bit."""
    from exact_attention_136_b200 import backward_varlen, flash_attn_varlen_func
    lens_q = [300, 1, 517]
    qkv, q, k, v, cu_q, cu_k = _packed(lens_q, lens_q, 4, 2, 128, "bf16", 880)
    do = inputs.make_qkv(1, sum(lens_q), 1, 4, 128, "bf16", seeds=(884, 885, 886)).q[0].to(DEV)
    qd, kd, vd = (t.contiguous().to(DEV).requires_grad_() for t in (q, k, v))
    cq, ck = cu_q.to(DEV), cu_k.to(DEV)
    out = flash_attn_varlen_func(qd, kd, vd, cq, ck, 517, 517, causal=True, window_size=(100, 0))
    out.backward(do)
    o2, l2 = forward_varlen(qd.detach(), kd.detach(), vd.detach(), cq, ck, 517, 517, 128 ** -0.5, True, 100)
    g2 = backward_varlen(qd.detach(), kd.detach(), vd.detach(), o2, l2, do, cq, ck, 517, 517, 128 ** -0.5, True, 100)
    torch.cuda.synchronize()
    assert torch.equal(out.detach(), o2)
    for got, want in zip((qd.grad, kd.grad, vd.grad), g2):
        assert torch.equal(got, want)
