"""Dropout on the GPU against the fp64 oracle.

The keep bits are compared bit for bit: with Q = 0 every visible key of a
row gets the same weight 1 / n, and with V_j = e_(j mod D) under a causal
window of D - 1 keys each output column holds exactly one key, so O is
nonzero exactly where that key was kept.  Outputs on random inputs are
compared with the oracle's dropout forward within the usual tolerances, and
the gradients element by element under the derived bounds.
"""

import math

import numpy as np
import pytest
import torch

from exact_attention_136_b200 import _lib, backward, device_status, forward, inputs
from oracle import attention_backward_ref, attention_ref, dropout_keep
from tests.oracle_cmp import TOL_LSE, TOL_O, backward_bounds, compare

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
U = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    _lib.lib()


@pytest.mark.parametrize("B,n,H,h_kv,D,dt,p,seed,offset", [
    (2, 700, 3, 3, 128, "bf16", 0.1, 0x0123456789ABCDEF, 0),
    (1, 1000, 4, 2, 64, "fp16", 0.5, 7, 12345),
    (1, 257, 2, 1, 128, "fp16", 0.9, (1 << 63) + 5, 0xFFFFFFFF),
])
def test_keep_bits_match_the_oracle_bit_for_bit(B, n, H, h_kv, D, dt, p, seed, offset):
    tdt = torch.float16 if dt == "fp16" else torch.bfloat16
    q = torch.zeros((B, n, H, D), dtype=tdt, device=DEV)
    k = inputs.make_qkv(B, n, n, h_kv, D, dt, seeds=(5, 6, 7)).k.to(DEV)
    eye = torch.eye(D, dtype=tdt)
    v = eye[torch.arange(n) % D][None, :, None, :].expand(B, n, h_kv, D).contiguous().to(DEV)
    wl = D - 1
    out, lse = forward(q, k, v, 1.0, True, wl, dropout_p=p, seed=seed, offset=offset)
    torch.cuda.synchronize()
    assert device_status()[0] == 0
    o = out.float().cpu().numpy()
    for b in range(B):
        for h in range(H):
            z = dropout_keep(seed, offset, b, h, H, np.arange(n), n, p)
            for i in range(n):
                keys = np.arange(max(0, i - wl), i + 1)
                want = np.zeros(D, dtype=bool)
                want[keys % D] = z[i, keys]
                got = o[b, i, h] != 0
                assert np.array_equal(got, want), f"b={b} h={h} row {i}: keep bits differ"
                # kept keys carry 1 / (n_i (1 - p)) each
                val = 1.0 / (len(keys) * (1.0 - p))
                assert np.allclose(o[b, i, h][want], val, rtol=2 * U[dt])
    # LSE is the softmax normaliser, untouched by dropout: ln(n_i)
    n_vis = np.minimum(np.arange(n) + 1, D)
    assert np.allclose(lse.cpu().numpy(), np.log(n_vis)[None, None, :], atol=1e-5)


@pytest.mark.parametrize("B,n_q,n_k,H,h_kv,D,dt,causal,wl,p", [
    (1, 384, 384, 2, 2, 128, "bf16", True, -1, 0.1),
    (2, 300, 300, 4, 2, 64, "fp16", False, -1, 0.3),
    (1, 513, 1025, 2, 1, 128, "fp16", True, 200, 0.5),
    (1, 100, 260, 2, 2, 64, "bf16", False, 50, 0.2),
])
def test_dropout_forward_matches_oracle(B, n_q, n_k, H, h_kv, D, dt, causal, wl, p):
    qkv = inputs.make_qkv(B, n_q, n_k, H, D, dt, seeds=(41 + n_q, 42, 43), h_kv=h_kv)
    q, k, v = qkv.q.to(DEV), qkv.k.to(DEV), qkv.v.to(DEV)
    scale = 1.0 / math.sqrt(D)
    out, lse = forward(q, k, v, scale, causal, wl, dropout_p=p, seed=99, offset=3)
    torch.cuda.synchronize()
    assert device_status()[0] == 0
    f64 = lambda t: t.double().numpy()
    ref_o, ref_l = attention_ref(f64(qkv.q), f64(qkv.k), f64(qkv.v), scale, causal, wl, dropout_p=p, seed=99,
                                 offset=3)
    d_o, d_l = compare(out, lse, ref_o, ref_l)
    assert d_o <= TOL_O[dt] and d_l <= TOL_LSE, (d_o, d_l)


def test_dropout_is_repeatable_and_offset_changes_the_mask():
    qkv = inputs.make_qkv(1, 512, 512, 2, 128, "bf16", seeds=(1, 2, 3))
    q, k, v = qkv.q.to(DEV), qkv.k.to(DEV), qkv.v.to(DEV)
    a, _ = forward(q, k, v, None, True, dropout_p=0.25, seed=11, offset=0)
    b, _ = forward(q, k, v, None, True, dropout_p=0.25, seed=11, offset=0)
    c, _ = forward(q, k, v, None, True, dropout_p=0.25, seed=11, offset=1)
    d, _ = forward(q, k, v, None, True, dropout_p=0.25, seed=12, offset=0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert not torch.equal(a, c) and not torch.equal(a, d)


@pytest.mark.parametrize("B,n_q,n_k,H,h_kv,D,dt,causal,wl,p", [
    (1, 256, 256, 2, 2, 128, "bf16", True, -1, 0.2),
    (1, 300, 411, 2, 1, 64, "fp16", False, -1, 0.5),
    (2, 384, 384, 4, 2, 128, "fp16", True, 130, 0.1),
])
def test_dropout_backward_matches_oracle(B, n_q, n_k, H, h_kv, D, dt, causal, wl, p):
    qkv = inputs.make_qkv(B, n_q, n_k, H, D, dt, seeds=(61, 62, 63), h_kv=h_kv)
    g = inputs.make_qkv(B, n_q, n_q, H, D, dt, seeds=(64, 65, 66)).q
    scale = 1.0 / math.sqrt(D)
    q, k, v, do = (t.to(DEV) for t in (qkv.q, qkv.k, qkv.v, g))
    out, lse = forward(q, k, v, scale, causal, wl, dropout_p=p, seed=2024, offset=9)
    dq, dk, dv = backward(q, k, v, out, lse, do, scale, causal, wl, dropout_p=p, seed=2024, offset=9)
    torch.cuda.synchronize()
    assert device_status()[0] == 0
    f64 = lambda t: t.detach().double().cpu().numpy()
    ref = attention_backward_ref(f64(q), f64(k), f64(v), f64(do), scale, causal, wl, dropout_p=p, seed=2024,
                                 offset=9)
    bounds = backward_bounds(f64(q), f64(k), f64(v), f64(do), f64(out), f64(lse), scale, causal, wl, U[dt],
                             dropout_p=p, seed=2024, offset=9)
    for name, got, want, bnd in zip(("dq", "dk", "dv"), (dq, dk, dv), ref, bounds):
        got = f64(got)
        assert np.all(np.isfinite(got)), name
        err = np.abs(got - want)
        allowed = bnd + U[dt] * np.abs(want) + 1e-6
        worst = float(np.max(err / allowed))
        assert worst <= 1.0, f"{name}: error exceeds its bound by x{worst:.3f}"


def test_dropout_arguments_validated():
    f = _lib.lib().fa_fwd_dropout
    A = 1 << 20
    for bad_p in (-0.1, 1.0, float("nan")):
        assert f(A, A, A, A, None, 1, 16, 16, 2, 2, 64, 0.1, 0, -1, _lib.FA_FP16, bad_p, 1, 0, None) == _lib.FA_ERR_ARG
    assert f(A, A, A, A, None, 1, 16, 16, 2, 2, 128, 0.1, 0, -1, _lib.FA_E4M3, 0.1, 1, 0, None) == \
        _lib.FA_ERR_UNSUPPORTED
