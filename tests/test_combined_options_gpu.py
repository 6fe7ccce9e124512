"""Options combined through fa_fwd_ex / fa_bwd_ex, against the fp64 oracle.

The pages' flash_attn_func takes dropout_p, causal and window_size=(left,
right) together (Flash Attention | Hermes Skill, Workflow 2, Steps 2-3).
Here dropout meets a non-causal two-sided window, and packed sequences meet
the right window and dropout.  Forward outputs are compared element by
element within the usual tolerances, gradients under the per-element bounds
of tests/oracle_cmp.backward_bounds.  A packed sequence b draws its dropout
keep bits as batch b of a padded batch would: the oracle sees it as the last
batch of a padded batch of b + 1 (the earlier batches zero).
"""

import math

import numpy as np
import pytest
import torch

from exact_attention_136_b200 import (_lib, backward, backward_varlen, device_status, forward, forward_varlen,
                                      inputs)
from oracle import attention_backward_ref, attention_ref
from tests.oracle_cmp import TOL_LSE, TOL_O, backward_bounds, compare

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)
U = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    _lib.lib()


def _f64(t):
    return t.detach().double().cpu().numpy()


def _check_grads(got, ref, bounds, dt, what):
    for name, g, want, bnd in zip(("dq", "dk", "dv"), got, ref, bounds):
        assert np.all(np.isfinite(g)), f"{what} {name}"
        err = np.abs(g - want)
        worst = float(np.max(err / (bnd + U[dt] * np.abs(want) + 1e-6))) if err.size else 0.0
        assert worst <= 1.0, f"{what} {name}: error exceeds its bound by x{worst:.3f}"


@pytest.mark.parametrize("B,n,H,h_kv,D,dt,wl,wr,p", [
    (1, 700, 2, 2, 128, "bf16", 256, 256, 0.1),     # the pages' window with the pages' dropout
    (2, 390, 4, 2, 64, "fp16", -1, 70, 0.3),
])
def test_dropout_with_a_two_sided_window(B, n, H, h_kv, D, dt, wl, wr, p):
    seed, offset = 0x5EED5EED12345678, 77
    qkv = inputs.make_qkv(B, n, n, H, D, dt, seeds=(710, 711, 712), h_kv=h_kv)
    do = inputs.make_qkv(B, n, n, H, D, dt, seeds=(713, 714, 715)).q
    q, k, v, g = (t.to(DEV) for t in (qkv.q, qkv.k, qkv.v, do))
    scale = 1.0 / math.sqrt(D)
    out, lse = forward(q, k, v, scale, False, wl, dropout_p=p, seed=seed, offset=offset, window_right=wr)
    dq, dk, dv = backward(q, k, v, out, lse, g, scale, False, wl, dropout_p=p, seed=seed, offset=offset,
                          window_right=wr)
    torch.cuda.synchronize()
    assert device_status()[0] == 0
    ref_o, ref_l = attention_ref(_f64(q), _f64(k), _f64(v), scale, False, wl, dropout_p=p, seed=seed,
                                 offset=offset, window_right=wr)
    d_o, d_l = compare(out, lse, ref_o, ref_l)
    assert d_o <= TOL_O[dt] and d_l <= TOL_LSE, (d_o, d_l)
    args = (_f64(q), _f64(k), _f64(v), _f64(g))
    ref = attention_backward_ref(*args, scale, False, wl, dropout_p=p, seed=seed, offset=offset, window_right=wr)
    bounds = backward_bounds(*args, _f64(out), _f64(lse), scale, False, wl, U[dt], dropout_p=p, seed=seed,
                             offset=offset, window_right=wr)
    _check_grads((_f64(dq), _f64(dk), _f64(dv)), ref, bounds, dt, "padded")


def _packed(lens, H, h_kv, D, dt, seed):
    t = int(sum(lens))
    qkv = inputs.make_qkv(1, t, t, H, D, dt, seeds=(seed, seed + 1, seed + 2), h_kv=h_kv)
    do = inputs.make_qkv(1, t, t, H, D, dt, seeds=(seed + 3, seed + 4, seed + 5)).q
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    return qkv.q[0], qkv.k[0], qkv.v[0], do[0], cu


def _as_last_batch(x, b):
    """[n, H, D] -> [b + 1, n, H, D] with x as batch b and zeros before it."""
    z = np.zeros((b + 1,) + x.shape)
    z[b] = x
    return z


@pytest.mark.parametrize("lens,H,h_kv,D,dt,causal,wl,wr,p", [
    ([1, 300, 128, 517], 2, 2, 128, "bf16", False, 64, 100, 0.0),    # packed + right window
    ([700, 5, 256], 4, 2, 64, "fp16", True, -1, -1, 0.2),            # packed + dropout
    ([200, 333, 1], 2, 1, 128, "bf16", False, 40, 40, 0.1),          # all three
])
def test_packed_sequences_with_window_and_dropout(lens, H, h_kv, D, dt, causal, wl, wr, p):
    seed, offset = 99, 5
    q, k, v, do, cu = _packed(lens, H, h_kv, D, dt, 720 + len(lens))
    qd, kd, vd, dod, cud = (t.contiguous().to(DEV) for t in (q, k, v, do, cu))
    scale = 1.0 / math.sqrt(D)
    kw = dict(window_right=wr, dropout_p=p, seed=seed if p else None, offset=offset)
    out, lse = forward_varlen(qd, kd, vd, cud, cud, max(lens), max(lens), scale, causal, wl, **kw)
    dq, dk, dv = backward_varlen(qd, kd, vd, out, lse, dod, cud, cud, max(lens), max(lens), scale, causal, wl, **kw)
    torch.cuda.synchronize()
    assert device_status()[0] == 0
    o_all, l_all = _f64(out), _f64(lse)
    gq, gk, gv = _f64(dq), _f64(dk), _f64(dv)
    for b in range(len(lens)):
        r0, r1 = int(cu[b]), int(cu[b + 1])
        args = [_as_last_batch(_f64(t[r0:r1]), b) for t in (q, k, v, do)]
        okw = dict(dropout_p=p, seed=seed, offset=offset, window_right=wr)
        ref_o, ref_l = attention_ref(*args[:3], scale, causal, wl, **okw)
        d_o = float(np.max(np.abs(o_all[r0:r1] - ref_o[b])))
        assert d_o <= TOL_O[dt], f"sequence {b}: max|dO| {d_o:.3e}"
        got_l, want_l = l_all[:, r0:r1], ref_l[b]
        assert np.array_equal(np.isfinite(got_l), np.isfinite(want_l)), f"sequence {b}: -inf pattern"
        fin = np.isfinite(want_l)
        if fin.any():
            assert float(np.max(np.abs(got_l[fin] - want_l[fin]))) <= TOL_LSE, f"sequence {b}: LSE"
        ref = attention_backward_ref(*args, scale, causal, wl, **okw)
        o_used = _as_last_batch(o_all[r0:r1], b)
        l_used = np.zeros((b + 1, H, r1 - r0))
        l_used[b] = l_all[:, r0:r1]
        bounds = backward_bounds(*args, o_used, l_used, scale, causal, wl, U[dt], **okw)
        _check_grads((gq[r0:r1], gk[r0:r1], gv[r0:r1]), [x[b] for x in ref], [x[b] for x in bounds], dt,
                     f"sequence {b}")
