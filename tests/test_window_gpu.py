"""Two-sided local attention on the GPU (fa_fwd_window / fa_bwd_window).

The pages' sliding-window call passes window_size=(256, 256): keys up to 256
positions before and after the query (Flash Attention | Hermes Skill,
Workflow 2, Step 3).  Forward outputs are compared with the fp64 oracle
element by element (sampled rows at the full size), the backward under the
per-element bounds of tests/oracle_cmp.backward_bounds, and the special
cases that must reproduce another entry point do so bit for bit: a right
window of 0 is causal, one reaching past the last key is no bound.
"""

import math

import numpy as np
import pytest
import torch

from exact_attention_136_b200 import _lib, backward, device_status, forward, forward_fp8, inputs
from oracle import attention_backward_ref
from tests.oracle_cmp import TOL_LSE, TOL_O, backward_bounds, compare, oracle

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda", 0)
U = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    _lib.lib()


def _fwd(qkv, scale, causal, wl, wr):
    q, k, v = qkv.q.to(DEV), qkv.k.to(DEV), qkv.v.to(DEV)
    if q.dtype == torch.float8_e4m3fn:
        out, lse = forward_fp8(q, k, v, qkv.q_descale, qkv.k_descale, qkv.v_descale, scale, causal, wl,
                               window_right=wr)
    else:
        out, lse = forward(q, k, v, scale, causal, wl, window_right=wr)
    torch.cuda.synchronize()
    rc, flags = device_status()
    assert rc == 0, f"device status {rc} flags {flags}"
    return out, lse


FWD_CASES = [
    # B, N_q, N_k, H, H_kv, D, dtype, window_left, window_right
    (1, 1000, 1000, 2, 2, 128, "bf16", 256, 256),    # the pages' window, ragged tail
    (1, 600, 600, 2, 2, 64, "fp16", -1, 100),        # right bound only
    (2, 300, 700, 4, 2, 128, "fp16", 50, 130),       # N_k > N_q, grouped K/V heads
    (1, 700, 300, 2, 1, 64, "bf16", 40, 0),          # rows past N_k + 40 see no key
    (1, 513, 513, 2, 2, 128, "e4m3", 256, 256),
    (1, 384, 384, 1, 1, 128, "bf16", 0, 5),          # a band inside every tile
    (1, 1, 300, 1, 1, 64, "bf16", -1, 3),
    (1, 300, 1, 1, 1, 128, "fp16", 2, 7),
    (1, 1030, 1030, 2, 2, 64, "bf16", 127, 129),     # bounds one off the tile edges
]


@pytest.mark.parametrize("B,n_q,n_k,H,h_kv,D,dt,wl,wr", FWD_CASES)
def test_window_forward_matches_oracle(B, n_q, n_k, H, h_kv, D, dt, wl, wr):
    qkv = inputs.make_qkv(B, n_q, n_k, H, D, dt, seeds=(610, 611, 612), h_kv=h_kv)
    scale = 1.0 / math.sqrt(D)
    out, lse = _fwd(qkv, scale, False, wl, wr)
    ref_o, ref_l = oracle(qkv, scale, False, wl, window_right=wr)
    d_o, d_l = compare(out, lse, ref_o, ref_l)
    assert d_o <= TOL_O[dt], f"max|dO| {d_o:.3e} > {TOL_O[dt]}"
    assert d_l <= TOL_LSE, f"max|dLSE| {d_l:.3e} > {TOL_LSE}"


def test_window_forward_full_size_sampled_rows():
    """B=2, H=16, N=8192, D=128 bf16 with window_size=(256, 256): sampled rows
    (tile edges, the first and last rows, random rows) of every (batch, head)."""
    B, n, H, D = 2, 8192, 16, 128
    qkv = inputs.make_qkv(B, n, n, H, D, "bf16", seeds=(620, 621, 622))
    scale = 1.0 / math.sqrt(D)
    out, lse = _fwd(qkv, scale, False, 256, 256)
    rng = np.random.default_rng(5)
    rows = sorted(set([0, 1, 127, 128, 255, 256, 257, 383, 4095, 4096, n - 257, n - 129, n - 1]
                      + rng.integers(0, n, 12).tolist()))
    ref_o, ref_l = oracle(qkv, scale, False, 256, rows=rows, window_right=256)
    d_o, d_l = compare(out, lse, ref_o, ref_l, rows=rows)
    assert d_o <= TOL_O["bf16"] and d_l <= TOL_LSE, (d_o, d_l)


@pytest.mark.parametrize("dt,D,wl", [("bf16", 128, -1), ("fp16", 64, 100), ("e4m3", 128, 37)])
def test_right_window_zero_is_causal_bit_for_bit(dt, D, wl):
    qkv = inputs.make_qkv(2, 777, 777, 3, D, dt, seeds=(630, 631, 632))
    o1, l1 = _fwd(qkv, 0.11, False, wl, 0)
    o2, l2 = _fwd(qkv, 0.11, True, wl, -1)
    o3, l3 = _fwd(qkv, 0.11, True, wl, 256)    # causal hides every later key whatever the right window says
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(o3, o2) and torch.equal(l3, l2)


def test_right_window_past_the_last_key_is_no_bound():
    qkv = inputs.make_qkv(1, 500, 640, 2, 128, "bf16", seeds=(640, 641, 642))
    o1, l1 = _fwd(qkv, 0.09, False, 64, 640)
    o2, l2 = _fwd(qkv, 0.09, False, 64, -1)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def _bwd_check(B, n_q, n_k, H, h_kv, D, dt, wl, wr, seed=0):
    qkv = inputs.make_qkv(B, n_q, n_k, H, D, dt, seeds=(650 + seed, 651 + seed, 652 + seed), h_kv=h_kv)
    do = inputs.make_qkv(B, n_q, n_q, H, D, dt, seeds=(653 + seed, 654 + seed, 655 + seed)).q
    scale = 1.0 / math.sqrt(D)
    q, k, v, g = (t.to(DEV) for t in (qkv.q, qkv.k, qkv.v, do))
    out, lse = forward(q, k, v, scale, False, wl, window_right=wr)
    dq, dk, dv = backward(q, k, v, out, lse, g, scale, False, wl, window_right=wr)
    torch.cuda.synchronize()
    rc, flags = device_status()
    assert rc == 0, f"device status {rc} flags {flags}"
    f64 = lambda t: t.detach().double().cpu().numpy()
    ref = attention_backward_ref(f64(q), f64(k), f64(v), f64(g), scale, False, wl, window_right=wr)
    bounds = backward_bounds(f64(q), f64(k), f64(v), f64(g), f64(out), f64(lse), scale, False, wl, U[dt],
                             window_right=wr)
    for name, got, want, bnd in zip(("dq", "dk", "dv"), (dq, dk, dv), ref, bounds):
        got = f64(got)
        assert np.all(np.isfinite(got)), name
        err = np.abs(got - want)
        allowed = bnd + U[dt] * np.abs(want) + 1e-6
        worst = float(np.max(err / allowed)) if err.size else 0.0
        assert worst <= 1.0, f"{name}: error exceeds its bound by x{worst:.3f}"
    return dq, dk, dv


BWD_CASES = [
    # B, N_q, N_k, H, H_kv, D, dtype, window_left, window_right
    (1, 520, 520, 2, 2, 128, "bf16", 130, 130),
    (1, 400, 400, 2, 1, 64, "fp16", -1, 70),
    (1, 1000, 1000, 1, 1, 128, "bf16", 256, 256),
    (1, 650, 300, 4, 2, 64, "bf16", 50, 0),
    (1, 384, 384, 2, 2, 128, "fp16", 0, 3),
]


@pytest.mark.parametrize("B,n_q,n_k,H,h_kv,D,dt,wl,wr", BWD_CASES)
def test_window_backward_matches_oracle(B, n_q, n_k, H, h_kv, D, dt, wl, wr):
    _bwd_check(B, n_q, n_k, H, h_kv, D, dt, wl, wr)


def test_window_backward_unseen_keys_get_zero_gradients():
    # N_k > N_q + window_right: keys 300 + 200 = 500 .. 649 are never seen
    _, dk, dv = _bwd_check(1, 300, 650, 2, 2, 128, "fp16", 60, 200, seed=3)
    assert torch.count_nonzero(dk[:, 500:]) == 0 and torch.count_nonzero(dv[:, 500:]) == 0
    assert torch.count_nonzero(dk[:, 499]) > 0


def test_window_rejected_combinations():
    q = torch.zeros((1, 128, 2, 64), device=DEV, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        forward(q, q, q, 0.1, False, -1, window_right=-2)
    with pytest.raises(ValueError):
        forward(q, q, q, 0.1, False, -1, window_right=4, num_splits=2)
    with pytest.raises(ValueError):
        forward(q, q, q, 0.1, False, -1, window_right=4, attn_mask=torch.ones(128, 128, dtype=torch.bool,
                                                                              device=DEV))


def test_right_window_with_automatic_slices_keeps_the_window():
    """num_splits=0 (pick slices automatically) must not drop the right window: few queries against
    many keys would otherwise take the key-range-slice path, which has no right bound."""
    qkv = inputs.make_qkv(1, 128, 4096, 2, 128, "bf16", seeds=(660, 661, 662))
    q, k, v = qkv.q.to(DEV), qkv.k.to(DEV), qkv.v.to(DEV)
    o1, l1 = forward(q, k, v, 0.1, False, -1, window_right=300, num_splits=0)
    o2, l2 = forward(q, k, v, 0.1, False, -1, window_right=300)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    ref_o, ref_l = oracle(qkv, 0.1, False, -1, window_right=300)
    d_o, d_l = compare(o1, l1, ref_o, ref_l)
    assert d_o <= TOL_O["bf16"] and d_l <= TOL_LSE, (d_o, d_l)
