"""Backward parity: the CUDA backward (through fa_bwd) against the fp64
oracle's exact gradients, element by element, within bounds derived from the
path's arithmetic (tests/oracle_cmp.backward_bounds)."""

import math

import numpy as np
import pytest
import torch

from exact_attention_136_b200 import backward, forward, inputs
from oracle import attention_backward_ref
from tests.oracle_cmp import backward_bounds

pytestmark = pytest.mark.gpu

U = {"fp16": 2.0 ** -11, "bf16": 2.0 ** -8}
DEV = torch.device("cuda", 0)


def _run_and_check(B, n_q, n_k, H, D, dt, causal, wl, seed=0, scale=None, h_kv=0):
    qkv = inputs.make_qkv(B, n_q, n_k, H, D, dt, seeds=(500 + seed, 501 + seed, 502 + seed), h_kv=h_kv or H)
    do = inputs.make_qkv(B, n_q, n_q, H, D, dt, seeds=(503 + seed, 504 + seed, 505 + seed)).q
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    q, k, v, g = (t.to(DEV) for t in (qkv.q, qkv.k, qkv.v, do))
    out, lse = forward(q, k, v, scale, causal, wl)
    dq, dk, dv = backward(q, k, v, out, lse, g, scale, causal, wl)
    torch.cuda.synchronize()
    f64 = lambda t: t.detach().double().cpu().numpy()
    ref = attention_backward_ref(f64(q), f64(k), f64(v), f64(g), scale, causal, wl)
    bounds = backward_bounds(f64(q), f64(k), f64(v), f64(g), f64(out), f64(lse), scale, causal, wl, U[dt])
    worst = {}
    for name, got, want, bnd in zip(("dq", "dk", "dv"), (dq, dk, dv), ref, bounds):
        got = f64(got)
        assert np.all(np.isfinite(got)), name
        # the output's own 16-bit rounding comes on top of the bound
        err = np.abs(got - want)
        allowed = bnd + U[dt] * np.abs(want) + 1e-6
        worst[name] = float(np.max(err / allowed)) if err.size else 0.0
        assert worst[name] <= 1.0, f"{name}: error exceeds its bound by x{worst[name]:.3f}"
    return worst


CASES = [
    # B, N_q, N_k, H, D, dtype, causal, window_left
    (1, 128, 128, 1, 64, "fp16", False, -1),
    (2, 256, 256, 2, 64, "bf16", True, -1),
    (1, 300, 300, 2, 128, "bf16", True, -1),
    (1, 384, 384, 2, 128, "fp16", False, -1),
    (1, 257, 411, 1, 64, "fp16", False, -1),
    (1, 411, 257, 1, 128, "bf16", True, -1),
    (1, 520, 520, 1, 128, "bf16", True, 130),
    (1, 400, 400, 2, 64, "fp16", False, 100),
    (1, 1, 200, 1, 64, "bf16", False, -1),
    (1, 200, 1, 1, 128, "fp16", True, -1),
]


@pytest.mark.parametrize("B,n_q,n_k,H,D,dt,causal,wl", CASES)
def test_backward_matches_oracle(B, n_q, n_k, H, D, dt, causal, wl):
    _run_and_check(B, n_q, n_k, H, D, dt, causal, wl)


def test_backward_bounds_are_tight():
    """The bounds are not vacuous: for a plain case the worst element uses a
    fair share of its bound, and the bound is small against the gradients."""
    worst = _run_and_check(1, 512, 512, 2, 128, "bf16", True, -1, seed=7)
    assert max(worst.values()) > 0.02


def test_backward_many_key_blocks_accumulate_dq():
    # dQ sums over 8 key blocks through the fp32 reductions
    _run_and_check(1, 1024, 1024, 1, 64, "fp16", False, -1, seed=3)


GQA_CASES = [
    # B, N_q, N_k, H, H_kv, D, dtype, causal, window_left
    (1, 256, 256, 4, 2, 128, "bf16", True, -1),
    (2, 300, 300, 4, 1, 64, "fp16", True, -1),
    (1, 411, 257, 6, 2, 128, "fp16", False, -1),
    (1, 520, 520, 4, 4, 64, "bf16", True, 130),
    (1, 384, 384, 8, 2, 128, "bf16", False, 100),
]


@pytest.mark.parametrize("B,n_q,n_k,H,h_kv,D,dt,causal,wl", GQA_CASES)
def test_backward_gqa_matches_oracle(B, n_q, n_k, H, h_kv, D, dt, causal, wl):
    """Grouped K/V heads: dK and dV of a K/V head sum the gradients of every
    query head of its group (fa_bwd_gqa), element by element under the bounds."""
    _run_and_check(B, n_q, n_k, H, D, dt, causal, wl, seed=11, h_kv=h_kv)


def test_backward_rejects_fp8():
    q = torch.zeros((1, 128, 2, 128), device=DEV, dtype=torch.float8_e4m3fn)
    lse = torch.zeros((1, 2, 128), device=DEV)
    with pytest.raises(ValueError):
        backward(q, q, q, q, lse, q)
