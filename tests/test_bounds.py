"""The error bounds the backward parity tests use, checked against the
backward's rounding steps emulated in numpy (torch casts round to nearest)."""

import math

import numpy as np
import torch

from exact_attention_136_b200 import inputs
from oracle import attention_ref


def _emulated_backward(q, k, v, do, o_used, scale, causal, dt):
    """The CUDA backward's arithmetic in numpy: P recomputed from the exact
    LSE, row term from o_used, P and dS rounded to the 16-bit type, fp64
    sums otherwise (one batch, heads equal)."""
    tdt = torch.float16 if dt == "fp16" else torch.bfloat16
    rnd = lambda x: torch.from_numpy(np.ascontiguousarray(x)).to(tdt).double().numpy()
    _, _, probs = attention_ref(q, k, v, scale, causal, -1, return_probs=True)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    group = q.shape[2] // k.shape[2]
    for h in range(q.shape[2]):
        hk = h // group
        p = probs[0, h]
        g = do[0, :, h]
        delta = (g * o_used[0, :, h]).sum(axis=1)
        ds = p * (g @ v[0, :, hk].T - delta[:, None])
        dv[0, :, hk] += rnd(p).T @ g
        dk[0, :, hk] += scale * rnd(ds).T @ q[0, :, h]
        dq[0, :, h] = scale * rnd(ds) @ k[0, :, hk]
    return dq, dk, dv


def test_backward_bounds_cover_emulated_rounding():
    from oracle import attention_backward_ref
    from tests.oracle_cmp import backward_bounds
    for dt, u, causal, h_kv in (("bf16", 2.0 ** -8, True, 2), ("fp16", 2.0 ** -11, False, 2),
                                ("bf16", 2.0 ** -8, True, 1)):
        qkv = inputs.make_qkv(1, 200, 200, 2, 32, dt, seeds=(51, 52, 53), h_kv=h_kv)
        do = inputs.make_qkv(1, 200, 200, 2, 32, dt, seeds=(54, 55, 56)).q
        f = lambda t: t.double().numpy()
        q, k, v, g = f(qkv.q), f(qkv.k), f(qkv.v), f(do)
        o, lse = attention_ref(q, k, v, 0.2, causal, -1)
        tdt = torch.float16 if dt == "fp16" else torch.bfloat16
        o_used = torch.from_numpy(o).to(tdt).double().numpy()   # the forward's rounded output
        got = _emulated_backward(q, k, v, g, o_used, 0.2, causal, dt)
        want = attention_backward_ref(q, k, v, g, 0.2, causal, -1)
        bounds = backward_bounds(q, k, v, g, o_used, lse, 0.2, causal, -1, u)
        ratios = []
        for a, w, bnd in zip(got, want, bounds):
            assert np.all(np.abs(a - w) <= bnd + 1e-12), float(np.max(np.abs(a - w) - bnd))
            ratios.append(float(np.max(np.abs(a - w) / (bnd + 1e-300))))
        # not vacuous: the worst element of each gradient uses a fair share of its bound
        assert min(ratios) > 0.05, ratios
