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
