"""Host-side FLOP accounting, row sampling and input generation (no GPU)."""

import math

import numpy as np
import torch

from exact_attention_136_b200 import inputs, workloads as W


def test_block_fractions():
    wl = W.WORKLOADS
    assert W.block_fraction(512, 512, False, -1) == 1.0
    # causal N=8192: 64 query blocks, blocks kb <= qb -> 64*65/2 of 64*64
    assert W.block_fraction(8192, 8192, True, -1) == 64 * 65 / 2 / 64 ** 2
    # window 4096 over N=32768: 32 ramp-up blocks then 33 per query block
    c4 = wl["swa4096_b1h32n32768d128_bf16"]
    f = W.block_fraction(c4.n_q, c4.n_k, c4.causal, c4.window_left)
    assert f == (sum(range(1, 33)) + (256 - 32) * 33) / 256 ** 2
    assert abs(W.block_fraction(16384, 16384, True, -1) - 0.5039) < 1e-4


def test_block_fraction_bruteforce_small():
    for n_q, n_k, causal, w in [(300, 300, True, -1), (300, 500, False, 100), (257, 129, True, 5)]:
        nqb, nkb = -(-n_q // 128), -(-n_k // 128)
        hit = 0
        for qb in range(nqb):
            for kb in range(nkb):
                found = False
                for i in range(qb * 128, min(n_q, qb * 128 + 128)):
                    for j in range(kb * 128, min(n_k, kb * 128 + 128)):
                        if (not causal or j <= i) and (w < 0 or j >= i - w):
                            found = True
                            break
                    if found:
                        break
                hit += found
        assert W.block_fraction(n_q, n_k, causal, w) == hit / (nqb * nkb)


def test_flops_headline():
    c3 = W.WORKLOADS[W.HEADLINE]
    assert math.isclose(W.flops(c3), 4 * 4 * 32 * 8192 * 8192 * 128 * 0.5078125)


def test_sample_rows():
    c4 = W.WORKLOADS["swa4096_b1h32n32768d128_bf16"]
    rows = W.sample_rows(c4)
    assert len(rows) == 512 and len(set(rows.tolist())) == 512
    for r in (0, 1, 127, 128, 32767, 4095, 4096, 4097):
        assert r in rows
    assert np.all(np.diff(rows) > 0)
    small = W.WORKLOADS["pr1_b1h8n512d64_fp16"]
    assert np.array_equal(W.sample_rows(small), np.arange(512))


def test_inputs_seeded_and_rounded():
    a = inputs.make_qkv(1, 33, 40, 2, 64, "bf16", seeds=(1, 2, 3))
    b = inputs.make_qkv(1, 33, 40, 2, 64, "bf16", seeds=(1, 2, 3))
    assert a.q.dtype == torch.bfloat16 and a.k.shape == (1, 40, 2, 64)
    assert torch.equal(a.q, b.q) and torch.equal(a.v, b.v)
    # RNE rounding of the fp32 draw
    ref = inputs.randn((1, 33, 2, 64), 1).to(torch.bfloat16)
    assert torch.equal(a.q, ref)


def test_fp8_quantisation():
    x = inputs.make_qkv(1, 64, 64, 2, 128, "e4m3", seeds=(5, 6, 7))
    assert x.q.dtype == torch.float8_e4m3fn
    src = inputs.randn((1, 64, 2, 128), 5)
    assert math.isclose(x.q_descale, float(src.abs().max()) / 448.0, rel_tol=1e-6)
    deq = x.q.to(torch.float64) * x.q_descale
    # e4m3 has 3 mantissa bits: relative error <= 2^-4 for normal values
    err = (deq - src.double()).abs()
    assert float((err / src.double().abs().clamp_min(1e-2 * x.q_descale * 64)).max()) <= 2 ** -4 + 1e-6
    assert float(x.q.to(torch.float32).abs().max()) <= 448.0


def test_binding_roofline_picks_the_exponential_unit_where_it_is_lower():
    """The bench line's roofline: one ex2 per score at 16 per clock per SM, 4 D
    counted FLOP per score; the lower of that and the tensor peak binds."""
    import bench
    tensor, _, _ = bench.measured_peaks("bf16")
    d64 = W.WORKLOADS["b2h8n2048d64_fp16"]
    bound, peak, _ = bench.binding_roofline(d64, 148, 1965.0)
    assert bound == "exp" and abs(peak - 16 * 4 * 64 * 148 * 1965e6 / 1e12) < 1e-6
    c3 = W.WORKLOADS["causal_b4h32n8192d128_bf16"]
    exp128 = 16 * 4 * 128 * 148 * 1965e6 / 1e12
    bound, peak, _ = bench.binding_roofline(c3, 148, 1965.0)
    assert (bound, peak) == (("tensor", tensor) if tensor < exp128 else ("exp", exp128))
    fp8 = W.WORKLOADS["fp8_causal_b2h16n16384d128"]
    bound, peak, _ = bench.binding_roofline(fp8, 148, 1965.0)
    assert peak == min(2 * tensor, exp128)


def test_clock_normalised_value():
    import bench
    assert bench.clock_normalised(1000.0, {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0}) == 1000.0 * 1965.0 / 1500.0
    assert bench.clock_normalised(1000.0, None) is None
    assert bench.clock_normalised(1000.0, {"sm_mhz": None, "sm_max_mhz": 1965.0}) is None
