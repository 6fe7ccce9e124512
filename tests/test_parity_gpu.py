"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small and ragged shapes are compared element by element on every output;
the full-size workloads (in the launch configuration bench.py times) are
compared on sampled query rows of every (batch, head).
"""

import json
import math
import os

import numpy as np
import pytest
import torch

from exact_attention_136_b200 import forward, forward_fp8, forward_host, device_status, wait_probe
from exact_attention_136_b200 import inputs, workloads as W
from exact_attention_136_b200 import _lib
from tests.oracle_cmp import TOL_LSE, TOL_O, compare, oracle

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_values.json")


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    _lib.lib()  # fails loudly when the library is missing


def run(qkv, scale, causal, wl, want_lse=True, stream=None, num_splits=1):
    dev = torch.device("cuda", 0)
    q, k, v = qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev)
    if q.dtype == torch.float8_e4m3fn:
        out, lse = forward_fp8(q, k, v, qkv.q_descale, qkv.k_descale, qkv.v_descale, scale, causal, wl,
                               return_lse=want_lse, stream=stream, num_splits=num_splits)
    else:
        out, lse = forward(q, k, v, scale, causal, wl, return_lse=want_lse, stream=stream, num_splits=num_splits)
    torch.cuda.synchronize()
    rc, flags = device_status()
    assert rc == 0, f"device status {rc} flags {flags}"
    return out, lse


def check(qkv, dtype, scale, causal, wl, rows=None):
    out, lse = run(qkv, scale, causal, wl)
    ref_o, ref_l = oracle(qkv, scale, causal, wl, rows=rows)
    d_o, d_l = compare(out, lse, ref_o, ref_l, rows=rows)
    assert d_o <= TOL_O[dtype], f"max|dO| {d_o:.3e} > {TOL_O[dtype]}"
    assert d_l <= TOL_LSE, f"max|dLSE| {d_l:.3e} > {TOL_LSE}"
    return d_o, d_l


# (B, N_q, N_k, H, D, dtype, causal, window_left)
SMALL = [
    (1, 128, 128, 1, 64, "fp16", False, -1),
    (1, 128, 128, 1, 128, "bf16", True, -1),
    (2, 256, 256, 3, 64, "bf16", False, -1),
    (2, 256, 256, 3, 128, "fp16", True, -1),
    (1, 1, 1, 2, 128, "bf16", False, -1),
    (1, 7, 7, 2, 64, "fp16", True, -1),
    (1, 127, 127, 2, 128, "bf16", True, -1),
    (1, 129, 129, 2, 64, "bf16", True, -1),
    (1, 255, 255, 1, 128, "fp16", False, -1),
    (1, 257, 257, 1, 128, "bf16", True, -1),
    (2, 300, 300, 2, 64, "fp16", True, -1),
    (1, 1000, 1000, 2, 128, "bf16", True, -1),
    (1, 100, 300, 2, 128, "bf16", False, -1),
    (1, 100, 300, 2, 64, "fp16", True, -1),
    (1, 300, 100, 2, 128, "bf16", True, -1),
    (1, 513, 1025, 1, 128, "fp16", True, -1),
    (1, 1025, 513, 1, 64, "bf16", False, -1),
    (1, 600, 600, 2, 128, "bf16", True, 0),
    (1, 600, 600, 2, 128, "bf16", True, 1),
    (1, 600, 600, 1, 64, "fp16", True, 127),
    (1, 600, 600, 1, 128, "bf16", True, 128),
    (1, 600, 600, 1, 128, "fp16", True, 129),
    (2, 1000, 1000, 2, 128, "bf16", True, 300),
    (1, 700, 700, 2, 64, "bf16", False, 200),
    (1, 600, 100, 2, 128, "bf16", True, 50),   # rows >= 151 see no key
    (1, 1000, 40, 1, 64, "fp16", True, 10),    # whole tiles with no key
    (1, 512, 512, 1, 128, "e4m3", False, -1),
    (2, 300, 300, 2, 128, "e4m3", True, -1),
    (1, 1000, 1000, 1, 128, "e4m3", True, 200),
    (1, 200, 333, 2, 128, "e4m3", True, -1),
]


@pytest.mark.parametrize("case", SMALL, ids=[
    f"B{c[0]}_q{c[1]}_k{c[2]}_H{c[3]}_D{c[4]}_{c[5]}_{'c' if c[6] else 'nc'}_w{c[7]}" for c in SMALL])
def test_small_exact_parity(case):
    B, nq, nk, H, D, dt, causal, wl = case
    qkv = inputs.make_qkv(B, nq, nk, H, D, dt, seeds=(11 + nq, 12 + nk, 13 + D))
    check(qkv, dt, 1.0 / math.sqrt(D), causal, wl)


# grouped / multi-query K/V heads: (B, N_q, N_k, H, H_kv, D, dtype, causal, window_left)
GQA = [
    (1, 256, 256, 8, 1, 128, "bf16", True, -1),     # multi-query
    (2, 300, 300, 8, 2, 64, "fp16", False, -1),
    (1, 700, 700, 6, 3, 128, "bf16", True, 200),
    (1, 513, 1025, 4, 2, 128, "fp16", True, -1),
    (1, 1000, 1000, 8, 4, 128, "e4m3", True, -1),
    (1, 129, 129, 4, 1, 64, "bf16", False, 50),
]


@pytest.mark.parametrize("case", GQA, ids=[
    f"B{c[0]}_q{c[1]}_k{c[2]}_H{c[3]}_Hkv{c[4]}_D{c[5]}_{c[6]}_{'c' if c[7] else 'nc'}_w{c[8]}" for c in GQA])
def test_gqa_parity(case):
    B, nq, nk, H, h_kv, D, dt, causal, wl = case
    qkv = inputs.make_qkv(B, nq, nk, H, D, dt, seeds=(41 + nq, 42 + nk, 43 + H), h_kv=h_kv)
    check(qkv, dt, 1.0 / math.sqrt(D), causal, wl)


def test_gqa_with_all_heads_equals_mha_entry():
    """fa_fwd_gqa with H_kv = H is the ordinary forward, bit for bit."""
    qkv = inputs.make_qkv(1, 384, 384, 4, 128, "bf16", seeds=(51, 52, 53))
    dev = torch.device("cuda", 0)
    q, k, v = qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev)
    o1, l1 = forward(q, k, v, 0.09, True, -1)
    o2 = torch.empty_like(o1)
    l2 = torch.empty_like(l1)
    s = torch.cuda.current_stream()
    rc = _lib.lib().fa_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr(), l2.data_ptr(), 1, 384, 384,
                               4, 4, 128, 0.09, 1, -1, _lib.FA_BF16, 1.0, 1.0, 1.0, s.cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# split key range: (B, N_q, N_k, H, H_kv, D, dtype, causal, window_left, num_splits)
SPLIT = [
    (2, 1, 4096, 8, 2, 128, "bf16", False, -1, 8),      # decode-like: one query row
    (1, 16, 3000, 4, 4, 64, "fp16", False, -1, 5),      # ragged last key block
    (1, 1000, 1000, 2, 2, 128, "bf16", True, -1, 3),    # causal: later slices empty for early rows
    (1, 2000, 2000, 2, 1, 128, "fp16", True, 300, 4),   # window: most slices empty for each row
    (1, 64, 5000, 4, 2, 128, "e4m3", False, -1, 6),
    (1, 200, 700, 2, 2, 64, "bf16", False, -1, 100),    # more slices than key blocks
    (1, 300, 40, 2, 2, 64, "fp16", True, 10, 4),        # one key block: no split, rows with no key
]


@pytest.mark.parametrize("case", SPLIT, ids=[
    f"B{c[0]}_q{c[1]}_k{c[2]}_H{c[3]}_Hkv{c[4]}_D{c[5]}_{c[6]}_{'c' if c[7] else 'nc'}_w{c[8]}_s{c[9]}"
    for c in SPLIT])
def test_splitkv_parity(case):
    B, nq, nk, H, h_kv, D, dt, causal, wl, ns = case
    qkv = inputs.make_qkv(B, nq, nk, H, D, dt, seeds=(61 + nq, 62 + nk, 63 + ns), h_kv=h_kv)
    dev = torch.device("cuda", 0)
    q, k, v = qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev)
    scale = 1.0 / math.sqrt(D)
    if dt == "e4m3":
        out, lse = forward_fp8(q, k, v, qkv.q_descale, qkv.k_descale, qkv.v_descale, scale, causal, wl,
                               num_splits=ns)
    else:
        out, lse = forward(q, k, v, scale, causal, wl, num_splits=ns)
    torch.cuda.synchronize()
    rc, flags = device_status()
    assert rc == 0, f"device status {rc} flags {flags}"
    ref_o, ref_l = oracle(qkv, scale, causal, wl)
    d_o, d_l = compare(out, lse, ref_o, ref_l)
    assert d_o <= TOL_O[dt], f"max|dO| {d_o:.3e} > {TOL_O[dt]}"
    assert d_l <= TOL_LSE, f"max|dLSE| {d_l:.3e} > {TOL_LSE}"


def test_splitkv_auto_slices():
    """num_splits = 0 picks the slices from the SM count; the result still matches the oracle."""
    from exact_attention_136_b200 import auto_splits
    assert auto_splits(1, 100, 4096, 2) > 1                 # 2 units, 148 SMs
    assert auto_splits(4, 8192, 8192, 32) == 1              # thousands of units
    assert auto_splits(1, 100, 256, 2) == 2                 # capped at the key blocks
    qkv = inputs.make_qkv(1, 100, 4096, 2, 128, "bf16", seeds=(81, 82, 83))
    dev = torch.device("cuda", 0)
    out, lse = forward(qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev), 0.1, False, -1, num_splits=0)
    torch.cuda.synchronize()
    ref_o, ref_l = oracle(qkv, 0.1, False, -1)
    d_o, d_l = compare(out, lse, ref_o, ref_l)
    assert d_o <= TOL_O["bf16"] and d_l <= TOL_LSE, (d_o, d_l)


def test_splitkv_one_slice_is_the_plain_forward():
    """num_splits = 1 takes the plain path: bit-identical to forward()."""
    qkv = inputs.make_qkv(1, 300, 900, 4, 128, "bf16", seeds=(71, 72, 73))
    dev = torch.device("cuda", 0)
    q, k, v = qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev)
    o1, l1 = forward(q, k, v, 0.1, False, -1)
    o2, l2 = forward(q, k, v, 0.1, False, -1, num_splits=1)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# attention mask: (B, N_q, N_k, H, D, dtype, causal, window_left, kind, mask batch, mask heads)
MASKED = [
    (2, 256, 256, 2, 128, "bf16", False, -1, "bool", 2, 2),
    (1, 300, 517, 2, 64, "fp16", True, -1, "bool", 1, 1),      # N_k not a multiple of 16: padded rows
    (2, 384, 384, 2, 128, "bf16", False, -1, "add", 2, 1),
    (1, 200, 333, 2, 128, "fp16", False, 100, "add", 1, 2),
    (1, 500, 500, 2, 128, "e4m3", True, -1, "add", 1, 1),
    (1, 257, 257, 1, 64, "bf16", False, -1, "bool_rows", 1, 1),  # some rows fully masked
]


def _make_mask(case, seed):
    B, nq, nk, H, D, dt, causal, wl, kind, mb, mh = case
    g = torch.Generator().manual_seed(seed)
    if kind.startswith("bool"):
        m = torch.rand((mb, mh, nq, nk), generator=g) > 0.3
        if kind == "bool_rows":
            m[:, :, ::7] = False
        return m, m.numpy()
    t = torch.float16 if dt == "fp16" else torch.bfloat16
    m = (2.0 * torch.randn((mb, mh, nq, nk), generator=g)).to(t)
    m[torch.rand((mb, mh, nq, nk), generator=g) < 0.1] = float("-inf")
    return m, m.to(torch.float64).numpy()


@pytest.mark.parametrize("case", MASKED, ids=[
    f"B{c[0]}_q{c[1]}_k{c[2]}_H{c[3]}_D{c[4]}_{c[5]}_{'c' if c[6] else 'nc'}_w{c[7]}_{c[8]}_mb{c[9]}mh{c[10]}"
    for c in MASKED])
def test_attn_mask_parity(case):
    B, nq, nk, H, D, dt, causal, wl, kind, mb, mh = case
    qkv = inputs.make_qkv(B, nq, nk, H, D, dt, seeds=(91 + nq, 92 + nk, 93 + H))
    mask_t, mask_np = _make_mask(case, 94 + nq)
    dev = torch.device("cuda", 0)
    q, k, v = qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev)
    scale = 1.0 / math.sqrt(D)
    if dt == "e4m3":
        out, lse = forward_fp8(q, k, v, qkv.q_descale, qkv.k_descale, qkv.v_descale, scale, causal, wl,
                               attn_mask=mask_t.to(dev))
    else:
        out, lse = forward(q, k, v, scale, causal, wl, attn_mask=mask_t.to(dev))
    torch.cuda.synchronize()
    rc, flags = device_status()
    assert rc == 0, f"device status {rc} flags {flags}"
    ref_o, ref_l = oracle(qkv, scale, causal, wl, mask=mask_np)
    d_o, d_l = compare(out, lse, ref_o, ref_l)
    assert d_o <= TOL_O[dt], f"max|dO| {d_o:.3e} > {TOL_O[dt]}"
    assert d_l <= TOL_LSE, f"max|dLSE| {d_l:.3e} > {TOL_LSE}"


def test_float_mask_of_another_type_is_rejected():
    """Like SDPA, an additive mask must have the inputs' 16-bit type: an fp32
    mask is refused rather than silently rounded."""
    dev = torch.device("cuda", 0)
    q = torch.zeros((1, 64, 2, 64), dtype=torch.bfloat16, device=dev)
    with pytest.raises(ValueError):
        forward(q, q, q, 0.125, False, -1, attn_mask=torch.zeros((64, 64), dtype=torch.float32, device=dev))
    with pytest.raises(ValueError):
        forward(q, q, q, 0.125, False, -1, attn_mask=torch.zeros((64, 64), dtype=torch.float16, device=dev))


def test_mask_passed_in_place_equals_padded_copy():
    """A mask whose rows are whole 16-byte chunks goes to the kernel as it is;
    a strided view of the same values is copied first.  Same result."""
    dev = torch.device("cuda", 0)
    qkv = inputs.make_qkv(1, 256, 512, 2, 128, "bf16", seeds=(31, 32, 33))
    q, k, v = qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev)
    g = torch.Generator().manual_seed(34)
    wide = (2.0 * torch.randn((2, 256, 1024), generator=g)).to(torch.bfloat16).to(dev)
    dense = wide[:, :, :512].contiguous()[None]         # [1, 2, 256, 512], taken as it is
    strided = wide[:, :, ::2][None]                     # last dim strided: copied
    strided_vals = strided.contiguous()
    o1, l1 = forward(q, k, v, 0.09, False, -1, attn_mask=dense)
    o2, l2 = forward(q, k, v, 0.09, False, -1, attn_mask=dense[:, :, :, :].expand(1, 2, 256, 512))
    o3, l3 = forward(q, k, v, 0.09, False, -1, attn_mask=strided)
    o4, l4 = forward(q, k, v, 0.09, False, -1, attn_mask=strided_vals)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert torch.equal(o3, o4) and torch.equal(l3, l4)
    ref_o, ref_l = oracle(qkv, 0.09, False, -1, mask=dense.to(torch.float64).cpu().numpy())
    d_o, d_l = compare(o1, l1, ref_o, ref_l)
    assert d_o <= TOL_O["bf16"] and d_l <= TOL_LSE


def test_temporaries_survive_a_side_stream():
    """The split forward's workspace and a padded mask copy are freed when the
    call returns; on a stream other than the current one they must stay
    reserved until the kernels have run, even if the caller allocates and
    overwrites memory right away."""
    dev = torch.device("cuda", 0)
    qkv = inputs.make_qkv(1, 128, 8192, 8, 128, "bf16", seeds=(41, 42, 43))
    q, k, v = qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev)
    # N_k - 3 keys: the boolean mask's rows are not whole 16-byte chunks, so it is copied
    mask = (torch.rand((1, 1, 128, 8192 - 3), generator=torch.Generator().manual_seed(44)) > 0.2).to(dev)
    kq, vm = k[:, :8192 - 3].contiguous(), v[:, :8192 - 3].contiguous()
    ref_s, ref_sl = forward(q, k, v, 0.09, False, -1, num_splits=8)
    ref_m, ref_ml = forward(q, kq, vm, 0.09, False, -1, attn_mask=mask)
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    for _ in range(3):
        o_s, l_s = forward(q, k, v, 0.09, False, -1, num_splits=8, stream=side)
        o_m, l_m = forward(q, kq, vm, 0.09, False, -1, attn_mask=mask, stream=side)
        # both streams allocate at once and scribble on what they get
        junk = [torch.full((1 << 22,), float("nan"), device=dev) for _ in range(8)]
        with torch.cuda.stream(side):
            junk += [torch.full((1 << 22,), float("nan"), device=dev) for _ in range(8)]
        del junk
        side.synchronize()
        assert torch.equal(o_s, ref_s) and torch.equal(l_s, ref_sl)
        assert torch.equal(o_m, ref_m) and torch.equal(l_m, ref_ml)


def test_causal_pattern_mask_equals_causal():
    """A boolean mask holding the causal pattern gives the causal forward (to rounding)."""
    qkv = inputs.make_qkv(1, 640, 640, 2, 128, "bf16", seeds=(95, 96, 97))
    dev = torch.device("cuda", 0)
    q, k, v = qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev)
    tri = torch.tril(torch.ones((640, 640), dtype=torch.bool, device=dev))
    o1, l1 = forward(q, k, v, 0.09, True, -1)
    o2, l2 = forward(q, k, v, 0.09, False, -1, attn_mask=tri)
    torch.cuda.synchronize()
    assert float((o1.float() - o2.float()).abs().max()) <= 8e-3
    assert float((l1 - l2).abs().max()) <= 1e-4


@pytest.mark.parametrize("dt,D", [("fp16", 64), ("bf16", 128), ("e4m3", 128)])
@pytest.mark.parametrize("mult", [4.0, 12.0])
def test_large_scores_exercise_rescaling(dt, D, mult):
    """Scores of tens to hundreds (log2 units): the max rises often, O is rescaled in place."""
    qkv = inputs.make_qkv(1, 700, 700, 2, D, "bf16" if dt == "e4m3" else dt, seeds=(21, 22, 23))
    if dt == "e4m3":
        q8, sq = inputs.quantize_e4m3(qkv.q.float() * mult)
        k8, sk = inputs.quantize_e4m3(qkv.k.float())
        v8, sv = inputs.quantize_e4m3(qkv.v.float())
        qkv = inputs.QKV(q8, k8, v8, sq, sk, sv)
    else:
        qkv = inputs.QKV((qkv.q.float() * mult).to(qkv.q.dtype), qkv.k, qkv.v)
    for causal in (False, True):
        check(qkv, dt, 1.0 / math.sqrt(D), causal, -1)


def test_many_units_per_cta():
    """More work units than SMs: barrier phases carry across units of one CTA."""
    qkv = inputs.make_qkv(4, 1024, 1024, 32, 64, "fp16", seeds=(31, 32, 33))
    rows = np.array([0, 1, 127, 128, 255, 256, 511, 700, 1023])
    for causal in (False, True):
        check(qkv, "fp16", 0.125, causal, -1, rows=rows)


def test_pages_accuracy_check_bound():
    """The pages' check (B1 H8 N512 D64 fp16, scores / 8) expects max diff < 1e-3."""
    g = json.load(open(GOLDEN))["accuracy_check"]
    w = W.WORKLOADS["pr1_b1h8n512d64_fp16"]
    assert (w.B, w.H, w.n_q, w.D) == (g["batch"], g["heads"], g["seqlen"], g["headdim"])
    assert w.scale == 1.0 / g["score_divisor"]
    qkv = inputs.make_qkv(w.B, w.n_q, w.n_k, w.H, w.D, w.dtype, seeds=w.seeds)
    d_o, d_l = check(qkv, "fp16", w.scale, w.causal, w.window_left)
    assert d_o < g["max_abs_diff_bound"]


@pytest.mark.parametrize("name", W.ORDER)
def test_full_workload_sampled_rows(name):
    """Every workload at full size; all rows finite, sampled rows of every head vs the oracle."""
    w = W.WORKLOADS[name]
    qkv = inputs.make_qkv(w.B, w.n_q, w.n_k, w.H, w.D, w.dtype, seeds=w.seeds, h_kv=w.h_kv)
    rows = W.sample_rows(w, count=64 if w.n_q > 4096 else 256)
    mask = W.make_mask(w)
    if mask is None:
        out, lse = run(qkv, w.scale, w.causal, w.window_left, num_splits=w.splits)
    else:
        dev = torch.device("cuda", 0)
        out, lse = forward(qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev), w.scale, w.causal, w.window_left,
                           attn_mask=mask.to(dev))
        torch.cuda.synchronize()
    assert bool(torch.isfinite(out).all()) and bool(torch.isfinite(lse).all())
    ref_o, ref_l = oracle(qkv, w.scale, w.causal, w.window_left, rows=rows,
                          mask=None if mask is None else mask.numpy())
    d_o, d_l = compare(out, lse, ref_o, ref_l, rows=rows)
    assert d_o <= TOL_O[w.dtype] and d_l <= TOL_LSE, (d_o, d_l)


def test_no_keys_gives_zero_and_neg_inf():
    qkv = inputs.make_qkv(2, 300, 1, 2, 64, "bf16", seeds=(41, 42, 43))
    dev = torch.device("cuda", 0)
    k0 = torch.empty((2, 0, 2, 64), dtype=torch.bfloat16, device=dev)
    out, lse = forward(qkv.q.to(dev), k0, k0.clone(), 0.125)
    torch.cuda.synchronize()
    assert bool((out == 0).all()) and bool(torch.isneginf(lse).all())


def test_lse_optional_and_guard_regions():
    """Writes stay inside out / lse: sentinels around both are untouched; lse=NULL works."""
    dev = torch.device("cuda", 0)
    B, n, H, D = 1, 333, 3, 128
    qkv = inputs.make_qkv(B, n, n, H, D, "bf16", seeds=(51, 52, 53))
    q, k, v = qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev)
    pad = 4096
    obuf = torch.full((pad + B * n * H * D + pad,), 7.0, dtype=torch.bfloat16, device=dev)
    lbuf = torch.full((pad + B * H * n + pad,), 7.0, dtype=torch.float32, device=dev)
    out = obuf[pad:pad + B * n * H * D].view(B, n, H, D)
    lse = lbuf[pad:pad + B * H * n].view(B, H, n)
    forward(q, k, v, 1 / math.sqrt(D), True, -1, out=out, lse=lse)
    out2, none = forward(q, k, v, 1 / math.sqrt(D), True, -1, return_lse=False)
    torch.cuda.synchronize()
    assert none is None
    assert bool((obuf[:pad] == 7).all()) and bool((obuf[-pad:] == 7).all())
    assert bool((lbuf[:pad] == 7).all()) and bool((lbuf[-pad:] == 7).all())
    assert torch.equal(out, out2)
    ref_o, ref_l = oracle(qkv, 1 / math.sqrt(D), True, -1)
    d_o, d_l = compare(out, lse, ref_o, ref_l)
    assert d_o <= TOL_O["bf16"] and d_l <= TOL_LSE


def test_side_stream_and_determinism():
    dev = torch.device("cuda", 0)
    qkv = inputs.make_qkv(2, 777, 777, 4, 128, "fp16", seeds=(61, 62, 63))
    q, k, v = qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        a, la = forward(q, k, v, None, True)
    b, lb = forward(q, k, v, None, True, stream=s)
    s.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_host_buffer_entry_point_matches_device_entry():
    dev = torch.device("cuda", 0)
    B, n, H, D = 1, 640, 4, 128
    qkv = inputs.make_qkv(B, n, n, H, D, "bf16", seeds=(71, 72, 73))
    staging = {"q": torch.empty_like(qkv.q, device=dev), "k": torch.empty_like(qkv.k, device=dev),
               "v": torch.empty_like(qkv.v, device=dev),
               "out": torch.empty((B, n, H, D), dtype=torch.bfloat16, device=dev),
               "lse": torch.empty((B, H, n), dtype=torch.float32, device=dev)}
    ho, hl = forward_host(qkv.q.pin_memory(), qkv.k.pin_memory(), qkv.v.pin_memory(), staging, 0.09, True)
    do, dl = forward(qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev), 0.09, True)
    torch.cuda.synchronize()
    assert torch.equal(ho, do.cpu()) and torch.equal(hl, dl.cpu())


def test_async_host_entry_point_on_three_streams():
    """fa_fwd_host_async: batches enqueued on three streams with their own
    staging, nothing synchronised between calls; after the streams complete
    every host result equals the device entry's for its batch."""
    dev = torch.device("cuda", 0)
    B, n, H, D = 1, 700, 4, 128
    batches = [inputs.make_qkv(B, n, n, H, D, "bf16", seeds=(81 + 3 * i, 82 + 3 * i, 83 + 3 * i)) for i in range(6)]
    streams = [torch.cuda.Stream(dev) for _ in range(3)]
    stagings = [{"q": torch.empty((B, n, H, D), dtype=torch.bfloat16, device=dev),
                 "k": torch.empty((B, n, H, D), dtype=torch.bfloat16, device=dev),
                 "v": torch.empty((B, n, H, D), dtype=torch.bfloat16, device=dev),
                 "out": torch.empty((B, n, H, D), dtype=torch.bfloat16, device=dev),
                 "lse": torch.empty((B, H, n), dtype=torch.float32, device=dev)} for _ in range(3)]
    pinned = [(b.q.pin_memory(), b.k.pin_memory(), b.v.pin_memory()) for b in batches]
    results = []
    for i, (hq, hk, hv) in enumerate(pinned):
        ho = torch.empty((B, n, H, D), dtype=torch.bfloat16, pin_memory=True)
        hl = torch.empty((B, H, n), dtype=torch.float32, pin_memory=True)
        results.append(forward_host(hq, hk, hv, stagings[i % 3], 0.09, True, out=ho, lse=hl,
                                    stream=streams[i % 3], synchronize=False))
    torch.cuda.synchronize()
    for b, (ho, hl) in zip(batches, results):
        do, dl = forward(b.q.to(dev), b.k.to(dev), b.v.to(dev), 0.09, True)
        torch.cuda.synchronize()
        assert torch.equal(ho, do.cpu()) and torch.equal(hl, dl.cpu())


def test_wait_timeout_reports_status_and_context_survives():
    """A wait that nothing completes ends after its limit with FA_ERR_TIMEOUT; later calls still work."""
    rc, _ = device_status()
    assert rc == 0
    wait_probe(2_000_000)  # 2 ms
    rc, flags = device_status()
    assert rc == _lib.FA_ERR_TIMEOUT and flags != 0
    rc, _ = device_status()
    assert rc == 0  # the word was cleared
    qkv = inputs.make_qkv(1, 256, 256, 2, 64, "fp16", seeds=(81, 82, 83))
    check(qkv, "fp16", 0.125, True, -1)
