"""fa_fwd_noalloc: the forward for callers that cannot allocate device memory.

Such callers (code that must draw every device byte from its own reserved
pool, or that may not take the allocator's locks or risk an allocation
failure on its launch path) get an entry point whose work-scheduler scratch
sits in a fixed device array inside the library.  This test calls it through
the C ABI and checks its outputs against fa_fwd's on two calls in a row: the
second call would read a left-over scheduler count from the first if the
shared scratch were not brought back to zero, and would then skip work.
Collected last (file name) so a failure here stops a -x run only after all
other tests have run.
"""

import math

import pytest
import torch

from exact_attention_136_b200 import _lib, device_status, forward, inputs
from tests.oracle_cmp import TOL_LSE, TOL_O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    _lib.lib()


# more work units than SMs, so units are claimed through the scratch counters
CASES = [
    (2, 2048, 2048, 16, 128, "bf16", True, -1),
    (1, 4096, 4096, 12, 64, "fp16", False, -1),
    (1, 2048, 2048, 40, 128, "e4m3", True, 512),
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[5]}_D{c[4]}" for c in CASES])
def test_noalloc_matches_fa_fwd_on_two_calls(case):
    B, n_q, n_k, H, D, dt, causal, wl = case
    dev = torch.device("cuda", 0)
    qkv = inputs.make_qkv(B, n_q, n_k, H, D, dt, seeds=(91 + D, 92, 93))
    q, k, v = qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev)
    scale = 1.0 / math.sqrt(D)
    if dt == "e4m3":
        from exact_attention_136_b200 import forward_fp8
        ref_o, ref_l = forward_fp8(q, k, v, qkv.q_descale, qkv.k_descale, qkv.v_descale, scale, causal, wl)
        code, descales = _lib.FA_E4M3, (qkv.q_descale, qkv.k_descale, qkv.v_descale)
    else:
        ref_o, ref_l = forward(q, k, v, scale, causal, wl)
        code = _lib.FA_FP16 if dt == "fp16" else _lib.FA_BF16
        descales = (1.0, 1.0, 1.0)
    out_dtype = torch.float16 if dt == "fp16" else torch.bfloat16
    stream = torch.cuda.current_stream(dev)
    for call in range(2):
        out = torch.full((B, n_q, H, D), float("nan"), dtype=out_dtype, device=dev)
        lse = torch.full((B, H, n_q), float("nan"), dtype=torch.float32, device=dev)
        rc = _lib.lib().fa_fwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                                       B, n_q, n_k, H, D, scale, int(causal), wl, code,
                                       descales[0], descales[1], descales[2], stream.cuda_stream)
        assert rc == _lib.FA_OK, _lib.status_string(rc)
        torch.cuda.synchronize()
        status, flags = device_status()
        assert status == _lib.FA_OK, (status, flags)
        assert bool(torch.isfinite(out).all()), f"call {call}: rows left unwritten"
        d_o = float((out.float() - ref_o.float()).abs().max())
        d_l = float((lse - ref_l).abs().max())
        assert d_o <= TOL_O[dt], f"call {call}: max|dO| {d_o:.3e}"
        assert d_l <= TOL_LSE, f"call {call}: max|dLSE| {d_l:.3e}"
        # the same kernel computes every work unit the same way whichever CTA
        # claims it, so the results are also identical bit for bit
        assert torch.equal(out.view(torch.int16), ref_o.view(torch.int16)), f"call {call}: O differs from fa_fwd"
        assert torch.equal(lse.view(torch.int32), ref_l.view(torch.int32)), f"call {call}: LSE differs from fa_fwd"


def test_noalloc_rejects_bad_arguments_on_host():
    # validated before any GPU work: same rules as fa_fwd
    f = _lib.lib().fa_fwd_noalloc
    A = 1 << 20
    assert f(A, A, A, A, None, 1, 128, 128, 1, 96, 0.1, 0, -1, 0, 1.0, 1.0, 1.0, None) == _lib.FA_ERR_UNSUPPORTED
    assert f(A, A, A, A, None, 0, 128, 128, 1, 64, 0.1, 0, -1, 0, 1.0, 1.0, 1.0, None) == _lib.FA_ERR_ARG
