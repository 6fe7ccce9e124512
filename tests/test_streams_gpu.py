"""Many streams at once: every stream gets its own scheduler counters.

fa_fwd's persistent CTAs claim work units from a pair of counters that
belongs to the launching stream.  Forwards issued on more streams than one
chunk of counter pairs holds (256) must still each get a pair of their own:
two overlapping launches that shared one would claim each other's units and
leave rows unwritten.  Raw CUDA streams are used (torch hands out streams from
a small pool, which would reuse handles).
"""

import math

import numpy as np
import pytest
import torch

from exact_attention_136_b200 import _lib, device_status, inputs
from tests.oracle_cmp import TOL_LSE, TOL_O, compare, oracle

pytestmark = pytest.mark.gpu

N_STREAMS = 300   # more than one chunk of 256 counter pairs


def _cudart():
    try:
        from cuda.bindings import runtime as rt
    except ImportError:
        from cuda import cudart as rt
    return rt


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    _lib.lib()


def test_forwards_on_300_streams_each_match_the_oracle():
    rt = _cudart()
    dev = torch.device("cuda", 0)
    # 40 heads x 4 units of 256 rows = 160 units > 148 SMs: units are claimed
    # through the counters, not only handed out by block index
    B, n, H, D = 1, 1024, 40, 64
    qkv = inputs.make_qkv(B, n, n, H, D, "fp16", seeds=(301, 302, 303))
    q, k, v = qkv.q.to(dev), qkv.k.to(dev), qkv.v.to(dev)
    scale = 1.0 / math.sqrt(D)
    outs = [torch.full((B, n, H, D), float("nan"), dtype=torch.float16, device=dev) for _ in range(N_STREAMS)]
    lses = [torch.full((B, H, n), float("nan"), dtype=torch.float32, device=dev) for _ in range(N_STREAMS)]
    torch.cuda.synchronize()
    streams = []
    try:
        for _ in range(N_STREAMS):
            err, s = rt.cudaStreamCreateWithFlags(rt.cudaStreamNonBlocking)
            assert int(err) == 0, err
            streams.append(s)
        # every launch is issued before any is waited for, so they overlap
        for s, out, lse in zip(streams, outs, lses):
            rc = _lib.lib().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(), B, n, n,
                                   H, D, scale, 1, -1, _lib.FA_FP16, int(s))
            assert rc == _lib.FA_OK, _lib.status_string(rc)
        torch.cuda.synchronize()
    finally:
        for s in streams:
            rt.cudaStreamDestroy(s)
    rc, flags = device_status()
    assert rc == 0, (rc, flags)
    rows = np.array([0, 1, 127, 128, 255, 256, 511, 700, 1000, n - 1])
    ref_o, ref_l = oracle(qkv, scale, True, -1, rows=rows)
    for i, (out, lse) in enumerate(zip(outs, lses)):
        assert bool(torch.isfinite(out).all()), f"stream {i}: rows left unwritten"
        d_o, d_l = compare(out, lse, ref_o, ref_l, rows=rows)
        assert d_o <= TOL_O["fp16"] and d_l <= TOL_LSE, f"stream {i}: max|dO| {d_o:.3e} max|dLSE| {d_l:.3e}"
        # the same units computed on every stream: identical results
        assert torch.equal(out, outs[0]) and torch.equal(lse, lses[0]), f"stream {i} differs from stream 0"
