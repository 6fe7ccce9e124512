"""The forward and the backward captured in a CUDA graph and replayed.

Every launch of the library is asynchronous on the caller's stream and
allocates nothing once a stream has been used (its scheduler counters are
taken on first use, and the backward's workspace comes from torch's pool),
so a training step built from them can be captured and replayed.  The
replayed results must be the eager ones bit for bit: the kernels take the
same arithmetic in the same order whatever CTA runs a unit.
"""

import pytest
import torch

from exact_attention_136_b200 import backward, forward

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


@pytest.mark.parametrize("dtype,D,causal,window_left", [(torch.bfloat16, 128, True, 256),
                                                         (torch.float16, 64, False, -1)])
def test_forward_backward_replay_in_a_cuda_graph(dtype, D, causal, window_left):
    dev = torch.device("cuda", 0)
    B, N, H = 2, 1000, 4
    gen = torch.Generator().manual_seed(71 + D)

    def fresh():
        return (torch.randn(B, N, H, D, generator=gen) * 1.5).to(dtype).to(dev)

    q, k, v, do = fresh(), fresh(), fresh(), fresh()
    scale = D ** -0.5
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        # warm-up on the capture stream: kernel attributes set, the stream's
        # scheduler counters taken
        for _ in range(2):
            out, lse = forward(q, k, v, scale, causal, window_left)
            backward(q, k, v, out, lse, do, scale, causal, window_left)
    torch.cuda.current_stream(dev).wait_stream(s)
    torch.cuda.synchronize()

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        g_out, g_lse = forward(q, k, v, scale, causal, window_left)
        g_dq, g_dk, g_dv = backward(q, k, v, g_out, g_lse, do, scale, causal, window_left)

    for trial in range(3):
        if trial:
            # new values in the captured input buffers
            for t in (q, k, v, do):
                t.copy_(fresh())
        graph.replay()
        torch.cuda.synchronize()
        e_out, e_lse = forward(q, k, v, scale, causal, window_left)
        e_dq, e_dk, e_dv = backward(q, k, v, e_out, e_lse, do, scale, causal, window_left)
        torch.cuda.synchronize()
        assert torch.isfinite(g_out.float()).all()
        for got, want in ((g_out, e_out), (g_lse, e_lse), (g_dq, e_dq), (g_dk, e_dk), (g_dv, e_dv)):
            assert torch.equal(got, want), f"trial {trial}: replay differs from the eager call"
