"""The passes inside a CUDA graph.  Every call is stream-ordered work on caller-owned buffers
(the plan, the kernel attributes and the tensor maps are set on the host), so a forward +
backward captured once replays to the outputs of the direct calls -- bit for bit, since
every sum has a fixed order -- and a replay reads the buffers' current contents."""
import pytest
import torch

import linear_attention_soft_b200 as ra
import race_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("causal", [True, False])
def test_forward_backward_replay_in_a_cuda_graph(causal):
    B, H, N, d, L, P, tau = 1, 2, 5000, 64, 16, 4, 0.5
    inp = race_inputs.small_normal(B, H, N, d, L, P, 21, dtype=torch.bfloat16, device=DEV)
    q, k, v, W, do = inp["q"], inp["k"], inp["v"], inp["W"], inp["do"]
    out, den = torch.empty_like(q), torch.empty((B, H, N), dtype=torch.float32, device=DEV)
    ctx = torch.empty(ra.race_attn_ctx_size(B, H, N, d, L, P, causal) // 4, dtype=torch.float32, device=DEV)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    wsf, wsb = ra._workspace(q, W, causal, False), ra._workspace(q, W, causal, True)
    results = (out, den, dq, dk, dv)

    def step():
        ra.race_attn_forward(q, k, v, W, out, den, ctx, tau, causal, wsf)
        ra.race_attn_backward(q, k, v, W, out, den, do, ctx, dq, dk, dv, tau, causal, wsb)

    def direct():
        step()
        torch.cuda.synchronize()
        return [t.clone() for t in results]

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # first calls outside the capture
        step()
    torch.cuda.current_stream().wait_stream(side)
    ref = direct()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for t in results:
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(results, ref):
        assert torch.equal(a, b)
    # new inputs in the same buffers: the replay follows them
    v.copy_(torch.flip(v, dims=[2]))
    do.mul_(-0.5)
    ref2 = direct()
    assert not torch.equal(ref2[0], ref[0])
    for t in results:
        t.zero_()
    g.replay()
    torch.cuda.synchronize()
    for a, b in zip(results, ref2):
        assert torch.equal(a, b)
    del g
