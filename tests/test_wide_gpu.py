"""GPU parity of the tensor-core path for d = 128 with 5 hyperplanes per table (bf16, causal):
the features are cut into groups of 8 tables and the value columns into two halves, and the
library adds the passes' partial sums.  Every output is compared with the fp64 oracle on the
same seeded inputs; the cases span L = 8 (one group) to L = 32 (four groups), several heads,
several segments per head and ragged last chunks."""
import numpy as np
import pytest
import torch

import linear_attention_soft_b200 as ra
from parity import TOL, gpu_backward, gpu_forward, oracle_backward, oracle_forward, rel_err
import race_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"

# (B, H, N, L): one to four feature groups; N spans one chunk, several segments (segments
# hold whole 128-token chunks) and ragged tails
CASES = [
    (1, 1, 1, 8),
    (1, 1, 129, 16),
    (1, 1, 1000, 32),
    (1, 2, 1537, 24),
    (2, 1, 2300, 8),
    (1, 1, 4100, 32),
]


def _inputs(B, H, N, L, seed, scale_qk=2.0):
    return race_inputs.small_normal(B, H, N, 128, L, 5, seed, dtype=torch.bfloat16, device=DEV,
                                    scale_qk=scale_qk)


def _ran(names):
    prof = ra.race_attn_profile_read()
    return all(n in prof for n in names), prof


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dN%d_L%d" % c)
def test_forward_matches_oracle(case):
    B, H, N, L = case
    inp = _inputs(B, H, N, L, seed=N + 7 * L)
    ra.race_attn_profile_reset()
    ra.race_attn_profile_enable(True)
    out, den, _ = gpu_forward(inp, 0.5, True)
    torch.cuda.synchronize()
    ran, prof = _ran(("wide_proj", "wide_agg_kv", "wide_fwd_walk"))
    ra.race_attn_profile_enable(False)
    assert ran, prof
    o_ref, den_ref = oracle_forward(inp, 0.5, True)
    errs = {"out": rel_err(out, o_ref), "den": rel_err(den, den_ref)}
    assert max(errs.values()) <= TOL[torch.bfloat16], errs


def test_forward_is_deterministic():
    inp = _inputs(1, 1, 3000, 32, seed=5)
    o1, d1, _ = gpu_forward(inp, 0.5, True)
    o2, d2, _ = gpu_forward(inp, 0.5, True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(d1, d2)


def test_forward_causality():
    """Changing the tokens after position n leaves rows 0..n unchanged, bit for bit."""
    inp = _inputs(1, 1, 2000, 16, seed=11)
    o1, d1, _ = gpu_forward(inp, 0.5, True)
    n = 777
    inp2 = {k: v.clone() for k, v in inp.items()}
    for name in ("q", "k", "v"):
        inp2[name][:, :, n + 1:] = torch.randn_like(inp2[name][:, :, n + 1:].float()).to(torch.bfloat16)
    o2, d2, _ = gpu_forward(inp2, 0.5, True)
    torch.cuda.synchronize()
    assert torch.equal(o1[:, :, :n + 1], o2[:, :, :n + 1]) and torch.equal(d1[:, :, :n + 1], d2[:, :, :n + 1])


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dN%d_L%d" % c)
def test_backward_matches_oracle(case):
    B, H, N, L = case
    inp = _inputs(B, H, N, L, seed=3 * N + L)
    out, den, _ = gpu_forward(inp, 0.5, True)
    ra.race_attn_profile_reset()
    ra.race_attn_profile_enable(True)
    dq, dk, dv = gpu_backward(inp, out, den, 0.5, True)
    torch.cuda.synchronize()
    ran, prof = _ran(("wide_rowc", "wide_agg_qdy", "wide_bwd_q_walk", "wide_bwd_kv_walk", "wide_dx"))
    ra.race_attn_profile_enable(False)
    assert ran, prof
    dq_ref, dk_ref, dv_ref = oracle_backward(inp, 0.5, True)
    # with one token, out_0 = v_0 whatever q and k are: dq = dk = 0 exactly, so the error is
    # measured against the scale of dO there
    fl = 1e-2 * float(inp["do"].abs().max()) if N == 1 else 0.0
    errs = {"dq": rel_err(dq, dq_ref, fl), "dk": rel_err(dk, dk_ref, fl), "dv": rel_err(dv, dv_ref)}
    assert max(errs.values()) <= TOL[torch.bfloat16], errs


def test_backward_is_deterministic():
    inp = _inputs(1, 1, 3000, 32, seed=9)
    out, den, _ = gpu_forward(inp, 0.5, True)
    g1 = gpu_backward(inp, out, den, 0.5, True)
    g2 = gpu_backward(inp, out, den, 0.5, True)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(g1, g2))


def test_backward_with_a_saved_context():
    """The bench passes the forward's context to the backward; the feature-group path
    leaves it aside and gives the same gradients."""
    inp = _inputs(1, 1, 1500, 16, seed=4)
    out, den, ctx = gpu_forward(inp, 0.5, True, save_ctx=True)
    g1 = gpu_backward(inp, out, den, 0.5, True, ctx=ctx)
    g2 = gpu_backward(inp, out, den, 0.5, True)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(g1, g2))


def test_context_left_by_another_path_is_not_read():
    """A forward that cannot take the feature-group path (its workspace holds only the segment
    statistics) leaves ctx in the general layout and clears the tag that the feature-group
    forward sets; the feature-group backward then recomputes the statistics."""
    B, H, N, L = 1, 1, 1500, 16
    inp = _inputs(B, H, N, L, seed=12)
    q, k, v, W = inp["q"], inp["k"], inp["v"], inp["W"]
    code = ra.RACE_BF16
    full = torch.empty(ra.race_attn_workspace_size(B, H, N, 128, L, 5, 1, 0, code), dtype=torch.uint8, device=DEV)
    small = torch.empty(ra.race_attn_workspace_size(B, H, N, 128, L, 5, 0, 0, code), dtype=torch.uint8,
                        device=DEV)  # the general path's need (bidirectional sizes)
    assert small.numel() < full.numel()
    ctx = torch.empty(ra.race_attn_ctx_size(B, H, N, 128, L, 5, 1) // 4, dtype=torch.float32, device=DEV)
    out, den = torch.empty_like(q), torch.empty((B, H, N), dtype=torch.float32, device=DEV)
    ra.race_attn_forward(q, k, v, W, out, den, ctx, 0.5, True, full)     # feature-group path: tag set
    g_ctx = gpu_backward(inp, out, den, 0.5, True, ctx=ctx)
    g_none = gpu_backward(inp, out, den, 0.5, True)
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(g_ctx, g_none))
    out2, den2 = torch.empty_like(q), torch.empty_like(den)
    ra.race_attn_forward(q, k, v, W, out2, den2, ctx, 0.5, True, small)  # general path: tag cleared
    g_ctx2 = gpu_backward(inp, out, den, 0.5, True, ctx=ctx)
    torch.cuda.synchronize()
    assert rel_err(out2, out.float().cpu().numpy()) <= TOL[torch.bfloat16]
    assert all(torch.equal(a, b) for a, b in zip(g_ctx2, g_none))


@pytest.mark.parametrize("tau", [0.25, 1.0, 3.0])
def test_other_temperatures(tau):
    """beta = 1 / tau enters the soft hash and its VJP: forward and backward at three more
    temperatures."""
    inp = _inputs(1, 1, 700, 16, seed=int(100 * tau))
    out, den, _ = gpu_forward(inp, tau, True)
    dq, dk, dv = gpu_backward(inp, out, den, tau, True)
    torch.cuda.synchronize()
    o_ref, den_ref = oracle_forward(inp, tau, True)
    dq_ref, dk_ref, dv_ref = oracle_backward(inp, tau, True)
    errs = {"out": rel_err(out, o_ref), "den": rel_err(den, den_ref), "dq": rel_err(dq, dq_ref),
            "dk": rel_err(dk, dk_ref), "dv": rel_err(dv, dv_ref)}
    assert max(errs.values()) <= TOL[torch.bfloat16], errs


def test_chunk_and_segment_edges():
    """Lengths at the edges of a 128-token chunk and of segments of one to four chunks."""
    bad = {}
    for N in (2, 127, 128, 129, 255, 256, 511, 512, 513, 1024, 1025):
        inp = _inputs(1, 1, N, 8, seed=N)
        out, den, _ = gpu_forward(inp, 0.5, True)
        dq, dk, dv = gpu_backward(inp, out, den, 0.5, True)
        torch.cuda.synchronize()
        o_ref, den_ref = oracle_forward(inp, 0.5, True)
        dq_ref, dk_ref, dv_ref = oracle_backward(inp, 0.5, True)
        errs = {"out": rel_err(out, o_ref), "den": rel_err(den, den_ref), "dq": rel_err(dq, dq_ref),
                "dk": rel_err(dk, dk_ref), "dv": rel_err(dv, dv_ref)}
        if max(errs.values()) > TOL[torch.bfloat16]:
            bad[N] = errs
    assert not bad, bad
