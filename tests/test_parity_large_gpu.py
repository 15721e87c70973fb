"""GPU parity at the workloads' full sizes, in the launch configuration the benchmark uses.

The whole sequence runs on the GPU.  The oracle then checks what it can compute one row at
a time, plus identities that hold at any size:

* forward rows sampled over the whole sequence (the causal oracle streams the keys once,
  keeping only the [L*2^P, d+1] statistics);
* out, den and dq on every row of a causal prefix (those rows depend on the first n
  tokens only, so an oracle run on the prefix is exact for them; dk and dv of the prefix
  depend on later rows and are covered by the identities below);
* every output (out, den, dq, dk, dv) of whole heads where the oracle finishes within a
  minute or two: c2, and the single head of the benchmark's workload (N = 4,194,304, cut
  into one segment per SM, so every cross-segment prefix and suffix state is exercised)
  and of the N = 2^22 point of the sequence-length sweep;
* identities at any size: each output row is a normalised average of values, so
  sum_j dv_j = sum_i dO_i; the output ignores the scale of q and k rows, so every
  dq_i is orthogonal to q_i and every dk_j to k_j.

Tolerance: normwise max relative error 2e-2 for bf16 inputs (fp32 accumulation).
"""
import gc
import json

import numpy as np
import pytest
import torch

import oracle
import race_inputs
from parity import rel_err, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = 2e-2


def _free():
    gc.collect()
    torch.cuda.empty_cache()


def _run(inp, w):
    import linear_attention_soft_b200 as ra
    out, den, ctx = ra.forward(inp["q"], inp["k"], inp["v"], inp["W"], w.tau, w.causal, save_ctx=True)
    dq, dk, dv = ra.backward(inp["q"], inp["k"], inp["v"], inp["W"], out, den, inp["do"], w.tau,
                             w.causal, ctx=ctx)
    torch.cuda.synchronize()
    del ctx
    return out, den, dq, dk, dv


def _identities(inp, dq, dk, dv, m, block=1 << 22):
    """sum_j dv_j = sum_i dO_i per head and column; dq_i . q_i = 0; dk_j . k_j = 0.
    Evaluated in row blocks so full-size workloads need little extra device memory.
    Records normwise errors into m."""
    B, H, N, d = dq.shape
    worst = 0.0
    for bh in range(B * H):
        lhs = torch.zeros(d, dtype=torch.float64, device=DEV)
        rhs = torch.zeros_like(lhs)
        sq = torch.zeros_like(lhs)
        for r0 in range(0, N, block):
            g = dv.view(B * H, N, d)[bh, r0:r0 + block].double()
            o = inp["do"].view(B * H, N, d)[bh, r0:r0 + block].double()
            lhs += g.sum(0)
            rhs += o.sum(0)
            sq += o.pow(2).sum(0)
        # a relative error e_i of row i's normaliser shifts the sum by sum_i e_i dO_i, of size
        # e * sqrt(sum_i dO_i^2) for independent rows; a dropped or wrong term shifts it by O(1)
        # in those units
        worst = max(worst, float(((lhs - rhs).abs() / sq.sqrt()).max()))
    m["sum_dv_eq_sum_dO"] = worst
    for name, x, gx in (("dq_orth_q", inp["q"], dq), ("dk_orth_k", inp["k"], dk)):
        xs_all = x.view(-1, d)
        gs_all = gx.view(-1, d)
        gmax = float(gs_all.abs().max().float())
        w_ = 0.0
        finite = True
        for r0 in range(0, xs_all.shape[0], block):
            xs = xs_all[r0:r0 + block].float()
            gs = gs_all[r0:r0 + block].float()
            finite = finite and bool(torch.isfinite(gs).all())
            xh = xs / xs.norm(dim=1, keepdim=True).clamp_min(1e-12)
            w_ = max(w_, float((xh * gs).sum(1).abs().max()))
            del xs, gs, xh
        m[name] = w_ / gmax if finite else float("inf")


def _prefix_check(inp, w, out, den, dq, heads, n, m):
    """Forward and dq on the first n rows of the given heads against the oracle."""
    BH = inp["q"].shape[0] * inp["q"].shape[1]
    W = to64(inp["W"])
    for bh in heads:
        sl = lambda t: to64(t.view(BH, *t.shape[2:])[bh, :n])
        o_ref, den_ref = oracle.forward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), W, w.tau, True)
        dq_ref, _, _ = oracle.backward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), W, sl(inp["do"]), w.tau, True)
        m["prefix_out_h%d" % bh] = rel_err(out.view(BH, -1, w.d)[bh, :n], o_ref)
        m["prefix_den_h%d" % bh] = rel_err(den.view(BH, -1)[bh, :n], den_ref)
        m["prefix_dq_h%d" % bh] = rel_err(dq.view(BH, -1, w.d)[bh, :n], dq_ref)


def _sampled_forward(inp, w, out, den, bh, nrows, m):
    N = w.N
    rows = np.unique(np.concatenate([np.linspace(0, N - 1, nrows).astype(np.int64),
                                     np.arange(min(256, N)), np.arange(max(0, N - 256), N)]))
    BH = inp["q"].shape[0] * inp["q"].shape[1]
    sl = lambda t: to64(t.view(BH, *t.shape[2:])[bh])
    o_ref, den_ref = oracle.forward(sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), to64(inp["W"]), w.tau,
                                    w.causal, rows=rows)
    ridx = torch.from_numpy(rows).to(DEV)
    m["sampled_out"] = rel_err(out.view(BH, N, w.d)[bh].index_select(0, ridx), o_ref)
    m["sampled_den"] = rel_err(den.view(BH, N)[bh].index_select(0, ridx), den_ref)


def _full_head(inp, w, bh, out, den, dq, dk, dv, m):
    """Every row of out, den, dq, dk and dv of head bh against the oracle on the whole
    sequence.  The oracle's inputs and results are fp64 copies on the host; the GPU results
    are compared one tensor at a time, so host memory stays near 12 fp64 copies of a head."""
    BH = w.B * w.H
    sl = lambda t: to64(t.view(BH, w.N, -1)[bh])
    q, k, v, do, W = sl(inp["q"]), sl(inp["k"]), sl(inp["v"]), sl(inp["do"]), to64(inp["W"])
    o_ref, den_ref = oracle.forward(q, k, v, W, w.tau, w.causal)
    m["h%d_out" % bh] = rel_err(out.view(BH, w.N, -1)[bh], o_ref)
    m["h%d_den" % bh] = rel_err(den.view(BH, w.N)[bh], den_ref)
    del o_ref, den_ref
    g_ref = oracle.backward(q, k, v, W, do, w.tau, w.causal)
    del q, k, v, do
    for nm, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), g_ref):
        m["h%d_%s" % (bh, nm)] = rel_err(got.view(BH, w.N, -1)[bh], ref)
    del g_ref
    gc.collect()


def _check(w, sampled=0, prefix_heads=(0,), prefix_n=4096, full_heads=()):
    """Run workload w on the GPU and collect error metrics; device memory is released before
    returning so a failing assertion does not keep ~100 GB alive."""
    m = {}
    inp = race_inputs.make_inputs(w, DEV)
    out, den, dq, dk, dv = _run(inp, w)
    try:
        for bh in full_heads:
            _full_head(inp, w, bh, out, den, dq, dk, dv, m)
        if sampled:
            _sampled_forward(inp, w, out, den, 0, sampled, m)
        if prefix_n:
            _prefix_check(inp, w, out, den, dq, list(prefix_heads), prefix_n, m)
        _identities(inp, dq, dk, dv, m)
        m["tail_finite"] = 0.0 if bool(torch.isfinite(out.view(-1, w.d)[-4:].float()).all()) else float("inf")
    finally:
        del inp, out, den, dq, dk, dv
        _free()
    return m


def test_c2_causal_b2h8_n64k_all_rows():
    """Workload c2 (B2 H8 N65536 d64 bf16, L16 P4 tau 0.5): every row of two heads."""
    w = race_inputs.WORKLOADS["c2_causal_b2h8_n64k"]
    m = _check(w, prefix_n=0, full_heads=(0, w.B * w.H - 1))
    assert max(m.values()) <= TOL, json.dumps(m)


def test_c3_causal_n4m_clusters_full_size():
    """Workload c3 (B1 H1 N=4,194,304 d64 bf16, clustered Q/K), the benchmark's workload in
    its launch configuration: every row of out, den, dq, dk and dv against the oracle."""
    m = _check(race_inputs.WORKLOADS["c3_causal_n4m_clusters"], prefix_n=0, full_heads=(0,))
    assert max(m.values()) <= TOL, json.dumps(m)


@pytest.mark.parametrize("N", race_inputs.SWEEP_N)
def test_c5_sequence_length_sweep(N):
    """Workload c5 (B1 H1 d64 bf16 L16 P4), N = 2^20, 2^22, 2^24 and 75,000,000.  Up to
    2^22 every output row is compared with the oracle; beyond, a causal prefix and the
    identities (the oracle would need minutes per pass)."""
    w = race_inputs.WORKLOADS["c5_sweep"].with_n(N)
    if N <= (1 << 22):
        m = _check(w, prefix_n=0, full_heads=(0,))
    else:
        m = _check(w, prefix_n=4096)
    assert max(m.values()) <= TOL, json.dumps(m)


def test_c4_causal_h4_n12m_d128():
    """Workload c4 (B1 H4 N=12,000,000 d128 bf16, L32 P5 = 1024 features, tau 0.5)."""
    w = race_inputs.WORKLOADS["c4_causal_h4_n12m_d128"]
    m = _check(w, prefix_heads=(0, 3), prefix_n=2048)
    assert max(m.values()) <= TOL, json.dumps(m)


def test_n1_noncausal_b2h8_n64k_all_rows():
    """Bidirectional (Algorithm 1) forward + backward, B2 H8 N65536 d64 bf16: every output of
    two whole heads."""
    w = race_inputs.WORKLOADS["n1_noncausal_b2h8_n64k"]
    m = _check(w, prefix_n=0, full_heads=(0, w.B * w.H - 1))
    assert max(m.values()) <= TOL, json.dumps(m)


def test_n1_noncausal_n4m_clusters_full_size():
    """Bidirectional forward + backward at N=4,194,304 (clustered Q/K): every row of out,
    den, dq, dk and dv against the oracle, and the gradient identities."""
    m = _check(race_inputs.WORKLOADS["n1_noncausal_n4m_clusters"], prefix_n=0, full_heads=(0,))
    assert max(m.values()) <= TOL, json.dumps(m)
