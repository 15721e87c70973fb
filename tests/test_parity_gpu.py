"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle on the same
seeded inputs, element by element, at sizes the oracle finishes in seconds.

Tolerance (normwise max relative error, max|gpu - oracle| / max|oracle|): 1e-4 for fp32
inputs, 2e-2 for bf16 inputs with fp32 accumulation; sign-hash bucket indices bit-exact
wherever no projection lies within 1e-5 of zero.
"""
import numpy as np
import pytest
import torch

import oracle
import linear_attention_soft_b200 as ra
import race_inputs
from parity import (TOL, gpu_backward, gpu_forward, oracle_backward, oracle_forward,
                    projection_margin, rel_err, to64)

pytestmark = pytest.mark.gpu

DEV = "cuda"

# (B, H, N, d, L, P): several chunks and segments with a ragged tail; cluster sizes
# G = ceil(L*2^P / 128) of 1, 2 and 8; d of 16..128; P of 1..5.
SHAPES = [
    (1, 2, 1000, 64, 16, 4),
    (2, 1, 700, 64, 8, 4),
    (1, 1, 300, 128, 32, 5),
    (1, 3, 257, 32, 3, 2),
    (1, 1, 2125, 64, 16, 4),
    (1, 1, 129, 16, 5, 1),
    (1, 1, 97, 128, 4, 3),
]


def make(shape, dtype, seed, scale_qk=1.0):
    B, H, N, d, L, P = shape
    return race_inputs.small_normal(B, H, N, d, L, P, seed, dtype=dtype, device=DEV,
                                    scale_qk=scale_qk)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", SHAPES)
def test_forward_backward_match_oracle(shape, dtype, causal):
    inp = make(shape, dtype, seed=hash(shape) % 1000, scale_qk=2.0)
    tau = 0.5
    out, den, _ = gpu_forward(inp, tau, causal)
    dq, dk, dv = gpu_backward(inp, out, den, tau, causal)
    torch.cuda.synchronize()
    o_ref, den_ref = oracle_forward(inp, tau, causal)
    dq_ref, dk_ref, dv_ref = oracle_backward(inp, tau, causal)
    tol = TOL[dtype]
    errs = {"out": rel_err(out, o_ref), "den": rel_err(den, den_ref), "dq": rel_err(dq, dq_ref),
            "dk": rel_err(dk, dk_ref), "dv": rel_err(dv, dv_ref)}
    assert all(e <= tol for e in errs.values()), errs


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_single_token_and_one_chunk_edges(dtype):
    tol = TOL[dtype]
    bad = {}
    for N in (1, 2, 31, 32, 33, 127, 128, 129, 512, 513):
        inp = make((1, 1, N, 64, 16, 4), dtype, seed=N)
        out, den, _ = gpu_forward(inp, 0.5, True)
        dq, dk, dv = gpu_backward(inp, out, den, 0.5, True)
        o_ref, den_ref = oracle_forward(inp, 0.5, True)
        dq_ref, dk_ref, dv_ref = oracle_backward(inp, 0.5, True)
        # with one token, out_0 = v_0 whatever q and k are: dq = dk = 0 exactly, so the
        # error is measured against the scale of dO instead
        fl = 1e-2 * float(inp["do"].abs().max())
        errs = {"out": rel_err(out, o_ref), "den": rel_err(den, den_ref), "dq": rel_err(dq, dq_ref, fl),
                "dk": rel_err(dk, dk_ref, fl), "dv": rel_err(dv, dv_ref)}
        if N == 1:  # causal row 0 reads only its own key: out_0 = v_0
            errs["out0_is_v0"] = rel_err(out[0, 0, 0], to64(inp["v"])[0, 0, 0])
        if max(errs.values()) > tol:
            bad[N] = errs
    assert not bad, bad


def test_empty_sequence_is_a_no_op():
    inp = make((1, 1, 0, 64, 16, 4), torch.bfloat16, seed=0)
    out, den, _ = gpu_forward(inp, 0.5, True)
    dq, dk, dv = gpu_backward(inp, out, den, 0.5, True)
    assert out.numel() == 0 and dq.numel() == 0


def test_c1_noncausal_forward_f32():
    """Workload c1: B1 H1 N1024 d64 fp32, L8 P4 tau 1, unit-norm Q/K, bidirectional."""
    w = race_inputs.WORKLOADS["c1_noncausal_fwd_f32"]
    inp = race_inputs.make_inputs(w, DEV, with_grad_out=True)
    out, den, _ = gpu_forward(inp, w.tau, w.causal)
    o_ref, den_ref = oracle_forward(inp, w.tau, w.causal)
    assert rel_err(out, o_ref) <= 1e-4
    assert rel_err(den, den_ref) <= 1e-4
    dq, dk, dv = gpu_backward(inp, out, den, w.tau, w.causal)
    dq_ref, dk_ref, dv_ref = oracle_backward(inp, w.tau, w.causal)
    assert max(rel_err(dq, dq_ref), rel_err(dk, dk_ref), rel_err(dv, dv_ref)) <= 1e-4


@pytest.mark.parametrize("causal", [True, False])
def test_general_path_at_short_lengths_is_repeatable(causal):
    """At short lengths the general path splits each segment's aggregate over a cluster of
    CTAs (and the bidirectional read-out over one CTA per chunk); the partial sums are added
    in a fixed order, so two runs agree bit for bit (fp32, two feature groups, two heads)."""
    inp = make((1, 2, 1000, 64, 16, 4), torch.float32, seed=77, scale_qk=2.0)
    runs = []
    for _ in range(2):
        out, den, _ = gpu_forward(inp, 0.5, causal)
        grads = gpu_backward(inp, out, den, 0.5, causal)
        torch.cuda.synchronize()
        runs.append((out, den) + tuple(grads))
    assert all(torch.equal(a, b) for a, b in zip(*runs))
    o_ref, den_ref = oracle_forward(inp, 0.5, causal)
    assert max(rel_err(runs[0][0], o_ref), rel_err(runs[0][1], den_ref)) <= TOL[torch.float32]


def _margined_inputs(shape, dtype, seed, margin=1e-3):
    """Inputs whose q/k rows keep every hyperplane projection away from zero, so fp32 and
    fp64 agree on every sign (rows failing the margin are redrawn)."""
    inp = make(shape, dtype, seed)
    W = to64(inp["W"])
    g = torch.Generator(device=DEV)
    g.manual_seed(seed + 1)
    for name in ("q", "k"):
        x = inp[name]
        for _ in range(50):
            bad = torch.from_numpy(projection_margin(to64(x), W) < margin).to(DEV)
            if not bool(bad.any()):
                break
            x = torch.where(bad[..., None], torch.randn(x.shape, generator=g, device=DEV).to(dtype), x)
        inp[name] = x.contiguous()
    return inp


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_hard_hash_forward(dtype, causal):
    """tau = 0: one-hot sign hashing; rows with no key in any of their buckets read 0."""
    inp = _margined_inputs((1, 2, 600, 64, 4, 3), dtype, seed=5)
    out, den, _ = gpu_forward(inp, 0.0, causal)
    o_ref, den_ref = oracle_forward(inp, 0.0, causal)
    np.testing.assert_array_equal(to64(den), den_ref)  # bucket counts are small integers
    assert rel_err(out, o_ref) <= TOL[dtype]
    if causal:
        z = den_ref == 0
        assert np.all(to64(out)[z] == 0)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_hash_indices_bit_exact(dtype):
    import linear_attention_soft_b200 as ra
    inp = make((2, 2, 500, 64, 16, 4), dtype, seed=9)
    x, W = inp["q"], inp["W"]
    idx = torch.empty((2, 2, 500, 16), dtype=torch.int32, device=DEV)
    ra.race_attn_hash_indices(x, W, idx)
    ref = oracle.hash_indices(to64(x), to64(W))
    xh = to64(x)
    proj = np.einsum("lpd,...d->...lp", to64(W), xh / np.linalg.norm(xh, axis=-1, keepdims=True))
    clear = (np.abs(proj) > 1e-5 * np.linalg.norm(to64(W), axis=-1)).all(-1)
    assert clear.mean() > 0.999
    np.testing.assert_array_equal(idx.cpu().numpy()[clear], ref[clear])


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("causal", [True, False])
def test_saved_ctx_backward_matches_recomputed(causal, dtype):
    """The forward can hand its segment statistics to the backward (ctx); with or without
    them the gradients match the oracle, and each other to rounding."""
    inp = make((1, 2, 3000, 64, 16, 4), dtype, seed=11)
    out, den, ctx = gpu_forward(inp, 0.5, causal, save_ctx=True)
    a = gpu_backward(inp, out, den, 0.5, causal, ctx=ctx)
    b = gpu_backward(inp, out, den, 0.5, causal)
    ref = oracle_backward(inp, 0.5, causal)
    for x, y, r in zip(a, b, ref):
        assert rel_err(x, r) <= TOL[dtype] and rel_err(y, r) <= TOL[dtype]
        assert rel_err(x, to64(y)) <= TOL[dtype]


def test_causal_output_ignores_later_tokens():
    inp = make((1, 1, 3000, 64, 16, 4), torch.bfloat16, seed=12)
    out, den, _ = gpu_forward(inp, 0.5, True)
    inp2 = {k: v.clone() for k, v in inp.items()}
    cut = 1777
    inp2["k"][..., cut:, :] = torch.randn_like(inp2["k"][..., cut:, :].float()).to(torch.bfloat16)
    inp2["v"][..., cut:, :] = 0
    out2, den2, _ = gpu_forward(inp2, 0.5, True)
    torch.cuda.synchronize()
    # the chunked scan sums the same prefix in the same order whatever follows
    assert torch.equal(out[..., :cut, :], out2[..., :cut, :])
    assert torch.equal(den[..., :cut], den2[..., :cut])


@pytest.mark.parametrize("shape", [(1, 1, 700, 64, 16, 4), (1, 1, 300, 128, 16, 5)])
def test_sixteen_byte_aligned_buffers_take_the_general_path(shape):
    """The tensor-core paths move rows in 32-byte accesses; with tensors only 16-byte aligned
    (valid for the ABI) the library runs the general path, with the same results."""
    B, H, N, d, L, P = shape
    inp = make(shape, torch.bfloat16, seed=77, scale_qk=2.0)

    def off16(t):  # the same values at an address 16 bytes past a 32-byte boundary
        raw = torch.empty(t.numel() + 16, dtype=t.dtype, device=DEV)
        v = raw[8:8 + t.numel()].view(t.shape)
        v.copy_(t)
        return v

    shifted = {n: (off16(x) if n != "W" else x) for n, x in inp.items()}
    assert shifted["q"].data_ptr() % 32 == 16
    ra.race_attn_profile_reset()
    ra.race_attn_profile_enable(True)
    out, den, _ = gpu_forward(shifted, 0.5, True)
    dq, dk, dv = gpu_backward(shifted, out, den, 0.5, True)
    torch.cuda.synchronize()
    prof = ra.race_attn_profile_read()
    ra.race_attn_profile_enable(False)
    assert not any(n.startswith(("tc_", "wide_")) for n in prof), prof
    o_ref, den_ref = oracle_forward(inp, 0.5, True)
    dq_ref, dk_ref, dv_ref = oracle_backward(inp, 0.5, True)
    errs = {"out": rel_err(out, o_ref), "den": rel_err(den, den_ref), "dq": rel_err(dq, dq_ref),
            "dk": rel_err(dk, dk_ref), "dv": rel_err(dv, dv_ref)}
    assert max(errs.values()) <= TOL[torch.bfloat16], errs
