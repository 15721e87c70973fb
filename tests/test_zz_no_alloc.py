"""The allocation-free forward (race_attn_forward_noalloc) against the regular forward and the
fp64 oracle.

Some callers cannot allocate device memory (their device memory belongs to a host
framework's allocator, or they cannot afford the synchronisation an allocation may cause),
so this entry point keeps its scratch in a fixed buffer inside the library.  The test calls
it through the C ABI twice in a row per case, on different inputs, and compares each result
with race_attn_forward given its own workspace and with the oracle, on the tensor-core paths
(bf16 d64 L16 P4; bf16 d128 L32 P5 causal, the feature-group path) and on the general path
(fp32, and bf16 bidirectional with 1,024 features over a thread-block cluster).  After the first call it checks that further calls change neither
the device's free memory nor torch's allocations, and that sizes needing more scratch than
the fixed buffer are refused before anything runs.  This file is collected last so a
failure here comes after every other test has run.
"""
import pytest
import torch

import linear_attention_soft_b200 as ra
import oracle
import race_inputs
from parity import TOL, rel_err, to64

pytestmark = pytest.mark.gpu

# (B, H, N, d, L, P, tau, causal, dtype): tensor-core path causal and bidirectional, the
# general fp32 path, the feature-group tensor-core path (d128 L32 P5 causal) and the general
# bf16 path with L * 2^P = 1024 features (bidirectional: 8 cluster CTAs)
CASES = [
    (1, 2, 3000, 64, 16, 4, 0.5, True, torch.bfloat16),
    (2, 1, 1300, 64, 16, 4, 0.5, False, torch.bfloat16),
    (1, 2, 2500, 64, 8, 4, 1.0, True, torch.float32),
    (2, 1, 1000, 32, 8, 3, 0.5, False, torch.float32),
    (1, 1, 1500, 128, 32, 5, 0.5, True, torch.bfloat16),
    (1, 1, 1200, 128, 32, 5, 0.5, False, torch.bfloat16),
]


def _inputs(case, seed):
    B, H, N, d, L, P, tau, causal, dtype = case
    return race_inputs.small_normal(B, H, N, d, L, P, seed, dtype=dtype, device="cuda")


def _noalloc(inp, tau, causal, out, den):
    out.fill_(float("nan"))
    den.fill_(float("nan"))
    ra.race_attn_forward_noalloc(inp["q"], inp["k"], inp["v"], inp["W"], out, den, tau, causal)


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dN%d_d%dL%dP%d_%s_%s" % (
    c[0], c[1], c[2], c[3], c[4], c[5], "causal" if c[7] else "bidir", str(c[8]).split(".")[-1]))
def test_noalloc_forward_matches_the_workspace_forward_and_the_oracle(case):
    B, H, N, d, L, P, tau, causal, dtype = case
    tol = TOL[dtype]
    for call, seed in enumerate((21, 22)):  # two calls in a row on different inputs
        inp = _inputs(case, seed + 10 * L)
        ref_out, ref_den, _ = ra.forward(inp["q"], inp["k"], inp["v"], inp["W"], tau, causal)
        out = torch.empty_like(inp["q"])
        den = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
        _noalloc(inp, tau, causal, out, den)
        torch.cuda.synchronize()
        o_ref, den_ref = oracle.forward(to64(inp["q"]), to64(inp["k"]), to64(inp["v"]), to64(inp["W"]),
                                        tau, causal)
        errs = {"out_vs_forward": rel_err(out, to64(ref_out)), "den_vs_forward": rel_err(den, to64(ref_den)),
                "out_vs_oracle": rel_err(out, o_ref), "den_vs_oracle": rel_err(den, den_ref)}
        assert max(errs.values()) <= tol, (call, errs)


def test_noalloc_forward_allocates_nothing_after_its_first_call():
    case = CASES[0]
    B, H, N, d, L, P, tau, causal, dtype = case
    inputs = [_inputs(case, s) for s in (31, 32)]
    out = torch.empty_like(inputs[0]["q"])
    den = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    _noalloc(inputs[0], tau, causal, out, den)  # the warm-up call
    torch.cuda.synchronize()
    free0, allocated0 = torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated()
    for i in range(6):
        _noalloc(inputs[i & 1], tau, causal, out, den)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == allocated0
    assert bool(torch.isfinite(out).all()) and bool(torch.isfinite(den).all())


def test_noalloc_forward_refuses_sizes_beyond_its_buffer():
    B, H, N, d, L, P = 64, 16, 1 << 16, 64, 16, 4
    need = ra.race_attn_workspace_size(B, H, N, d, L, P, True, 0, ra.RACE_BF16)
    assert need > ra.RACE_NOALLOC_SCRATCH_BYTES
    lib = ra.load_library()
    rc = lib.race_attn_forward_noalloc(16, 16, 16, 16, 16, 16, B, H, N, d, L, P, 0.5, 1, ra.RACE_BF16, None)
    assert rc == ra.RACE_ERR_WORKSPACE
