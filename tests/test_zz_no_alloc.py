"""The allocation-free forward (race_attn_forward_noalloc) against the regular forward.

Some callers cannot allocate device memory (their device memory belongs to a host
framework's allocator, or they cannot afford the synchronisation an allocation may cause),
so this entry point keeps its scratch in a fixed buffer inside the library.  The test calls
it through the C ABI twice in a row, on different inputs, and compares each result with
race_attn_forward given its own workspace; it also checks that sizes needing more scratch
than the fixed buffer are refused before anything runs.  This file is collected last so a
failure here comes after every other test has run.
"""
import pytest
import torch

import linear_attention_soft_b200 as ra
import race_inputs
from parity import TOL, rel_err, to64

pytestmark = pytest.mark.gpu


def test_noalloc_forward_matches_the_workspace_forward_on_consecutive_calls():
    for seed, causal, shape in ((21, True, (1, 2, 3000)), (22, False, (2, 1, 1300))):
        B, H, N = shape
        inp = race_inputs.small_normal(B, H, N, 64, 16, 4, seed, dtype=torch.bfloat16, device="cuda")
        ref_out, ref_den, _ = ra.forward(inp["q"], inp["k"], inp["v"], inp["W"], 0.5, causal)
        out = torch.full_like(inp["q"], float("nan"))
        den = torch.full((B, H, N), float("nan"), dtype=torch.float32, device="cuda")
        ra.race_attn_forward_noalloc(inp["q"], inp["k"], inp["v"], inp["W"], out, den, 0.5, causal)
        torch.cuda.synchronize()
        assert rel_err(out, to64(ref_out)) <= TOL[torch.bfloat16]
        assert rel_err(den, to64(ref_den)) <= TOL[torch.bfloat16]


def test_noalloc_forward_refuses_sizes_beyond_its_buffer():
    B, H, N, d, L, P = 64, 16, 1 << 16, 64, 16, 4
    need = ra.race_attn_workspace_size(B, H, N, d, L, P, True, 0, ra.RACE_BF16)
    assert need > ra.RACE_NOALLOC_SCRATCH_BYTES
    lib = ra.load_library()
    rc = lib.race_attn_forward_noalloc(16, 16, 16, 16, 16, 16, B, H, N, d, L, P, 0.5, 1, ra.RACE_BF16, None)
    assert rc == ra.RACE_ERR_WORKSPACE
