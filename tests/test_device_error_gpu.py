"""Failure detection without a GPU fault: a kernel wait that runs out is reported to the host
and leaves the CUDA context usable (the wait is bounded by time, on a barrier nothing
arrives on)."""
import pytest
import torch

import linear_attention_soft_b200 as ra
import race_inputs
from parity import TOL, gpu_forward, oracle_forward, rel_err

pytestmark = pytest.mark.gpu


def test_timed_out_wait_is_reported_and_the_context_survives():
    assert ra.race_attn_device_error() == 0
    ra.race_attn_selftest_wait_timeout(1_000_000)  # 1 ms
    assert ra.race_attn_device_error() == 1
    assert ra.race_attn_device_error() == 0        # cleared by the read
    inp = race_inputs.small_normal(1, 1, 500, 64, 16, 4, 31, dtype=torch.bfloat16, device="cuda")
    out, den, _ = gpu_forward(inp, 0.5, True)
    torch.cuda.synchronize()
    assert ra.race_attn_device_error() == 0
    o_ref, _ = oracle_forward(inp, 0.5, True)
    assert rel_err(out, o_ref) <= TOL[torch.bfloat16]


def test_selftest_rejects_bad_limits():
    with pytest.raises(ra.RaceError):
        ra.race_attn_selftest_wait_timeout(0)
    with pytest.raises(ra.RaceError):
        ra.race_attn_selftest_wait_timeout(10 ** 10)
