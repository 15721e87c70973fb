"""GPU parity of the streaming (decode-time) step and of the prefix statistics.

Algorithm 2 (zh §2.3) carries cumulative bucket statistics, so after a prompt of N0 tokens
(race_attn_state) each further token needs one step (race_attn_decode_step): the step's
outputs must be the causal forward's rows N0, N0+1, ... and the statistics after the last
step those of the whole sequence.  Both are compared with the fp64 oracle on the same
seeded inputs (oracle.forward with the causal rows, oracle.state).
"""
import numpy as np
import pytest
import torch

import linear_attention_soft_b200 as ra
import oracle
import race_inputs
from parity import TOL, rel_err, to64

pytestmark = pytest.mark.gpu

DEV = "cuda"

# (B, H, d, L, P), dtype, tau; the last two are hard sign hashing
CASES = [
    ((2, 3, 64, 16, 4), torch.bfloat16, 0.5),
    ((1, 2, 64, 16, 4), torch.float32, 0.5),
    ((1, 1, 128, 32, 5), torch.bfloat16, 0.25),
    ((2, 1, 16, 5, 1), torch.float32, 1.0),
    ((1, 1, 32, 16, 5), torch.float32, 0.5),
    ((1, 2, 32, 4, 3), torch.float32, 0.0),
    ((1, 1, 64, 16, 4), torch.bfloat16, 0.0),
]


def _run(shape, dtype, tau, n0, steps, seed):
    B, H, d, L, P = shape
    inp = race_inputs.small_normal(B, H, n0 + steps, d, L, P, seed, dtype=dtype, device=DEV, scale_qk=2.0)
    q, k, v, W = inp["q"], inp["k"], inp["v"], inp["W"]
    st = ra.state(k[:, :, :n0].contiguous(), v[:, :, :n0].contiguous(), W, tau)
    outs, dens = [], []
    for t in range(n0, n0 + steps):
        o, dn = ra.decode_step(q[:, :, t].contiguous(), k[:, :, t].contiguous(), v[:, :, t].contiguous(), W, st,
                               tau)
        outs.append(o)
        dens.append(dn)
    torch.cuda.synchronize()
    out = torch.stack(outs, 2)
    den = torch.stack(dens, 2)
    q64, k64, v64, W64 = (to64(x) for x in (q, k, v, W))
    o_ref, den_ref = oracle.forward(q64, k64, v64, W64, tau, True, rows=np.arange(n0, n0 + steps))
    h_ref = oracle.state(k64, v64, W64, tau).reshape(B * H, L << P, d + 1)
    return {"out": rel_err(out, o_ref), "den": rel_err(den, den_ref), "state": rel_err(st, h_ref)}


@pytest.mark.parametrize("shape,dtype,tau", CASES)
def test_prompt_then_steps_match_causal_rows(shape, dtype, tau):
    errs = _run(shape, dtype, tau, n0=300, steps=24, seed=sum(shape) + int(4 * tau))
    assert max(errs.values()) <= TOL[dtype], errs


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_steps_from_an_empty_prompt(dtype):
    """An empty prompt is the zero state; the first step reads only its own key."""
    errs = _run((1, 2, 64, 16, 4), dtype, 0.5, n0=0, steps=40, seed=7)
    assert max(errs.values()) <= TOL[dtype], errs


def test_many_heads_one_cta_per_head():
    """B*H large enough that each head's rows stay in one CTA."""
    errs = _run((16, 40, 64, 16, 4), torch.bfloat16, 0.5, n0=64, steps=3, seed=8)
    assert max(errs.values()) <= TOL[torch.bfloat16], errs


def test_prompt_statistics_at_size():
    """race_attn_state over N = 262,144 tokens (the tensor-core segment totals for this
    shape) against the oracle's statistics."""
    w = race_inputs.WORKLOADS["c5_sweep"].with_n(1 << 18)
    inp = race_inputs.make_inputs(w, DEV)
    st = ra.state(inp["k"], inp["v"], inp["W"], w.tau)
    torch.cuda.synchronize()
    h_ref = oracle.state(to64(inp["k"]), to64(inp["v"]), to64(inp["W"]), w.tau).reshape(1, w.L << w.P, w.d + 1)
    assert rel_err(st, h_ref) <= TOL[torch.bfloat16]


def test_decode_rejects_bad_arguments():
    B, H, d, L, P = 1, 1, 64, 16, 4
    x = torch.zeros((B, H, d), dtype=torch.bfloat16, device=DEV)
    W = torch.zeros((L, P, d), dtype=torch.float32, device=DEV)
    st = torch.zeros((B * H, L << P, d + 1), dtype=torch.float32, device=DEV)
    ws = torch.empty(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(ra.RaceError) as e:
        ra.race_attn_decode_step(x, x, x, W, st, x, None, 0.5, ws)
    assert e.value.status == ra.RACE_ERR_WORKSPACE
    with pytest.raises(ra.RaceError) as e:
        ra.race_attn_decode_step(x, x, x, W, st, x, None, -1.0, ws)
    assert e.value.status == ra.RACE_ERR_INVALID_ARG
