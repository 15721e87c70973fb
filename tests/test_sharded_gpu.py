"""GPU parity of the sequence-sharded passes, with the shards run one after another on one
device: every shard's first half, the library's shard combine on the side-by-side totals
(what an all-gather leaves), every shard's second half.  The concatenated outputs and
gradients must match the oracle on the whole sequence (Algorithm 2, zh §2.3: the
statistics are sums over tokens, so a shard needs only the other shards' totals)."""
import pytest
import torch

import linear_attention_soft_b200 as ra
import race_inputs
from parity import TOL, oracle_backward, oracle_forward, rel_err

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _sharded(inp, bounds, tau, causal):
    q, k, v, W, do = (inp[n] for n in ("q", "k", "v", "W", "do"))
    B, H, N, d = q.shape
    L, P = W.shape[0], W.shape[1]
    code = ra.RACE_F32 if q.dtype == torch.float32 else ra.RACE_BF16
    sh = []
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        s = {n: inp[n][:, :, lo:hi].contiguous() for n in ("q", "k", "v", "do")}
        n = hi - lo
        s["ctx"] = torch.empty(max(ra.race_attn_ctx_size(B, H, n, d, L, P, causal) // 4, 4), dtype=torch.float32,
                               device=DEV)
        s["wsf"] = torch.empty(max(ra.race_attn_workspace_size(B, H, n, d, L, P, causal, 0, code), 16),
                               dtype=torch.uint8, device=DEV)
        s["wsb"] = torch.empty(max(ra.race_attn_workspace_size(B, H, n, d, L, P, causal, 1, code), 16),
                               dtype=torch.uint8, device=DEV)
        sh.append(s)
    shape = (B * H, L << P, d + 1)
    ht = torch.empty((len(sh),) + shape, dtype=torch.float32, device=DEV)
    for i, s in enumerate(sh):
        ra.race_attn_forward_begin(s["k"], s["v"], W, s["ctx"], ht[i], tau, causal, s["wsf"])
    for i, s in enumerate(sh):
        h_init = torch.empty(shape, dtype=torch.float32, device=DEV)
        ra.race_attn_shard_combine(ht, i, 0 if causal else 2, h_init)
        s["out"] = torch.empty_like(s["q"])
        s["den"] = torch.empty(s["q"].shape[:3], dtype=torch.float32, device=DEV)
        ra.race_attn_forward_end(s["q"], s["k"], s["v"], W, h_init, s["out"], s["den"], s["ctx"], tau, causal,
                                 s["wsf"])
    gt = torch.empty_like(ht)
    for i, s in enumerate(sh):
        s["dq"] = torch.empty_like(s["q"])
        ra.race_attn_backward_begin(s["q"], s["k"], s["v"], W, s["out"], s["den"], s["do"], s["ctx"], None,
                                    s["dq"], gt[i], tau, causal, s["wsb"])
    for i, s in enumerate(sh):
        g_init = torch.empty(shape, dtype=torch.float32, device=DEV)
        ra.race_attn_shard_combine(gt, i, 1 if causal else 2, g_init)
        s["dk"], s["dv"] = torch.empty_like(s["k"]), torch.empty_like(s["v"])
        ra.race_attn_backward_end(s["q"], s["k"], s["v"], W, s["out"], s["den"], s["do"], g_init, s["dk"], s["dv"],
                                  tau, causal, s["wsb"])
    torch.cuda.synchronize()
    return {n: torch.cat([s[n] for s in sh], 2) for n in ("out", "den", "dq", "dk", "dv")}


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("dtype,shape,bounds", [
    (torch.bfloat16, (1, 2, 1000, 64, 16, 4), (0, 384, 640, 1000)),   # tensor-core path, ragged shards
    (torch.bfloat16, (1, 1, 700, 64, 16, 4), (0, 0, 300, 700)),       # an empty shard
    (torch.float32, (1, 2, 520, 32, 4, 3), (0, 130, 520)),            # general path
])
def test_sharded_passes_match_the_whole_sequence(dtype, shape, bounds, causal):
    B, H, N, d, L, P = shape
    inp = race_inputs.small_normal(B, H, N, d, L, P, seed=N + len(bounds), dtype=dtype, device=DEV, scale_qk=2.0)
    got = _sharded(inp, bounds, 0.5, causal)
    o_ref, den_ref = oracle_forward(inp, 0.5, causal)
    dq_ref, dk_ref, dv_ref = oracle_backward(inp, 0.5, causal)
    errs = {"out": rel_err(got["out"], o_ref), "den": rel_err(got["den"], den_ref), "dq": rel_err(got["dq"], dq_ref),
            "dk": rel_err(got["dk"], dk_ref), "dv": rel_err(got["dv"], dv_ref)}
    assert max(errs.values()) <= TOL[dtype], errs


def test_one_shard_equals_the_single_call():
    """begin + end with no other shards is the one-call pass, bit for bit."""
    inp = race_inputs.small_normal(1, 2, 900, 64, 16, 4, seed=3, dtype=torch.bfloat16, device=DEV)
    got = _sharded(inp, (0, 900), 0.5, True)
    out, den, ctx = ra.forward(inp["q"], inp["k"], inp["v"], inp["W"], 0.5, True, save_ctx=True)
    dq, dk, dv = ra.backward(inp["q"], inp["k"], inp["v"], inp["W"], out, den, inp["do"], 0.5, True, ctx=ctx)
    torch.cuda.synchronize()
    for n, ref in (("out", out), ("den", den), ("dq", dq), ("dk", dk), ("dv", dv)):
        assert torch.equal(got[n], ref), n


def test_driver_on_one_rank_equals_the_single_call():
    """linear_attention_soft_b200.sharded through a one-rank NCCL group: the exchange leaves
    zero statistics from other shards, so the result is the single-call pass bit for bit."""
    import os
    import socket

    import torch.distributed as dist

    from linear_attention_soft_b200 import sharded

    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device(DEV, 0))
    try:
        inp = race_inputs.small_normal(1, 2, 900, 64, 16, 4, seed=4, dtype=torch.bfloat16, device=DEV)
        q, k, v, W, do = (inp[n] for n in ("q", "k", "v", "W", "do"))
        out, den, ctx = sharded.forward(q, k, v, W, 0.5, True)
        dq, dk, dv = sharded.backward(q, k, v, W, out, den, do, 0.5, True, ctx)
        ro, rd, rc = ra.forward(q, k, v, W, 0.5, True, save_ctx=True)
        rq, rk, rv = ra.backward(q, k, v, W, ro, rd, do, 0.5, True, ctx=rc)
        torch.cuda.synchronize()
        for a, b in ((out, ro), (den, rd), (dq, rq), (dk, rk), (dv, rv)):
            assert torch.equal(a, b)
    finally:
        dist.destroy_process_group()
