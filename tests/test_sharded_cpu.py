"""The exchange of the sequence-sharded passes on CPU (gloo, 3 ranks): every rank holds a
contiguous slice of one sequence; the forward must start rank s from the key statistics of
the tokens before its slice (bidirectional: of every other slice) and the backward's key
side from the query statistics of the ranks after it.  The library calls are replaced by a
CPU stand-in: the statistics come from the fp64 oracle, and the test checks what the
driver hands to the second half of each pass."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SPLIT = (0, 37, 80, 128)  # uneven slices of N = 128 tokens


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class _StandIn:
    """CPU stand-in for the library: statistics from the oracle, shard sums in numpy."""

    def __init__(self, oracle, tau, rank):
        self.oracle, self.tau, self.rank = oracle, tau, rank
        self.seen = {}

    def forward_begin(self, k, v, W, ctx, h_total, tau, causal, ws):
        h = self.oracle.state(k.double().numpy(), v.double().numpy(), W.double().numpy(), tau)
        h_total.copy_(torch.from_numpy(h.reshape(h_total.shape)).float())

    def forward_end(self, q, k, v, W, h_init, out, den, ctx, tau, causal, ws):
        self.seen["h_init"] = h_init.double().numpy().copy()
        out.zero_()
        den.zero_()

    def backward_begin(self, q, k, v, W, out, den, dout, ctx, dq, g_total, tau, causal, ws):
        g_total.fill_(float(self.rank + 1))  # a value that names the rank
        dq.zero_()

    def backward_end(self, q, k, v, W, out, den, dout, g_init, dk, dv, tau, causal, ws):
        self.seen["g_init"] = g_init.double().numpy().copy()
        dk.zero_()
        dv.zero_()

    def combine(self, gathered, shard, which, out):
        acc = torch.zeros_like(out, dtype=torch.float64)
        for s in range(gathered.shape[0]):
            if (which == 0 and s < shard) or (which == 1 and s > shard) or (which == 2 and s != shard):
                acc += gathered[s].double()
        out.copy_(acc.float())


def _rank_main(rank, world, port, causal, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import race_inputs
        from linear_attention_soft_b200 import sharded
        inp = race_inputs.small_normal(1, 2, SPLIT[-1], 16, 4, 3, 11)
        lo, hi = SPLIT[rank], SPLIT[rank + 1]
        sl = {n: inp[n][:, :, lo:hi].contiguous() for n in ("q", "k", "v", "do")}
        lib = _StandIn(oracle, 0.5, rank)
        o, den, ctx = sharded.forward(sl["q"], sl["k"], sl["v"], inp["W"], 0.5, causal, lib=lib)
        sharded.backward(sl["q"], sl["k"], sl["v"], inp["W"], o, den, sl["do"], 0.5, causal, ctx, lib=lib)
        out[rank] = (lib.seen["h_init"], lib.seen["g_init"])
    finally:
        dist.barrier()
        dist.destroy_process_group()


@pytest.mark.parametrize("causal", [True, False])
def test_three_rank_exchange(causal):
    import oracle
    import race_inputs
    world = 3
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), causal, out), nprocs=world,
                       start_method="spawn", join=True)
    inp = race_inputs.small_normal(1, 2, SPLIT[-1], 16, 4, 3, 11)
    k, v, W = (inp[n].double().numpy() for n in ("k", "v", "W"))
    for r in range(world):
        h_init, g_init = out[r]
        lo, hi = SPLIT[r], SPLIT[r + 1]
        # keys the rank must start from: those before its slice, or all but its own
        if causal:
            want = oracle.state(k[:, :, :lo], v[:, :, :lo], W, 0.5)
        else:
            keep = np.r_[0:lo, hi:SPLIT[-1]]
            want = oracle.state(k[:, :, keep], v[:, :, keep], W, 0.5)
        np.testing.assert_allclose(h_init, want.reshape(h_init.shape), rtol=1e-5, atol=1e-4)
        # queries the key side must start from: ranks after it, or all but itself
        others = range(r + 1, world) if causal else [s for s in range(world) if s != r]
        np.testing.assert_array_equal(g_init, np.full(g_init.shape, float(sum(s + 1 for s in others))))
