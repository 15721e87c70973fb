"""The benchmark's multi-rank path on CPU (gloo, world size 2): every rank gets its own
independent sequence, the job time is the slowest rank's and the throughput counts every
rank's tokens.  The per-rank work here is the fp64 oracle on a tiny causal problem, so the
whole path runs without a GPU."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        import race_inputs
        w = race_inputs.WORKLOADS["c5_sweep"].with_n(64)
        wr = bench.rank_workload(w, rank)
        inp = race_inputs.make_inputs(wr, "cpu")
        o, _ = oracle.forward(inp["q"][0, 0].double().numpy(), inp["k"][0, 0].double().numpy(),
                              inp["v"][0, 0].double().numpy(), inp["W"].double().numpy(), w.tau, True)
        ms_local = 10.0 * (rank + 1)  # rank 1 is the slow one
        ms, tps = bench.job_throughput(ms_local, w.B * w.N, world)
        out[rank] = (float(o.sum()), ms, tps, wr.seed)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_weak_scaling_bookkeeping():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, start_method="spawn",
                       join=True)
    (s0, ms0, tps0, seed0), (s1, ms1, tps1, seed1) = out[0], out[1]
    assert seed0 != seed1 and s0 != s1          # independent sequences per rank
    assert ms0 == ms1 == 20.0                   # max over ranks
    assert np.isclose(tps0, 2 * 64 / 0.020)     # all ranks' tokens over the slowest time
    assert tps0 == tps1


class _StatsStandIn:
    """CPU stand-in for the library in the sharded passes: the key statistics of a slice from
    the fp64 oracle, the combine in rank order; records what each rank is handed."""

    def __init__(self, oracle):
        self.oracle = oracle
        self.seen = {}

    def forward_begin(self, k, v, W, ctx, h_total, tau, causal, ws):
        h = self.oracle.state(k.double().numpy(), v.double().numpy(), W.double().numpy(), tau)
        h_total.copy_(torch.from_numpy(h.reshape(h_total.shape)).float())

    def forward_end(self, q, k, v, W, h_init, out, den, ctx, tau, causal, ws):
        self.seen["h_init"] = h_init.double().numpy().copy()
        out.zero_()
        den.fill_(1.0)

    def backward_begin(self, q, k, v, W, out, den, dout, ctx, dq, g_total, tau, causal, ws):
        g_total.zero_()
        dq.zero_()

    def backward_end(self, q, k, v, W, out, den, dout, g_init, dk, dv, tau, causal, ws):
        dk.zero_()
        dv.zero_()

    def combine(self, gathered, shard, which, out):
        acc = torch.zeros_like(out, dtype=torch.float64)
        for s in range(gathered.shape[0]):
            if (which == 0 and s < shard) or (which == 1 and s > shard) or (which == 2 and s != shard):
                acc += gathered[s].double()
        out.copy_(acc.float())


def _sharded_rank_main(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        import race_inputs
        w = race_inputs.WORKLOADS["c5_sweep"].with_n(96)
        inp = bench.shard_inputs(w, rank, "cpu")
        lib = _StatsStandIn(oracle)
        res = bench.sharded_step(inp, w, lib=lib)
        ms, tps = bench.job_throughput(5.0 + rank, w.B * w.N, world)
        out[rank] = (inp["W"].numpy().copy(), inp["q"].float().numpy().copy(), lib.seen["h_init"],
                     [tuple(t.shape) for t in res], ms, tps)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_rank_sharded_sequence_bookkeeping():
    """bench.py's default multi-rank mode: the ranks hold consecutive slices of one sequence
    (the same hyperplanes W, their own rows), rank 1 starts its causal scan from the key
    statistics of rank 0's slice, and the job throughput counts both slices over the slower
    rank's time."""
    import bench
    import oracle
    import race_inputs
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_sharded_rank_main, args=(world, _free_port(), out), nprocs=world,
                       start_method="spawn", join=True)
    (W0, q0, h0, shapes0, ms0, tps0), (W1, q1, h1, shapes1, ms1, tps1) = out[0], out[1]
    np.testing.assert_array_equal(W0, W1)
    assert not np.array_equal(q0, q1)
    w = race_inputs.WORKLOADS["c5_sweep"].with_n(96)
    assert shapes0 == shapes1 == [(1, 1, 96, 64), (1, 1, 96), (1, 1, 96, 64), (1, 1, 96, 64), (1, 1, 96, 64)]
    assert not np.any(h0)  # nothing precedes the first slice
    s0 = bench.shard_inputs(w, 0, "cpu")
    want = oracle.state(s0["k"].double().numpy(), s0["v"].double().numpy(), s0["W"].double().numpy(), w.tau)
    np.testing.assert_allclose(h1, want.reshape(h1.shape), rtol=1e-5, atol=1e-4)
    assert ms0 == ms1 == 6.0 and np.isclose(tps0, 2 * 96 / 0.006) and tps0 == tps1
