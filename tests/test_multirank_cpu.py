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
