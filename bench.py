#!/usr/bin/env python
"""Benchmark: causal RACE attention forward + backward on one B200 per rank.

Default workload: B1 H1 N=4,194,304 d64 bf16, L16 P4 tau 0.5, clustered Q/K (the
sequence-length headline).  One step = race_attn_forward + race_attn_backward through the
C ABI on device-resident inputs (each input tensor is 512 MiB, larger than the 126 MB L2,
so no L2 flush is needed between steps).  Prints one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU, NCCL) the ranks run ONE sequence of N times the
workload's tokens, cut into contiguous slices in rank order, through the sequence-sharded
passes (one all-gather of per-slice bucket statistics per pass): weak scaling, the tokens
per rank fixed.  ``--independent`` runs N independent sequences instead (no collective on
the data path).  The timed region is bracketed by barriers and the time is the max over
ranks.  ``--impl reference`` times the fp64 CPU oracle instead, on a bounded prefix of the
same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import race_inputs  # noqa: E402

METRIC = "causal RACE attn fwd+bwd tokens/s at N=4M,d=64 (1 B200); % of roofline"
METRIC_FWD = "RACE attn forward tokens/s (1 B200); % of roofline"  # forward-only workloads


def metric_of(w):
    return METRIC if w.backward else METRIC_FWD


def pass_name(w):
    return "%s %s" % ("causal" if w.causal else "bidirectional", "fwd+bwd" if w.backward else "forward")
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
FP32_LANES_PER_SM = 128  # FMA units per SM (4 partitions x 32)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


# ---- algorithmic work (per token per head; s = element size; M = L*2^P) ---------------
def step_work(w: race_inputs.Workload):
    s = 4 if w.dtype == "f32" else 2
    M, d, LP = w.L * w.R, w.d, w.L * w.P
    if not w.backward:  # q, k, v in; out and den out; projections, aggregate, read-out
        return 4 * d * s + 4, 4 * M * (d + 1) + 4 * LP * d
    byts = 12 * d * s + 8
    flops = 12 * M * (d + 1) + 12 * LP * d
    return byts, flops


def kernel_work(name: str, w: race_inputs.Workload):
    """(algorithmic bytes, algorithmic flops) per token per head of one kernel over a step
    (all its launches: one per step for the d = 64 kernels; for the feature-group kernels of
    d = 128 one per head and pass, whose shares add up to these figures)."""
    s = 4 if w.dtype == "f32" else 2
    M, d, LP, D = w.L * w.R, w.d, w.L * w.P, w.d + 1
    pb = 4 * LP  # one side's projections p^ (fp32), the feature-group path's intermediate
    wide = {
        "wide_proj": (2 * d * s + 2 * pb, 4 * LP * d),                    # q, k in; p^ out
        "wide_agg_kv": (pb + d * s, 2 * M * D),                          # p^_k, v in
        "wide_fwd_walk": (2 * pb + 2 * d * s + 4, 4 * M * D),            # p^, v in; out, den out
        "wide_rowc": (2 * d * s + 4, 2 * d),                             # o, dO in; c out
        "wide_agg_qdy": (pb + d * s + 8, 2 * M * D),                     # p^_q, dO, den, c in
        "wide_bwd_q_walk": (3 * pb + 2 * d * s + 8, 4 * M * D),          # p^, v, dO, den, c in; dp^ out
        "wide_bwd_kv_walk": (3 * pb + 3 * d * s + 8, 6 * M * D),         # and dv out
        "wide_dx": (2 * pb + 4 * d * s, 4 * LP * d),                     # dp^, x in; dx out (both sides)
    }
    if name in wide:
        return wide[name]
    if w.causal:
        q_walk = (6 * d * s + 8, 4 * M * D + 6 * LP * d)    # q, k, v, o, dO, den in; dq, c_i out
        kv_walk = (6 * d * s + 8, 6 * M * D + 6 * LP * d)   # q, k, v, dO, den, c_i in; dk, dv out
    else:  # against the total statistics: no key (query) rows on the query (key) side
        q_walk = (4 * d * s + 8, 2 * M * D + 4 * LP * d)    # q, o, dO, den in; dq, c_i out
        kv_walk = (4 * d * s, 4 * M * D + 4 * LP * d)       # k, v in; dk, dv out
    table = {
        "agg_kv": (2 * d * s, 2 * M * D + 2 * LP * d),
        # causal walk: q, k, v in, out and den out; the general path's bidirectional pass of
        # the same name is a read-out (q in, out and den out)
        "fwd_walk": (4 * d * s + 4, 4 * M * D + 4 * LP * d) if w.causal else (2 * d * s + 4, 2 * M * D + 2 * LP * d),
        # bidirectional read-out: q in, out and den out
        "readout": (2 * d * s + 4, 2 * M * D + 2 * LP * d),
        "bwd_q_walk": q_walk,
        # q, dO, den, c_i in
        "agg_qdy": (2 * d * s + 8, 2 * M * D + 2 * LP * d),
        "bwd_kv_walk": kv_walk,
        "bwd_walk": (10 * d * s + 4, 10 * M * D + 12 * LP * d),
    }
    for key, val in table.items():
        if name.endswith(key):
            return val
    return None


# DRAM bytes per token (dram__bytes_read.sum + dram__bytes_write.sum) per kernel, from one
# ncu capture of the causal forward + backward at B1 H1 N = 2^20 d64 (traffic grows in
# proportion to the tokens), valid only for the kernel code and the segment planner it was
# taken on: the sha1 of the d = 64 kernel sources and of the planner, comments and
# whitespace removed.
NCU_TRAFFIC = {
    "code_sha1": {"race_tc.cuh": "9f7bf0221539d6a3842be7ef8a0990eddbcd37bf",
                  "race_tc_util.cuh": "574225aad3a9d82eef836e6f2c9f235ec0df8d12",
                  "race_attn.cu:make_plan": "368b30caf4555ce78bb0b9b31efea22157570d7e"},
    "bytes_per_token": {"tc_agg_kv": 259.9, "tc_fwd_walk": 502.3, "tc_bwd_q_walk": 769.9,
                        "tc_agg_qdy": 264.3, "tc_bwd_kv_walk": 756.6},
}


def code_sha1(path: str, function: str = "") -> str:
    """sha1 of a C++ source (or of one function in it: from its signature to the first line
    that closes it) without comments and whitespace: what the compiler sees."""
    import hashlib
    import re
    src = open(path, encoding="utf-8").read()
    if function:
        i = src.index(function)
        src = src[i:src.index("\n}\n", i) + 3]
    src = re.sub(r"//[^\n]*", "", src)
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return hashlib.sha1(re.sub(r"\s+", "", src).encode()).hexdigest()


def measured_traffic(name: str, tokens: int, causal: bool = True):
    """DRAM bytes per launch of kernel `name` from the recorded ncu capture (a causal pass),
    or None for a bidirectional pass or when the kernel code changed since (the counters
    would describe another kernel)."""
    if not causal:
        return None
    csrc = os.path.join(ROOT, "linear_attention_soft_b200", "csrc")
    for key, sha in NCU_TRAFFIC["code_sha1"].items():
        fn, _, function = key.partition(":")
        path = os.path.join(csrc, fn)
        if not os.path.exists(path) or code_sha1(path, ("Plan " + function + "(") if function else "") != sha:
            return None
    bpt = NCU_TRAFFIC["bytes_per_token"].get(name)
    return None if bpt is None else bpt * tokens


def is_tensor_core_kernel(name: str) -> bool:
    return name.startswith("tc_") or (name.startswith("wide_") and name != "wide_rowc")


# ---- clocks ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---- CPU baseline (the fp64 oracle) -----------------------------------------------------
def oracle_step(inp_cpu, w, n):
    import numpy as np
    import oracle
    q, k, v = (inp_cpu[x][0, 0, :n].to(torch.float64).numpy() for x in ("q", "k", "v"))
    do = inp_cpu["do"][0, 0, :n].to(torch.float64).numpy() if w.backward else None
    W = inp_cpu["W"].to(torch.float64).numpy()
    t0 = time.perf_counter()
    oracle.forward(q, k, v, W, w.tau, w.causal)
    if w.backward:
        oracle.backward(q, k, v, W, do, w.tau, w.causal)
    return time.perf_counter() - t0


def oracle_sample_size(inp_cpu, w, target_s):
    n = 2048
    t = oracle_step(inp_cpu, w, n)
    n2 = int(n * target_s / max(t, 1e-3))
    n2 = max(1024, min(n2, w.N, 1 << 20))
    return n2


def cpu_baseline(w, target_s=12.0):
    import oracle
    small = race_inputs.make_inputs(w.with_n(min(w.N, 1 << 20)), "cpu")
    n = oracle_sample_size(small, w, target_s)
    t = oracle_step(small, w, n)
    return {"value": n / t, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": "%s of the first %d tokens of head 0 (inputs drawn with the "
                      "workload's recipe), fp64, wall clock %.1f s" % (pass_name(w), n, t)}


def run_reference(args, w):
    """Time the fp64 oracle, as it stands, on a bounded prefix of the workload."""
    import oracle
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    budget = 150.0 / max(1, args.steps + args.warmup)
    small = race_inputs.make_inputs(w.with_n(min(w.N, 1 << 20)), "cpu")
    n = oracle_sample_size(small, w, min(10.0, budget))
    for _ in range(args.warmup):
        oracle_step(small, w, min(n, 2048))
    times = [oracle_step(small, w, n) for _ in range(args.steps)]
    t = statistics.mean(times)
    val = n / t
    line = {"impl": "reference", "metric": metric_of(w), "value": val, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": t * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "L": w.L,
                       "P": w.P, "tau": w.tau, "causal": w.causal,
                       "sample_tokens_per_step": n},
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": oracle.num_threads(),
                             "kind": "oracle",
                             "sample": "%s of the first %d tokens of head 0 per step"
                                       % (pass_name(w), n)},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---- multi-rank bookkeeping ----------------------------------------------------------------
def rank_workload(w: race_inputs.Workload, rank: int) -> race_inputs.Workload:
    """The workload rank `rank` runs with --independent: same shape, its own seed."""
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + 1000 * rank)


def shard_inputs(w: race_inputs.Workload, rank: int, device):
    """Rank `rank`'s slice (tokens [rank N, (rank + 1) N) of every head) of one sequence of
    world * N tokens: the hyperplanes W are the same on every rank, the rows are the slice's
    own draw."""
    return race_inputs.make_inputs(w, device, slice_index=rank)


def sharded_step(inp, w: race_inputs.Workload, lib=None, events=None):
    """One forward + backward of this rank's slice through the sequence-sharded passes (one
    all-gather per pass).  `lib` replaces the CUDA library (a CPU stand-in in the tests);
    `events` collects CUDA event pairs around each exchange."""
    from linear_attention_soft_b200 import sharded
    out, den, ctx = sharded.forward(inp["q"], inp["k"], inp["v"], inp["W"], w.tau, w.causal, lib=lib,
                                    events=events)
    if not w.backward:
        return out, den, None, None, None
    dq, dk, dv = sharded.backward(inp["q"], inp["k"], inp["v"], inp["W"], out, den, inp["do"], w.tau,
                                  w.causal, ctx, lib=lib, events=events)
    return out, den, dq, dk, dv


def job_throughput(ms_local: float, tokens_local: int, world: int, device=None):
    """(max ms over ranks, whole-job tokens/s): every rank's tokens over the slowest rank's
    time.  Collective only when world > 1."""
    t = torch.tensor([ms_local, float(tokens_local)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    if world > 1:
        import torch.distributed as dist
        mx = t.clone()
        dist.all_reduce(mx, op=dist.ReduceOp.MAX)
        sm = t.clone()
        dist.all_reduce(sm, op=dist.ReduceOp.SUM)
        ms, tokens = float(mx[0]), float(sm[1])
    else:
        ms, tokens = float(t[0]), float(t[1])
    return ms, tokens / (ms / 1e3)


# ---- the CUDA library -------------------------------------------------------------------
def run_ours(args, w):
    import linear_attention_soft_b200 as ra
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    peaks = load_peaks()
    sharded_mode = world > 1 and not args.independent
    if sharded_mode and args.dw:
        raise SystemExit("--dw is not offered by the sequence-sharded passes; use --independent")
    # one sequence sliced over the ranks, or (--independent) one sequence per rank
    inp = shard_inputs(w, rank, dev) if sharded_mode else race_inputs.make_inputs(rank_workload(w, rank), dev)
    q, k, v, W, do = inp["q"], inp["k"], inp["v"], inp["W"], inp.get("do")
    B, H, N, d = q.shape
    L, P = w.L, w.P
    out = torch.empty_like(q)
    den = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    code = ra.RACE_F32 if w.dtype == "f32" else ra.RACE_BF16
    # one scratch buffer serves the forward and the backward, which run in turn on one stream
    ws_f = ws_b = torch.empty(max(ra.race_attn_workspace_size(B, H, N, d, L, P, w.causal, 0, code),
                                  ra.race_attn_dw_workspace_size(B, H, N, d, L, P, w.causal, code) if args.dw
                                  else ra.race_attn_workspace_size(B, H, N, d, L, P, w.causal, 1, code)),
                              dtype=torch.uint8, device=dev)
    dW = torch.empty(W.shape, dtype=torch.float32, device=dev)
    ctx = torch.empty(ra.race_attn_ctx_size(B, H, N, d, L, P, w.causal) // 4,
                      dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(qq=q, kk=k, vv=v, dd=do, res=None, events=None):
        """One forward + backward (a forward alone for forward-only workloads); returns the
        five result tensors."""
        if sharded_mode:
            return sharded_step({"q": qq, "k": kk, "v": vv, "do": dd, "W": W}, w, events=events)
        o_, den_, dq_, dk_, dv_ = res if res is not None else (out, den, dq, dk, dv)
        ra.race_attn_forward(qq, kk, vv, W, o_, den_, ctx, w.tau, w.causal, ws_f, stream)
        if not w.backward:
            return o_, den_, dq_, dk_, dv_
        if args.dw:
            ra.race_attn_backward_dw(qq, kk, vv, W, o_, den_, dd, ctx, dq_, dk_, dv_, dW, w.tau, w.causal, ws_b,
                                     stream)
        else:
            ra.race_attn_backward(qq, kk, vv, W, o_, den_, dd, ctx, dq_, dk_, dv_, w.tau, w.causal,
                                  ws_b, stream)
        return o_, den_, dq_, dk_, dv_

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    ra.race_attn_profile_reset()
    ra.race_attn_profile_enable(True)
    torch.cuda.synchronize(dev)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    xevents = [] if sharded_mode else None
    e0.record(stream)
    for _ in range(args.steps):
        step(events=xevents)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    ra.race_attn_profile_enable(False)
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    prof = ra.race_attn_profile_read()
    ms_max, value = job_throughput(ms, B * N, world, dev)
    # the exchanges (all-gather + shard-order combine), timed on this rank, max over ranks
    x_ms_max = None
    if sharded_mode:
        x_ms = sum(a.elapsed_time(b) for a, b in xevents) / args.steps
        x_ms_max = job_throughput(x_ms, 0, world, dev)[0]

    # ---- end to end through the C ABI with host buffers --------------------------------
    e2e_val = h2d = d2h = None
    if not args.no_e2e:
        # Every step copies its inputs in from pinned host memory and its results out, on their
        # own streams: step i+1's inputs go in and step i-1's results go out while step i
        # computes (two device buffer sets, ordered by events).
        host = {n: t.cpu().pin_memory() for n, t in (("q", q), ("k", k), ("v", v), ("do", do))
                if t is not None}
        host_out = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                    for n, t in ((("out", out), ("dq", dq), ("dk", dk), ("dv", dv)) if w.backward
                                 else (("out", out),))}
        dev_in = [{n: torch.empty_like(host[n], device=dev) for n in host} for _ in range(2)]
        dev_res = [(out, den, dq, dk, dv),
                   (torch.empty_like(out), torch.empty_like(den), torch.empty_like(dq), torch.empty_like(dk),
                    torch.empty_like(dv))]
        h2d = sum(t.numel() * t.element_size() for t in host.values())
        d2h = sum(t.numel() * t.element_size() for t in host_out.values())
        e2e_steps = max(2, args.steps)  # the same K steps as the device-timed leg
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_run(n_steps):
            s_in.wait_stream(stream)  # nothing of the run starts before what the stream already holds
            for i in range(n_steps):
                b = i & 1
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev_done[b])  # step i-2 has finished reading these inputs
                    for n in host:
                        dev_in[b][n].copy_(host[n], non_blocking=True)
                    ev_in[b].record(s_in)
                stream.wait_event(ev_in[b])
                if i >= 2:
                    stream.wait_event(ev_out[b])    # step i-2's results are out
                res = step(dev_in[b]["q"], dev_in[b]["k"], dev_in[b]["v"], dev_in[b].get("do"), dev_res[b])
                ev_done[b].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[b])
                    if sharded_mode:  # the driver's own results, made on the compute stream
                        for t in res:
                            if t is not None:
                                t.record_stream(s_out)
                    for n, t in zip(("out", None, "dq", "dk", "dv"), res):
                        if n in host_out:
                            host_out[n].copy_(t, non_blocking=True)
                    ev_out[b].record(s_out)
            stream.wait_event(ev_out[(n_steps - 1) & 1])

        e2e_run(2)
        torch.cuda.synchronize(dev)
        barrier()
        e0.record(stream)
        e2e_run(e2e_steps)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        _, e2e_val = job_throughput(e0.elapsed_time(e1) / e2e_steps, B * N, world, dev)

    # ---- roofline of the dominant kernel and of the whole step ------------------------
    launches = sum(c for _, c in prof.values())
    top = max(prof.items(), key=lambda kv: kv[1][0]) if prof else None
    roof = None
    if top:
        name, (tot_ms, cnt) = top
        per_launch_s = tot_ms / cnt / 1e3
        per_step_s = tot_ms / args.steps / 1e3  # all the kernel's launches in one step
        work = kernel_work(name, w)
        units = B * H * N
        share = tot_ms / sum(t for t, _ in prof.values())
        if work:
            byts, flops = work[0] * units, work[1] * units
            if is_tensor_core_kernel(name):
                peak_c = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
                t_c = flops / (peak_c * 1e12)
            else:
                peak_c = (torch.cuda.get_device_properties(dev).multi_processor_count
                          * FP32_LANES_PER_SM * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12)
                t_c = flops / (peak_c * 1e12)
            t_m = byts / (peaks["hbm_gbs"] * 1e9)
            if t_m >= t_c:
                roof = {"bound": "hbm", "achieved": byts / per_step_s / 1e9,
                        "peak": peaks["hbm_gbs"], "unit": "GB/s"}
            else:
                roof = {"bound": "tensor" if is_tensor_core_kernel(name) else "alu",
                        "achieved": flops / per_step_s / 1e12, "peak": peak_c, "unit": "TFLOP/s"}
            roof["frac"] = roof["achieved"] / roof["peak"]
            roof["traffic"] = measured_traffic(name, units, w.causal)
            roof.update({"kernel": name, "ms_per_launch": per_launch_s * 1e3,
                         "launches_per_step": cnt / args.steps,
                         "share_of_step": share, "peak_source": peaks["source"]})
    sb, sf = step_work(w)
    t_step_roof = max(sb * B * H * N / (peaks["hbm_gbs"] * 1e9),
                      sf * B * H * N / (peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * 1e12))
    step_roof = {"bytes_per_token": sb, "flops_per_token": sf, "roofline_ms": t_step_roof * 1e3,
                 "frac": t_step_roof * 1e3 / ms_max}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w)

    if rank == 0:
        line = {"metric": metric_of(w), "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
                "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                           "L": w.L, "P": w.P, "tau": w.tau, "causal": w.causal,
                           "dist": w.dist, "l2": "inputs larger than L2 (no flush)", "dW": bool(args.dw),
                           "head_tokens_per_s": B * H * N * world / (ms_max / 1e3),
                           "parallelism": ("sequence sharded over %d ranks (%d tokens each, one all-gather "
                                           "per pass)" % (world, N)) if sharded_mode else
                                          ("%d independent sequences" % world if world > 1 else "one GPU"),
                           "exchange_ms_per_step": x_ms_max,
                           "exchange_share_of_step": x_ms_max / ms_max if sharded_mode else None},
                "e2e": None if args.no_e2e else {"value": e2e_val, "unit": "tokens/s",
                                                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
                "gpu_launches": launches,
                "roofline": roof, "step_roofline": step_roof,
                "kernels": {n: {"ms_total": t, "launches": c} for n, (t, c) in prof.items()},
                "clocks": clk, "cpu_baseline": cpu}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


# ---- decode-time streaming step ---------------------------------------------------------
DECODE = {"B": 128, "H": 32, "d": 64, "L": 16, "P": 4, "tau": 0.5, "prompt": 256, "seed": 9}


def run_decode(args):
    """One step = race_attn_decode_step for every (b, h) (one new token per head).  The
    B*H = 4096 states (272 MB fp32) exceed L2, so every step streams them from HBM."""
    import linear_attention_soft_b200 as ra
    c = DECODE
    B, H, d, L, P, tau = c["B"], c["H"], c["d"], c["L"], c["P"], c["tau"]
    BH, M, D = B * H, L << P, d + 1
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    n_tok = args.warmup + args.steps
    inp = race_inputs.small_normal(B, H, c["prompt"] + n_tok, d, L, P, c["seed"], dtype=torch.bfloat16, device=dev)
    W = inp["W"]
    state = ra.state(inp["k"][:, :, :c["prompt"]].contiguous(), inp["v"][:, :, :c["prompt"]].contiguous(), W, tau)
    toks = {n: inp[n][:, :, c["prompt"]:].permute(2, 0, 1, 3).contiguous() for n in ("q", "k", "v")}
    out = torch.empty((B, H, d), dtype=torch.bfloat16, device=dev)
    den = torch.empty((B, H), dtype=torch.float32, device=dev)
    ws = torch.empty(ra.race_attn_decode_workspace_size(B, H, d, L, P), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i, q=None, k=None, v=None):
        ra.race_attn_decode_step(toks["q"][i] if q is None else q, toks["k"][i] if k is None else k,
                                 toks["v"][i] if v is None else v, W, state, out, den, tau, ws, stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    ra.race_attn_profile_reset()
    ra.race_attn_profile_enable(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.warmup, n_tok):
        step(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ra.race_attn_profile_enable(False)
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    prof = ra.race_attn_profile_read()
    # end to end: the step's tokens from pinned host memory in, out and den back
    hq, hk, hv = (toks[n][0].cpu().pin_memory() for n in ("q", "k", "v"))
    dq_, dk_, dv_ = (torch.empty_like(t, device=dev) for t in (hq, hk, hv))
    ho = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    hd = torch.empty(den.shape, dtype=den.dtype, pin_memory=True)
    e0.record(stream)
    for _ in range(args.steps):
        dq_.copy_(hq, non_blocking=True)
        dk_.copy_(hk, non_blocking=True)
        dv_.copy_(hv, non_blocking=True)
        step(0, dq_, dk_, dv_)
        ho.copy_(out, non_blocking=True)
        hd.copy_(den, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / args.steps
    upd_ms, upd_n = prof.get("decode_update", (0.0, 1))
    per_launch_s = upd_ms / upd_n / 1e3
    byts = BH * (2 * M * D * 4 + 3 * d * 2)      # the state read and written, the token read
    roof = {"bound": "hbm", "achieved": byts / per_launch_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "traffic": None, "kernel": "decode_update", "ms_per_launch": per_launch_s * 1e3,
            "peak_source": peaks["source"]}
    roof["frac"] = roof["achieved"] / roof["peak"]
    line = {"metric": "RACE decode step tokens/s (one token per head, B*H=4096 heads, L16 P4 d64)",
            "value": BH / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "decode_b128h32", "B": B, "H": H, "d": d, "L": L, "P": P, "tau": tau,
                       "prompt": c["prompt"], "l2": "states larger than L2 (no flush)"},
            "e2e": {"value": BH / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": 3 * BH * d * 2,
                    "d2h_bytes_per_step": BH * d * 2 + BH * 4},
            "gpu_launches": sum(n for _, n in prof.values()), "roofline": roof,
            "kernels": {n: {"ms_total": t, "launches": k} for n, (t, k) in prof.items()},
            "clocks": clk, "cpu_baseline": None}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="c3_causal_n4m_clusters",
                    choices=sorted(race_inputs.WORKLOADS))
    ap.add_argument("--n", type=int, default=0, help="override the sequence length")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end leg (it holds a second device copy of inputs and results)")
    ap.add_argument("--dw", action="store_true", help="also compute the gradient of the hyperplanes W")
    ap.add_argument("--independent", action="store_true",
                    help="with several ranks: one independent sequence per rank instead of one "
                         "sequence sharded over the ranks")
    ap.add_argument("--decode", action="store_true",
                    help="time the streaming decode step instead (one token per head, 4096 heads)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = race_inputs.WORKLOADS[args.workload]
    if args.n:
        w = w.with_n(args.n)
    if args.decode:
        run_decode(args)
    elif args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
