"""Seeded synthetic inputs for RACE attention runs.

This module only draws random numbers; it holds none of the method's arithmetic.  The
tests, the benchmark and the smoke check take their inputs from here and hand the very
same values to both the CUDA library and the fp64 oracle.

Recipe (torch generator seeded per workload, on the device the inputs are made on; draws
in the order W, Q, K, V, dO; bf16 workloads draw fp32 normals and round them to bf16
with round-to-nearest-even):

* W [L, P, d] fp32, i.i.d. N(0, 1): the Gaussian hyperplanes of every table.
* "normal":   Q, K, V, dO i.i.d. N(0, 1).
* "clusters": 256 centres mu_c ~ N(0, I_d) shared by Q and K; every Q row and every K row
  picks a centre uniformly and independently and adds 0.1 * N(0, I_d) noise, so bucket
  occupancy is far from uniform.  V, dO i.i.d. N(0, 1).
* ``unit_qk``: Q and K rows are scaled to unit L2 norm after drawing.

Large sequences are drawn in fixed blocks of rows so that the values do not depend on
available memory.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import torch

_BLOCK_ROWS = 1 << 22


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    L: int
    P: int
    tau: float
    causal: bool
    dtype: str          # "f32" or "bf16"
    seed: int
    dist: str = "normal"
    unit_qk: bool = False
    backward: bool = True

    @property
    def R(self) -> int:
        return 1 << self.P

    def with_n(self, N: int, name: Optional[str] = None) -> "Workload":
        return dataclasses.replace(self, N=N, name=name or f"{self.name}-N{N}")


# The workloads the benchmark and the parity tests use.
WORKLOADS: Dict[str, Workload] = {
    "c1_noncausal_fwd_f32": Workload("c1_noncausal_fwd_f32", 1, 1, 1024, 64, 8, 4, 1.0, False,
                                     "f32", 0, "normal", unit_qk=True, backward=False),
    "c2_causal_b2h8_n64k": Workload("c2_causal_b2h8_n64k", 2, 8, 65536, 64, 16, 4, 0.5, True,
                                    "bf16", 1),
    "c3_causal_n4m_clusters": Workload("c3_causal_n4m_clusters", 1, 1, 4_194_304, 64, 16, 4, 0.5,
                                       True, "bf16", 2, "clusters"),
    "c4_causal_h4_n12m_d128": Workload("c4_causal_h4_n12m_d128", 1, 4, 12_000_000, 128, 32, 5,
                                       0.5, True, "bf16", 3),
    "c5_sweep": Workload("c5_sweep", 1, 1, 1 << 20, 64, 16, 4, 0.5, True, "bf16", 4),
    # bidirectional (Algorithm 1) forward + backward at the c2 and c3 sizes
    "n1_noncausal_b2h8_n64k": Workload("n1_noncausal_b2h8_n64k", 2, 8, 65536, 64, 16, 4, 0.5, False,
                                       "bf16", 5),
    "n1_noncausal_n4m_clusters": Workload("n1_noncausal_n4m_clusters", 1, 1, 4_194_304, 64, 16, 4, 0.5,
                                          False, "bf16", 6, "clusters"),
}
SWEEP_N = (1 << 20, 1 << 22, 1 << 24, 75_000_000)


def torch_dtype(w: Workload) -> torch.dtype:
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def _normal_rows(gen, rows: int, d: int, device, dtype) -> torch.Tensor:
    out = torch.empty((rows, d), dtype=dtype, device=device)
    for r0 in range(0, rows, _BLOCK_ROWS):
        r1 = min(rows, r0 + _BLOCK_ROWS)
        out[r0:r1] = torch.randn((r1 - r0, d), generator=gen, device=device,
                                 dtype=torch.float32).to(dtype)
    return out


def _cluster_rows(gen, centres: torch.Tensor, rows: int, device, dtype) -> torch.Tensor:
    d = centres.shape[1]
    out = torch.empty((rows, d), dtype=dtype, device=device)
    for r0 in range(0, rows, _BLOCK_ROWS):
        r1 = min(rows, r0 + _BLOCK_ROWS)
        pick = torch.randint(0, centres.shape[0], (r1 - r0,), generator=gen, device=device)
        noise = torch.randn((r1 - r0, d), generator=gen, device=device, dtype=torch.float32)
        out[r0:r1] = (centres[pick] + 0.1 * noise).to(dtype)
    return out


def make_inputs(w: Workload, device="cpu", with_grad_out: Optional[bool] = None, slice_index: int = 0):
    """Draw W, q, k, v (and dO) for workload ``w`` on ``device``.

    Sequence tensors are [B, H, N, d] in the workload's dtype; W is [L, P, d] fp32.
    ``slice_index`` s > 0 draws slice s of a longer sequence cut into slices of N tokens:
    W (and the cluster centres) as for slice 0, the rows from a generator reseeded with
    seed + 1000 s.  Slice 0 is the workload itself.
    """
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(w.seed)
    dt = torch_dtype(w)
    rows = w.B * w.H * w.N
    W = torch.randn((w.L, w.P, w.d), generator=gen, device=device, dtype=torch.float32)
    centres = None
    if w.dist == "clusters":
        centres = torch.randn((256, w.d), generator=gen, device=device, dtype=torch.float32)
    if slice_index:
        gen.manual_seed(w.seed + 1000 * slice_index)
    if w.dist == "clusters":
        q = _cluster_rows(gen, centres, rows, device, dt)
        k = _cluster_rows(gen, centres, rows, device, dt)
    elif w.dist == "normal":
        q = _normal_rows(gen, rows, w.d, device, dt)
        k = _normal_rows(gen, rows, w.d, device, dt)
    else:
        raise ValueError(w.dist)
    v = _normal_rows(gen, rows, w.d, device, dt)
    if w.unit_qk:
        q = (q.float() / q.float().norm(dim=-1, keepdim=True)).to(dt)
        k = (k.float() / k.float().norm(dim=-1, keepdim=True)).to(dt)
    shape = (w.B, w.H, w.N, w.d)
    out = {"W": W, "q": q.view(shape), "k": k.view(shape), "v": v.view(shape)}
    if w.backward if with_grad_out is None else with_grad_out:
        out["do"] = _normal_rows(gen, rows, w.d, device, dt).view(shape)
    return out


def small_normal(B, H, N, d, L, P, seed, dtype=torch.float32, device="cpu", scale_qk=1.0):
    """Small i.i.d. N(0,1) case for unit tests: dict with W, q, k, v, do."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    W = torch.randn((L, P, d), generator=gen, device=device, dtype=torch.float32)
    shape = (B, H, N, d)
    t = [torch.randn(shape, generator=gen, device=device, dtype=torch.float32) for _ in range(4)]
    t[0] = t[0] * scale_qk
    t[1] = t[1] * scale_qk
    q, k, v, do = (x.to(dtype) for x in t)
    return {"W": W, "q": q, "k": k, "v": v, "do": do}
