"""Shared helpers of the GPU parity tests: run the CUDA library through its C ABI and the
fp64 oracle on the very same seeded inputs, and measure the difference."""
from __future__ import annotations

import numpy as np
import torch

import linear_attention_soft_b200 as ra
import oracle

# parity tolerances: normwise max relative error (fp32 inputs: fp32 arithmetic; bf16 inputs:
# bf16 operands with fp32 accumulation)
TOL = {torch.float32: 1e-4, torch.bfloat16: 2e-2}


def to64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def rel_err(gpu, ref, floor: float = 0.0) -> float:
    """max |gpu - ref| / max(max |ref|, floor) over the whole tensor.  ``floor`` only
    matters where the exact result is zero (e.g. dq, dk of a one-token causal sequence)."""
    g = to64(gpu) if isinstance(gpu, torch.Tensor) else np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    if g.size == 0:
        return 0.0
    scale = max(float(np.abs(r).max()), floor)
    return float(np.abs(g - r).max() / (scale if scale > 0 else 1.0))


def gpu_forward(inp, tau, causal, save_ctx=False):
    return ra.forward(inp["q"], inp["k"], inp["v"], inp["W"], tau, causal, save_ctx=save_ctx)


def gpu_backward(inp, out, den, tau, causal, ctx=None):
    return ra.backward(inp["q"], inp["k"], inp["v"], inp["W"], out, den, inp["do"], tau, causal,
                       ctx=ctx)


def oracle_forward(inp, tau, causal, rows=None, heads=None):
    q, k, v = (to64(inp[n]) for n in ("q", "k", "v"))
    if heads is not None:
        q, k, v = (x.reshape(-1, *x.shape[2:])[heads] for x in (q, k, v))
    return oracle.forward(q, k, v, to64(inp["W"]), tau, causal, rows=rows)


def oracle_backward(inp, tau, causal, n=None, heads=None):
    q, k, v, do = (to64(inp[x]) for x in ("q", "k", "v", "do"))
    if heads is not None:
        q, k, v, do = (x.reshape(-1, *x.shape[2:])[heads] for x in (q, k, v, do))
    if n is not None:
        q, k, v, do = (x[..., :n, :] for x in (q, k, v, do))
    return oracle.backward(q, k, v, to64(inp["W"]), do, tau, causal)


def projection_margin(x: np.ndarray, W: np.ndarray) -> np.ndarray:
    """min over tables and planes of |W_lp . x^| / |W_lp| per row (sign-hash robustness)."""
    xh = x / np.maximum(np.linalg.norm(x, axis=-1, keepdims=True), 1e-12)
    proj = np.einsum("lpd,...d->...lp", W, xh) / np.linalg.norm(W, axis=-1)
    return np.abs(proj).min(axis=(-1, -2))
