"""One sequence sharded over the ranks of a torch.distributed group.

Every rank holds a contiguous slice of the tokens of every head; rank order is token order
(rank 0 holds the first slice).  The statistics of Algorithm 2 ("RACE Attention: A Strictly
Linear-Time Attention for Long-Sequence Training", zh §2.3) are sums over tokens, so each
pass needs from the other ranks only their totals:

* forward: each rank's key-side total H_s = sum over its keys of phi(k)[v, 1]^T is
  all-gathered; rank s starts its causal scan from sum_{s' < s} H_s' (bidirectional: from
  every other rank's total);
* backward: each rank's query-side total G_s = sum over its queries of phi(q) dY^T is
  all-gathered; rank s starts the key side's suffix from sum_{s' > s} G_s' (bidirectional:
  every other rank's).

One all-gather of B*H*L*2^P*(d+1) fp32 values per pass (66.5 KB per head at L16 P4 d64);
the sums over ranks run in rank order in the library's combine kernel, so every rank gets
bitwise the same result for the same inputs.  The collective is torch.distributed's (NCCL
over NVLink on GPUs); all arithmetic runs in the CUDA library.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import (_dims, _dtype_code, race_attn_backward_begin, race_attn_backward_end, race_attn_ctx_size,
               race_attn_forward_begin, race_attn_forward_end, race_attn_shard_combine,
               race_attn_workspace_size)

BEFORE, AFTER, OTHERS = 0, 1, 2


class Library:
    """The library calls the sharded passes make (a stand-in with the same methods can be
    passed instead, e.g. to test the exchange on CPU)."""

    def forward_begin(self, k, v, W, ctx, h_total, tau, causal, ws):
        race_attn_forward_begin(k, v, W, ctx, h_total, tau, causal, ws)

    def forward_end(self, q, k, v, W, h_init, out, den, ctx, tau, causal, ws):
        race_attn_forward_end(q, k, v, W, h_init, out, den, ctx, tau, causal, ws)

    def backward_begin(self, q, k, v, W, out, den, dout, ctx, dq, g_total, tau, causal, ws):
        race_attn_backward_begin(q, k, v, W, out, den, dout, ctx, None, dq, g_total, tau, causal, ws)

    def backward_end(self, q, k, v, W, out, den, dout, g_init, dk, dv, tau, causal, ws):
        race_attn_backward_end(q, k, v, W, out, den, dout, g_init, dk, dv, tau, causal, ws)

    def combine(self, gathered, shard, which, out):
        race_attn_shard_combine(gathered, shard, which, out)


def exchange(local: torch.Tensor, which: int, group=None, lib=None, events=None) -> torch.Tensor:
    """All-gather every rank's `local` statistics and return the sum of the ranks selected by
    `which` (BEFORE, AFTER or OTHERS this rank), in rank order.  With `events` (a list), a
    pair of CUDA events recorded on the current stream around the exchange is appended, so a
    caller can time it."""
    lib = lib or Library()
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if events is not None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
    gathered = torch.empty((world,) + tuple(local.shape), dtype=local.dtype, device=local.device)
    dist.all_gather(list(gathered.unbind(0)), local.contiguous(), group=group)
    out = torch.empty_like(local)
    lib.combine(gathered, rank, which, out)
    if events is not None:
        e1.record()
        events.append((e0, e1))
    return out


def _state_shape(q, W):
    B, H, N, d, L, P = _dims(q, W)
    return (B * H, L << P, d + 1)


def forward(q, k, v, W, tau: float, causal: bool, group=None, lib=None, events=None):
    """Forward of this rank's shard ([B, H, n, d]): returns (out, den, ctx); ctx is kept for
    the backward.  `events`: as for exchange."""
    lib = lib or Library()
    B, H, N, d, L, P = _dims(q, W)
    ctx = torch.empty(max(race_attn_ctx_size(B, H, N, d, L, P, causal) // 4, 4), dtype=torch.float32,
                      device=q.device)
    ws = torch.empty(max(race_attn_workspace_size(B, H, N, d, L, P, causal, False, _dtype_code(q)), 16),
                     dtype=torch.uint8, device=q.device)
    h_total = torch.empty(_state_shape(q, W), dtype=torch.float32, device=q.device)
    lib.forward_begin(k, v, W, ctx, h_total, tau, causal, ws)
    h_init = exchange(h_total, BEFORE if causal else OTHERS, group, lib, events)
    out = torch.empty_like(q)
    den = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    lib.forward_end(q, k, v, W, h_init, out, den, ctx, tau, causal, ws)
    return out, den, ctx


def backward(q, k, v, W, out, den, dout, tau: float, causal: bool, ctx, group=None, lib=None, events=None):
    """Backward of this rank's shard, with the ctx its forward returned: (dq, dk, dv).
    `events`: as for exchange."""
    lib = lib or Library()
    B, H, N, d, L, P = _dims(q, W)
    ws = torch.empty(max(race_attn_workspace_size(B, H, N, d, L, P, causal, True, _dtype_code(q)), 16),
                     dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q)
    g_total = torch.empty(_state_shape(q, W), dtype=torch.float32, device=q.device)
    lib.backward_begin(q, k, v, W, out, den, dout, ctx, dq, g_total, tau, causal, ws)
    g_init = exchange(g_total, AFTER if causal else OTHERS, group, lib, events)
    dk, dv = torch.empty_like(k), torch.empty_like(v)
    lib.backward_end(q, k, v, W, out, den, dout, g_init, dk, dv, tau, causal, ws)
    return dq, dk, dv
