"""RACE Attention for NVIDIA B200: Python binding of the C ABI in ``include/race_attn.h``.

Argument marshalling only: each function below passes torch tensors' device pointers, the
sizes read from their shapes and the current CUDA stream to the entry point of the same
name in ``librace_attn.so``.  Every step of the computation runs in that library's
kernels.  There is no CPU fallback: if the library is missing, importing the functions
works but the first call raises.

Method: "RACE Attention: A Strictly Linear-Time Attention for Long-Sequence Training"
(zh §2.2 Algorithm 1, zh §2.3 Algorithm 2).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "RACE_OK", "RACE_ERR_INVALID_ARG", "RACE_ERR_UNSUPPORTED", "RACE_ERR_WORKSPACE",
    "RACE_ERR_CUDA", "RACE_F32", "RACE_BF16", "RaceError", "library_path", "load_library",
    "race_status_string", "race_attn_workspace_size", "race_attn_ctx_size",
    "race_attn_forward", "race_attn_backward", "race_attn_hash_indices",
    "forward", "backward", "race_attn_profile_enable", "race_attn_profile_reset",
    "race_attn_profile_read", "race_attn_forward_noalloc", "RACE_NOALLOC_SCRATCH_BYTES",
    "race_attn_device_error", "race_attn_selftest_wait_timeout", "race_attn_state",
    "race_attn_decode_workspace_size", "race_attn_decode_step", "state", "decode_step",
    "race_attn_forward_begin", "race_attn_forward_end", "race_attn_backward_begin",
    "race_attn_backward_end", "race_attn_shard_combine", "race_attn_dw_workspace_size",
    "race_attn_backward_dw", "backward_dw",
]

HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_NAME = "librace_attn.so"

RACE_OK, RACE_ERR_INVALID_ARG, RACE_ERR_UNSUPPORTED, RACE_ERR_WORKSPACE, RACE_ERR_CUDA = range(5)
RACE_F32, RACE_BF16 = 0, 1
RACE_NOALLOC_SCRATCH_BYTES = 24 << 20

_vp = ctypes.c_void_p
_i64 = ctypes.c_int64
_int = ctypes.c_int
_sz = ctypes.c_size_t
_lib = None


class RaceError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s failed: %s" % (what, race_status_string(status)))


def library_path() -> str:
    return os.path.join(HERE, _LIB_NAME)


def load_library():
    """Load ``librace_attn.so`` (built in place by ``build.py``); raise if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError("%s is not built; run `python linear_attention_soft_b200/build.py`"
                           % path)
    lib = ctypes.CDLL(path)
    lib.race_status_string.argtypes = [_int]
    lib.race_status_string.restype = ctypes.c_char_p
    lib.race_attn_workspace_size.argtypes = [_int, _int, _i64, _int, _int, _int, _int, _int, _int,
                                             ctypes.POINTER(_sz)]
    lib.race_attn_workspace_size.restype = _int
    lib.race_attn_ctx_size.argtypes = [_int, _int, _i64, _int, _int, _int, _int,
                                       ctypes.POINTER(_sz)]
    lib.race_attn_ctx_size.restype = _int
    lib.race_attn_forward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _int, _int, _i64,
                                      _int, _int, _int, ctypes.c_float, _int, _int, _vp, _sz, _vp]
    lib.race_attn_forward.restype = _int
    lib.race_attn_backward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp,
                                       _int, _int, _i64, _int, _int, _int, ctypes.c_float, _int,
                                       _int, _vp, _sz, _vp]
    lib.race_attn_backward.restype = _int
    lib.race_attn_hash_indices.argtypes = [_vp, _vp, _vp, _int, _int, _i64, _int, _int, _int, _int,
                                           _vp]
    lib.race_attn_hash_indices.restype = _int
    lib.race_attn_device_error.argtypes = [ctypes.POINTER(_int), _vp]
    lib.race_attn_device_error.restype = _int
    lib.race_attn_selftest_wait_timeout.argtypes = [_i64, _vp]
    lib.race_attn_selftest_wait_timeout.restype = _int
    lib.race_attn_forward_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _i64, _int,
                                              _int, _int, ctypes.c_float, _int, _int, _vp]
    lib.race_attn_forward_noalloc.restype = _int
    lib.race_attn_state.argtypes = [_vp, _vp, _vp, _vp, _int, _int, _i64, _int, _int, _int,
                                    ctypes.c_float, _int, _vp, _sz, _vp]
    lib.race_attn_state.restype = _int
    lib.race_attn_decode_workspace_size.argtypes = [_int, _int, _int, _int, _int, ctypes.POINTER(_sz)]
    lib.race_attn_decode_workspace_size.restype = _int
    lib.race_attn_decode_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int,
                                          _int, ctypes.c_float, _int, _vp, _sz, _vp]
    lib.race_attn_decode_step.restype = _int
    lib.race_attn_forward_begin.argtypes = [_vp, _vp, _vp, _vp, _sz, _vp, _int, _int, _i64, _int, _int, _int,
                                            ctypes.c_float, _int, _int, _vp, _sz, _vp]
    lib.race_attn_forward_begin.restype = _int
    lib.race_attn_forward_end.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _int, _int, _i64, _int,
                                          _int, _int, ctypes.c_float, _int, _int, _vp, _sz, _vp]
    lib.race_attn_forward_end.restype = _int
    lib.race_attn_backward_begin.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp, _int,
                                             _int, _i64, _int, _int, _int, ctypes.c_float, _int, _int, _vp,
                                             _sz, _vp]
    lib.race_attn_backward_begin.restype = _int
    lib.race_attn_backward_end.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _int, _int, _i64,
                                           _int, _int, _int, ctypes.c_float, _int, _int, _vp, _sz, _vp]
    lib.race_attn_backward_end.restype = _int
    lib.race_attn_dw_workspace_size.argtypes = [_int, _int, _i64, _int, _int, _int, _int, _int, ctypes.POINTER(_sz)]
    lib.race_attn_dw_workspace_size.restype = _int
    lib.race_attn_backward_dw.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp, _vp, _vp, _int, _int,
                                          _i64, _int, _int, _int, ctypes.c_float, _int, _int, _vp, _sz, _vp]
    lib.race_attn_backward_dw.restype = _int
    lib.race_attn_shard_combine.argtypes = [_vp, _int, _int, _int, _i64, _vp, _vp]
    lib.race_attn_shard_combine.restype = _int
    lib.race_attn_profile_enable.argtypes = [_int]
    lib.race_attn_profile_enable.restype = None
    lib.race_attn_profile_reset.argtypes = []
    lib.race_attn_profile_reset.restype = None
    lib.race_attn_profile_read.argtypes = [ctypes.c_char_p, ctypes.POINTER(ctypes.c_float),
                                           ctypes.POINTER(_i64), _int]
    lib.race_attn_profile_read.restype = _int
    _lib = lib
    return lib


def race_status_string(status: int) -> str:
    return load_library().race_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != RACE_OK:
        raise RaceError(status, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return RACE_F32
    if t.dtype == torch.bfloat16:
        return RACE_BF16
    raise TypeError("RACE attention takes float32 or bfloat16 tensors, got %s" % t.dtype)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _nbytes(t: Optional[torch.Tensor]) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dims(q: torch.Tensor, W: torch.Tensor) -> Tuple[int, int, int, int, int, int]:
    B, H, N, d = q.shape
    L, P, dw = W.shape
    if dw != d:
        raise ValueError("W is [L, P, d] with the d of q")
    return B, H, N, d, L, P


def race_attn_workspace_size(B, H, N, d, L, P, causal, backward, dtype) -> int:
    out = _sz()
    _check(load_library().race_attn_workspace_size(B, H, N, d, L, P, int(causal), int(backward),
                                                   int(dtype), ctypes.byref(out)),
           "race_attn_workspace_size")
    return out.value


def race_attn_ctx_size(B, H, N, d, L, P, causal) -> int:
    out = _sz()
    _check(load_library().race_attn_ctx_size(B, H, N, d, L, P, int(causal), ctypes.byref(out)),
           "race_attn_ctx_size")
    return out.value


def race_attn_forward(q, k, v, W, out, den, ctx, tau: float, causal: bool, workspace,
                      stream=None) -> None:
    """C ABI forward on torch tensors ([B,H,N,d] q/k/v/out, [B,H,N] fp32 den, [L,P,d] W)."""
    B, H, N, d, L, P = _dims(q, W)
    _check(load_library().race_attn_forward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(out), _ptr(den), _ptr(ctx), _nbytes(ctx),
        B, H, N, d, L, P, float(tau), int(bool(causal)), _dtype_code(q), _ptr(workspace),
        _nbytes(workspace), _stream(stream)), "race_attn_forward")


def race_attn_backward(q, k, v, W, out, den, dout, ctx, dq, dk, dv, tau: float, causal: bool,
                       workspace, stream=None) -> None:
    """C ABI backward on torch tensors; dq/dk/dv are overwritten."""
    B, H, N, d, L, P = _dims(q, W)
    _check(load_library().race_attn_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(out), _ptr(den), _ptr(dout), _ptr(ctx),
        _nbytes(ctx), _ptr(dq), _ptr(dk), _ptr(dv), B, H, N, d, L, P, float(tau),
        int(bool(causal)), _dtype_code(q), _ptr(workspace), _nbytes(workspace), _stream(stream)),
        "race_attn_backward")


def race_attn_hash_indices(x, W, idx, stream=None) -> None:
    """C ABI hard sign-hash indices: idx is [B,H,N,L] int32."""
    B, H, N, d, L, P = _dims(x, W)
    _check(load_library().race_attn_hash_indices(
        _ptr(x), _ptr(W), _ptr(idx), B, H, N, d, L, P, _dtype_code(x), _stream(stream)),
        "race_attn_hash_indices")


def race_attn_forward_noalloc(q, k, v, W, out, den, tau: float, causal: bool, stream=None) -> None:
    """C ABI forward that takes no workspace: the library's fixed device buffer is used, so
    nothing is allocated (for callers that cannot allocate device memory)."""
    B, H, N, d, L, P = _dims(q, W)
    _check(load_library().race_attn_forward_noalloc(
        _ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(out), _ptr(den), B, H, N, d, L, P, float(tau),
        int(bool(causal)), _dtype_code(q), _stream(stream)), "race_attn_forward_noalloc")


def race_attn_state(k, v, W, state, tau: float, workspace, stream=None) -> None:
    """C ABI bucket statistics of every key: state is [B*H, L*2^P, d+1] fp32, written."""
    B, H, N, d, L, P = _dims(k, W)
    _check(load_library().race_attn_state(
        _ptr(k), _ptr(v), _ptr(W), _ptr(state), B, H, N, d, L, P, float(tau), _dtype_code(k),
        _ptr(workspace), _nbytes(workspace), _stream(stream)), "race_attn_state")


def race_attn_decode_workspace_size(B, H, d, L, P) -> int:
    out = _sz()
    _check(load_library().race_attn_decode_workspace_size(B, H, d, L, P, ctypes.byref(out)),
           "race_attn_decode_workspace_size")
    return out.value


def race_attn_decode_step(q, k, v, W, state, out, den, tau: float, workspace, stream=None) -> None:
    """C ABI streaming step: q, k, v, out are [B,H,d]; den [B,H] fp32 or None; state is
    updated in place."""
    B, H, d = q.shape
    L, P, dw = W.shape
    if dw != d:
        raise ValueError("W is [L, P, d] with the d of q")
    _check(load_library().race_attn_decode_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(state), _ptr(out), _ptr(den), B, H, d, L, P,
        float(tau), _dtype_code(q), _ptr(workspace), _nbytes(workspace), _stream(stream)),
        "race_attn_decode_step")


def race_attn_forward_begin(k, v, W, ctx, h_total, tau: float, causal: bool, workspace, stream=None) -> None:
    """C ABI forward, first half: h_total [B*H, L*2^P, d+1] fp32 receives this shard's
    key-side total."""
    B, H, N, d, L, P = _dims(k, W)
    _check(load_library().race_attn_forward_begin(
        _ptr(k), _ptr(v), _ptr(W), _ptr(ctx), _nbytes(ctx), _ptr(h_total), B, H, N, d, L, P, float(tau),
        int(bool(causal)), _dtype_code(k), _ptr(workspace), _nbytes(workspace), _stream(stream)),
        "race_attn_forward_begin")


def race_attn_forward_end(q, k, v, W, h_init, out, den, ctx, tau: float, causal: bool, workspace,
                          stream=None) -> None:
    """C ABI forward, second half, from the other shards' key statistics h_init (or None)."""
    B, H, N, d, L, P = _dims(q, W)
    _check(load_library().race_attn_forward_end(
        _ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(h_init), _ptr(out), _ptr(den), _ptr(ctx), _nbytes(ctx),
        B, H, N, d, L, P, float(tau), int(bool(causal)), _dtype_code(q), _ptr(workspace), _nbytes(workspace),
        _stream(stream)), "race_attn_forward_end")


def race_attn_backward_begin(q, k, v, W, out, den, dout, ctx, h_init, dq, g_total, tau: float, causal: bool,
                             workspace, stream=None) -> None:
    """C ABI backward, first half: dq and this shard's query-side total g_total."""
    B, H, N, d, L, P = _dims(q, W)
    _check(load_library().race_attn_backward_begin(
        _ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(out), _ptr(den), _ptr(dout), _ptr(ctx), _nbytes(ctx),
        _ptr(h_init), _ptr(dq), _ptr(g_total), B, H, N, d, L, P, float(tau), int(bool(causal)),
        _dtype_code(q), _ptr(workspace), _nbytes(workspace), _stream(stream)), "race_attn_backward_begin")


def race_attn_backward_end(q, k, v, W, out, den, dout, g_init, dk, dv, tau: float, causal: bool, workspace,
                           stream=None) -> None:
    """C ABI backward, second half: dk, dv from the other shards' query statistics g_init."""
    B, H, N, d, L, P = _dims(q, W)
    _check(load_library().race_attn_backward_end(
        _ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(out), _ptr(den), _ptr(dout), _ptr(g_init), _ptr(dk),
        _ptr(dv), B, H, N, d, L, P, float(tau), int(bool(causal)), _dtype_code(q), _ptr(workspace),
        _nbytes(workspace), _stream(stream)), "race_attn_backward_end")


def race_attn_shard_combine(gathered, shard: int, which: int, out, stream=None) -> None:
    """C ABI: out = sum of the selected shards of gathered [nshards, ...] in shard order
    (which: 0 before `shard`, 1 after it, 2 every other)."""
    n = gathered.shape[0]
    elems = gathered.numel() // max(n, 1)
    if out.numel() != elems:
        raise ValueError("out holds one shard's elements")
    _check(load_library().race_attn_shard_combine(_ptr(gathered), n, int(shard), int(which), elems, _ptr(out),
                                                  _stream(stream)), "race_attn_shard_combine")


def race_attn_dw_workspace_size(B, H, N, d, L, P, causal, dtype) -> int:
    out = _sz()
    _check(load_library().race_attn_dw_workspace_size(B, H, N, d, L, P, int(causal), int(dtype), ctypes.byref(out)),
           "race_attn_dw_workspace_size")
    return out.value


def race_attn_backward_dw(q, k, v, W, out, den, dout, ctx, dq, dk, dv, dW, tau: float, causal: bool, workspace,
                          stream=None) -> None:
    """C ABI backward that also writes dW [L, P, d] fp32 (gradient of the hyperplanes)."""
    B, H, N, d, L, P = _dims(q, W)
    _check(load_library().race_attn_backward_dw(
        _ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(out), _ptr(den), _ptr(dout), _ptr(ctx), _nbytes(ctx),
        _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dW), B, H, N, d, L, P, float(tau), int(bool(causal)), _dtype_code(q),
        _ptr(workspace), _nbytes(workspace), _stream(stream)), "race_attn_backward_dw")


def race_attn_device_error(stream=None) -> int:
    """1 if a tensor-core kernel gave up waiting on an MMA since the last call (and clear)."""
    flag = _int()
    _check(load_library().race_attn_device_error(ctypes.byref(flag), _stream(stream)),
           "race_attn_device_error")
    return flag.value


def race_attn_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    _check(load_library().race_attn_selftest_wait_timeout(int(limit_ns), _stream(stream)),
           "race_attn_selftest_wait_timeout")


def race_attn_profile_enable(on: bool) -> None:
    load_library().race_attn_profile_enable(int(bool(on)))


def race_attn_profile_reset() -> None:
    load_library().race_attn_profile_reset()


def race_attn_profile_read(max_kernels: int = 32):
    """{kernel name: (total ms, launches)} accumulated since the last reset."""
    names = ctypes.create_string_buffer(64 * max_kernels)
    ms = (ctypes.c_float * max_kernels)()
    cnt = (_i64 * max_kernels)()
    n = load_library().race_attn_profile_read(names, ms, cnt, max_kernels)
    if n < 0:
        raise RuntimeError("race_attn_profile_read: a recorded event reported an error")
    out = {}
    for i in range(min(n, max_kernels)):
        nm = names.raw[64 * i: 64 * i + 64].split(b"\0", 1)[0].decode()
        out[nm] = (float(ms[i]), int(cnt[i]))
    return out


# ---- conveniences that allocate with torch (device memory is plumbing) ---------------

def _workspace(q, W, causal, backward) -> torch.Tensor:
    B, H, N, d, L, P = _dims(q, W)
    n = race_attn_workspace_size(B, H, N, d, L, P, causal, backward, _dtype_code(q))
    return torch.empty(max(n, 16), dtype=torch.uint8, device=q.device)


def forward(q, k, v, W, tau: float, causal: bool, save_ctx: bool = False, stream=None):
    """Allocate and run the forward: returns (out, den, ctx or None)."""
    B, H, N, d, L, P = _dims(q, W)
    out = torch.empty_like(q)
    den = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    ctx = None
    if save_ctx:
        ctx = torch.empty(race_attn_ctx_size(B, H, N, d, L, P, causal) // 4, dtype=torch.float32,
                          device=q.device)
    race_attn_forward(q, k, v, W, out, den, ctx, tau, causal, _workspace(q, W, causal, False),
                      stream)
    return out, den, ctx


def backward(q, k, v, W, out, den, dout, tau: float, causal: bool, ctx=None, stream=None):
    """Allocate and run the backward: returns (dq, dk, dv)."""
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    race_attn_backward(q, k, v, W, out, den, dout, ctx, dq, dk, dv, tau, causal,
                       _workspace(q, W, causal, True), stream)
    return dq, dk, dv


def state(k, v, W, tau: float, stream=None) -> torch.Tensor:
    """Allocate and compute the bucket statistics of every key: [B*H, L*2^P, d+1] fp32."""
    B, H, N, d, L, P = _dims(k, W)
    st = torch.empty((B * H, L << P, d + 1), dtype=torch.float32, device=k.device)
    race_attn_state(k, v, W, st, tau, _workspace(k, W, False, False), stream)
    return st


def decode_step(q, k, v, W, state, tau: float, stream=None):
    """Allocate and run one streaming step ([B,H,d] q/k/v): returns (out, den); `state` is
    updated in place."""
    B, H, d = q.shape
    L, P, _ = W.shape
    out = torch.empty_like(q)
    den = torch.empty((B, H), dtype=torch.float32, device=q.device)
    ws = torch.empty(max(race_attn_decode_workspace_size(B, H, d, L, P), 16), dtype=torch.uint8,
                     device=q.device)
    race_attn_decode_step(q, k, v, W, state, out, den, tau, ws, stream)
    return out, den


def backward_dw(q, k, v, W, out, den, dout, tau: float, causal: bool, ctx=None, stream=None):
    """Allocate and run the backward with the hyperplane gradient: (dq, dk, dv, dW)."""
    B, H, N, d, L, P = _dims(q, W)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dW = torch.empty(W.shape, dtype=torch.float32, device=q.device)
    ws = torch.empty(max(race_attn_dw_workspace_size(B, H, N, d, L, P, causal, _dtype_code(q)), 16),
                     dtype=torch.uint8, device=q.device)
    race_attn_backward_dw(q, k, v, W, out, den, dout, ctx, dq, dk, dv, dW, tau, causal, ws, stream)
    return dq, dk, dv, dW
