"""fp64 CPU oracle for RACE Attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg import this package.
The CUDA library never loads it, and the two share no code.

``race_oracle.c`` holds the method written as plain loops in fp64 (the sources it follows
are cited in its header: the gist.science summaries of "RACE Attention: A Strictly
Linear-Time Attention for Long-Sequence Training", zh §2.2 Algorithm 1, zh §2.3 Algorithm 2).
``bruteforce.py`` holds two O(N^2) forms used to pin it: the same estimator written pairwise,
and the sharpened angular-kernel attention that RACE approximates.

Parity status of each function (what pins it is in ``tests/test_oracle.py``):

* ``features``            pinned: corners sum to one; equals the per-plane sigmoid product;
                          corner mean of c_p equals tanh(beta*u_p); beta -> inf gives the sign
                          hash; worked examples in ``tests/golden``.
* ``hash_indices``        pinned: hand-worked golden example; agrees with the soft argmax at
                          large beta.
* ``forward``             pinned: equals the pairwise O(N^2) estimator; converges to the
                          angular-kernel attention with gamma = P as L grows (hard hashing);
                          causality, convexity and invariances; golden worked examples.
* ``backward``            pinned: central finite differences of ``forward`` in fp64, plus
                          the identity sum_j dv_j = sum_i dO_i.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "race_oracle.c")
_LIB_PATH = os.path.join(_HERE, "librace_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_i32p = ctypes.POINTER(ctypes.c_int32)


def build(force: bool = False) -> str:
    """Compile ``race_oracle.c`` (gcc, -O2, OpenMP, IEEE semantics kept) next to itself."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB_PATH)
        lib.race_oracle_features.argtypes = [_dp, ctypes.c_int, _dp, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_double, ctypes.c_int, _dp]
        lib.race_oracle_features.restype = None
        lib.race_oracle_hash_indices.argtypes = [_dp, ctypes.c_int, _dp, ctypes.c_int,
                                                 ctypes.c_int, _i32p]
        lib.race_oracle_hash_indices.restype = None
        lib.race_oracle_features_backward.argtypes = [_dp, ctypes.c_int, _dp, ctypes.c_int,
                                                      ctypes.c_int, ctypes.c_double, _dp, _dp]
        lib.race_oracle_features_backward.restype = None
        lib.race_oracle_forward.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64,
                                            ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_double, ctypes.c_int, ctypes.c_int64,
                                            _i64p, _dp, _dp]
        lib.race_oracle_forward.restype = ctypes.c_int
        lib.race_oracle_backward.argtypes = [_dp, _dp, _dp, _dp, _dp, ctypes.c_int64,
                                             ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_double, ctypes.c_int,
                                             _dp, _dp, _dp, _dp]
        lib.race_oracle_backward.restype = ctypes.c_int
        lib.race_oracle_state.argtypes = [_dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_double, _dp]
        lib.race_oracle_state.restype = ctypes.c_int
        lib.race_oracle_num_threads.argtypes = []
        lib.race_oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def num_threads() -> int:
    """OpenMP threads the oracle uses (set OMP_NUM_THREADS before the first call)."""
    return int(_load().race_oracle_num_threads())


def features(x, W, tau: float) -> np.ndarray:
    """phi(x) for rows x[..., d] -> [..., L*R]; tau = 0 gives the one-hot sign hash."""
    x = _f64(x)
    W = _f64(W)
    L, P, d = W.shape
    R = 1 << P
    rows = x.reshape(-1, d)
    out = np.empty((rows.shape[0], L * R), dtype=np.float64)
    lib = _load()
    beta = 0.0 if tau == 0 else 1.0 / tau
    for i in range(rows.shape[0]):
        r = np.ascontiguousarray(rows[i])
        o = np.empty(L * R, dtype=np.float64)
        lib.race_oracle_features(_ptr(r), d, _ptr(W), L, P, beta, int(tau == 0), _ptr(o))
        out[i] = o
    return out.reshape(x.shape[:-1] + (L * R,))


def features_backward(x, W, tau: float, dphi) -> np.ndarray:
    """Vector-Jacobian product of ``features`` (soft hashing)."""
    x = _f64(x)
    W = _f64(W)
    L, P, d = W.shape
    R = 1 << P
    rows = x.reshape(-1, d)
    g = _f64(dphi).reshape(-1, L * R)
    out = np.empty_like(rows)
    lib = _load()
    for i in range(rows.shape[0]):
        r = np.ascontiguousarray(rows[i])
        gi = np.ascontiguousarray(g[i])
        o = np.empty(d, dtype=np.float64)
        lib.race_oracle_features_backward(_ptr(r), d, _ptr(W), L, P, 1.0 / tau, _ptr(gi), _ptr(o))
        out[i] = o
    return out.reshape(x.shape)


def hash_indices(x, W) -> np.ndarray:
    """Hard sign-hash bucket of every table: [..., d] -> [..., L] int32."""
    x = _f64(x)
    W = _f64(W)
    L, P, d = W.shape
    rows = x.reshape(-1, d)
    out = np.empty((rows.shape[0], L), dtype=np.int32)
    lib = _load()
    for i in range(rows.shape[0]):
        r = np.ascontiguousarray(rows[i])
        o = np.empty(L, dtype=np.int32)
        lib.race_oracle_hash_indices(_ptr(r), d, _ptr(W), L, P, o.ctypes.data_as(_i32p))
        out[i] = o
    return out.reshape(x.shape[:-1] + (L,))


def forward(q, k, v, W, tau: float, causal: bool, rows=None):
    """RACE attention forward.  q, k, v: [..., N, d]; W: [L, P, d].

    Returns (out [..., n, d], den [..., n]) with n = N, or n = len(rows) when ``rows``
    (ascending query indices) selects a subset.  Causal runs stream the keys in order,
    so a subset costs one pass over the sequence and O(L*R*d) memory.
    """
    q, k, v, W = _f64(q), _f64(k), _f64(v), _f64(W)
    *lead, N, d = q.shape
    BH = int(np.prod(lead)) if lead else 1
    L, P, dw = W.shape
    assert dw == d and k.shape == q.shape and v.shape == q.shape
    if rows is None:
        n = N
        rows_arr = None
        rows_ptr = ctypes.cast(None, _i64p)
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        assert np.all(np.diff(rows_arr) > 0) and (rows_arr.size == 0 or (rows_arr[0] >= 0 and rows_arr[-1] < N))
        n = rows_arr.size
        rows_ptr = rows_arr.ctypes.data_as(_i64p)
    out = np.empty((BH, n, d), dtype=np.float64)
    den = np.empty((BH, n), dtype=np.float64)
    rc = _load().race_oracle_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(W), BH, N, d, L, P,
                                     float(tau), int(bool(causal)), n, rows_ptr,
                                     _ptr(out), _ptr(den))
    if rc != 0:
        raise RuntimeError("race_oracle_forward failed with code %d" % rc)
    return out.reshape(tuple(lead) + (n, d)), den.reshape(tuple(lead) + (n,))


def backward(q, k, v, W, dout, tau: float, causal: bool, with_dw: bool = False):
    """Gradients (dq, dk, dv) of sum(out * dout) for the forward above (soft hashing); with
    ``with_dw`` also dW [L, P, d], the gradient with respect to the hyperplanes (shared by
    every head, so summed over them)."""
    q, k, v, W, dout = _f64(q), _f64(k), _f64(v), _f64(W), _f64(dout)
    *lead, N, d = q.shape
    BH = int(np.prod(lead)) if lead else 1
    L, P, _ = W.shape
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    dW = np.empty_like(W) if with_dw else None
    rc = _load().race_oracle_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(W), _ptr(dout), BH, N, d,
                                      L, P, float(tau), int(bool(causal)),
                                      _ptr(dq), _ptr(dk), _ptr(dv),
                                      _ptr(dW) if with_dw else ctypes.cast(None, _dp))
    if rc != 0:
        raise RuntimeError("race_oracle_backward failed with code %d" % rc)
    return (dq, dk, dv, dW) if with_dw else (dq, dk, dv)

def state(k, v, W, tau: float) -> np.ndarray:
    """Bucket statistics H[m, c] = sum_j phi(k_j)[m] [v_j, 1][c] over every key of each head
    (zh §2.2: A = column d, B = columns 0..d-1 of every table).  k, v: [..., N, d];
    returns [..., L*2^P, d+1]."""
    k, v, W = _f64(k), _f64(v), _f64(W)
    *lead, N, d = k.shape
    BH = int(np.prod(lead)) if lead else 1
    L, P, dw = W.shape
    assert dw == d and v.shape == k.shape
    H = np.empty((BH, L << P, d + 1), dtype=np.float64)
    rc = _load().race_oracle_state(_ptr(k), _ptr(v), _ptr(W), BH, N, d, L, P, float(tau), _ptr(H))
    if rc != 0:
        raise RuntimeError("race_oracle_state failed with code %d" % rc)
    return H.reshape(tuple(lead) + (L << P, d + 1))
