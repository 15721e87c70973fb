"""O(N^2) forms used to pin the oracle -- TEST INFRASTRUCTURE ONLY.

* ``angular_attention``: the target the pages say RACE approximates, the sharpened angular
  kernel sim(q,k) = (1 - arccos(q^.k^)/pi)^gamma used in place of exp(q.k) inside an
  attention row ("RACE Attention: A Strictly Linear-Time Attention for Long-Sequence
  Training", es §2.1, fr §2A, zh §2.1; gamma plays the role of P, es §2.1).
* ``pairwise_attention``: the RACE estimator written pair by pair,
  o_i = sum_j w_ij v_j / sum_j w_ij with w_ij = phi(q_i) . phi(k_j) summed over the tables
  (zh §2.2, the read-out sum_l phi_l(q)^T B_l / sum_l phi_l(q)^T A_l expanded over keys),
  with j <= i for the causal form (zh §2.3).

Both are plain numpy in fp64 and share nothing with the scan form in ``race_oracle.c``
except the feature vectors handed to ``pairwise_attention``.
"""
from __future__ import annotations

import numpy as np


def angular_kernel(q, k, gamma: float) -> np.ndarray:
    """(1 - theta/pi)^gamma for every query/key pair, theta the angle between them."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    qh = q / np.linalg.norm(q, axis=-1, keepdims=True)
    kh = k / np.linalg.norm(k, axis=-1, keepdims=True)
    cos = np.clip(qh @ kh.T, -1.0, 1.0)
    return (1.0 - np.arccos(cos) / np.pi) ** gamma


def _masked_rows(w: np.ndarray, v: np.ndarray, causal: bool):
    if causal:
        w = np.tril(w)
    num = w @ v
    den = w.sum(axis=1)
    out = np.where(den[:, None] != 0, num / np.where(den == 0, 1.0, den)[:, None], 0.0)
    return out, den


def angular_attention(q, k, v, gamma: float, causal: bool = False):
    """Attention with the sharpened angular kernel in place of softmax: (out, den)."""
    w = angular_kernel(q, k, gamma)
    return _masked_rows(w, np.asarray(v, dtype=np.float64), causal)


def pairwise_attention(phi_q, phi_k, v, causal: bool = False):
    """RACE estimator from feature vectors, pair by pair: (out, den)."""
    w = np.asarray(phi_q, dtype=np.float64) @ np.asarray(phi_k, dtype=np.float64).T
    return _masked_rows(w, np.asarray(v, dtype=np.float64), causal)
