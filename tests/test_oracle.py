"""Pins for the fp64 oracle: what the pages and the mathematics fix, independent of the oracle.

Each test names the fact it checks.  Sources: "RACE Attention: A Strictly Linear-Time
Attention for Long-Sequence Training" (gist.science summaries of arXiv 2510.04008): the
sharpened angular kernel (es §2.1, zh §2.1), soft bucketization with tanh and a softmax
over hypercube corners (zh §2.2, pt §2), bucket statistics and the global read-out (zh
§2.2, Algorithm 1), cumulative statistics for the causal form (zh §2.3, Algorithm 2),
the error bound of Theorem 2 (zh §3).
"""
import json
import os

import numpy as np
import pytest
from scipy.special import expit

import oracle
from oracle import bruteforce

RNG = np.random.default_rng(1234)


def _case(N=12, d=6, L=3, P=3, seed=0, scale=1.0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((N, d)) * scale
    k = rng.standard_normal((N, d)) * scale
    v = rng.standard_normal((N, d))
    W = rng.standard_normal((L, P, d))
    return q, k, v, W


# ------------------------------------------------------------------------------------------
# Soft hash (zh §2.2): each table's assignment is a distribution over the 2^P corners
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("P", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("tau", [0.25, 1.0, 3.0])
def test_features_are_distributions_over_corners(P, tau):
    q, _, _, W = _case(N=7, d=5, L=4, P=P, seed=P)
    phi = oracle.features(q, W, tau).reshape(7, 4, 1 << P)
    assert np.all(phi > 0)
    np.testing.assert_allclose(phi.sum(-1), 1.0, rtol=0, atol=1e-14)


@pytest.mark.parametrize("P", [1, 2, 3, 4])
@pytest.mark.parametrize("tau", [0.5, 1.0, 2.0])
def test_softmax_over_corners_equals_product_of_plane_sigmoids(P, tau):
    """softmax_r(beta * c_r . u) factorises over planes, because the logit is linear in the
    corner's signs: phi_r = prod_p sigmoid(2 beta c_rp u_p).  A wrong corner enumeration,
    sign convention or beta scaling breaks the identity."""
    q, _, _, W = _case(N=5, d=7, L=3, P=P, seed=10 + P)
    beta = 1.0 / tau
    phi = oracle.features(q, W, tau).reshape(5, 3, 1 << P)
    u = np.tanh(np.einsum("lpd,nd->nlp", W, q / np.linalg.norm(q, axis=1, keepdims=True)))
    for r in range(1 << P):
        signs = np.array([1.0 if (r >> p) & 1 else -1.0 for p in range(P)])
        expect = np.prod(expit(2.0 * beta * signs * u), axis=-1)
        np.testing.assert_allclose(phi[:, :, r], expect, rtol=1e-12, atol=1e-15)


def test_corner_mean_of_each_sign_is_tanh_of_beta_u():
    """Under the corner distribution each sign c_p is an independent +-1 variable with mean
    tanh(beta u_p) -- a closed form of the soft assignment."""
    q, _, _, W = _case(N=4, d=9, L=2, P=4, seed=3)
    tau = 0.7
    phi = oracle.features(q, W, tau).reshape(4, 2, 16)
    u = np.tanh(np.einsum("lpd,nd->nlp", W, q / np.linalg.norm(q, axis=1, keepdims=True)))
    for p in range(4):
        signs = np.array([1.0 if (r >> p) & 1 else -1.0 for r in range(16)])
        np.testing.assert_allclose((phi * signs).sum(-1), np.tanh(u[:, :, p] / tau), rtol=1e-12,
                                   atol=1e-14)


def test_large_beta_recovers_sign_hash():
    """beta -> infinity turns the soft assignment into the one-hot sign hash (Theorem 2's
    bias term P/beta vanishes)."""
    q, _, _, W = _case(N=50, d=8, L=6, P=3, seed=4)
    idx = oracle.hash_indices(q, W)
    phi = oracle.features(q, W, 1e-4).reshape(50, 6, 8)
    u = np.tanh(np.einsum("lpd,nd->nlp", W, q / np.linalg.norm(q, axis=1, keepdims=True)))
    clear = np.min(np.abs(u), axis=-1) > 5e-3  # margins where 1e4 * |u| dominates
    assert clear.mean() > 0.9
    np.testing.assert_array_equal(phi.argmax(-1)[clear], idx[clear])
    assert np.all(phi.max(-1)[clear] > 0.99)
    hard = oracle.features(q, W, 0.0).reshape(50, 6, 8)
    np.testing.assert_array_equal(hard.argmax(-1), idx)
    np.testing.assert_array_equal(hard.sum(-1), 1.0)


# ------------------------------------------------------------------------------------------
# Golden worked examples
# ------------------------------------------------------------------------------------------

def test_golden_angular_kernel(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "angular_kernel.json")))
    for c in g["cases"]:
        t = np.pi * c["theta_over_pi"]
        val = bruteforce.angular_kernel(np.array([[1.0, 0.0]]),
                                        np.array([[np.cos(t), np.sin(t)]]), c["gamma"])
        np.testing.assert_allclose(val[0, 0], c["sim"], rtol=1e-12, atol=1e-15)


def test_golden_hard_hash(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "hard_hash_example.json")))
    W = np.array(g["W"])
    keys = np.array(g["keys"], dtype=float)
    vals = np.array(g["values"], dtype=float)
    np.testing.assert_array_equal(oracle.hash_indices(keys, W), np.array(g["hash_indices"]))
    # bidirectional (Algorithm 1): the queries read every key
    qn = np.array(g["noncausal_queries"], dtype=float)
    n = len(qn)
    # forward takes equal-length q/k/v: pad the query list, read back the first n rows
    qpad = np.concatenate([qn, np.ones((len(keys) - n, 2))])
    o, den = oracle.forward(qpad, keys, vals, W, 0.0, False)
    np.testing.assert_allclose(o[:n], g["noncausal_out"], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(den[:n], g["noncausal_den"], rtol=0, atol=0)
    # causal (Algorithm 2)
    o, den = oracle.forward(np.array(g["causal_queries"], float), keys, vals, W, 0.0, True)
    np.testing.assert_allclose(o, g["causal_out"], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(den, g["causal_den"], rtol=0, atol=0)
    s = g["single_table"]
    o, den = oracle.forward(np.array(s["queries"], float), np.array(s["keys"], float),
                            np.array(s["values"], float), np.array(s["W"]), 0.0, True)
    np.testing.assert_allclose(o, s["causal_out"], rtol=0, atol=0)
    np.testing.assert_allclose(den, s["causal_den"], rtol=0, atol=0)


# ------------------------------------------------------------------------------------------
# The scan form equals the pairwise estimator; convergence to the angular kernel
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau", [0.0, 0.5, 2.0])
def test_scan_equals_pairwise_estimator(causal, tau):
    """Algorithms 1/2 keep per-bucket sums instead of the N x N matrix; expanding the sums
    back over keys must give the same numbers (zh §2.2-2.3)."""
    q, k, v, W = _case(N=40, d=8, L=3, P=3, seed=5)
    o, den = oracle.forward(q, k, v, W, tau, causal)
    po, pden = bruteforce.pairwise_attention(oracle.features(q, W, tau), oracle.features(k, W, tau),
                                             v, causal)
    np.testing.assert_allclose(den, pden, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(o, po, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("P", [1, 2, 3])
def test_hard_hash_converges_to_angular_attention(P, causal):
    """With sign hashing, two vectors share a bucket of a table with probability
    (1 - theta/pi)^P, so averaging over L tables converges to attention with the sharpened
    angular kernel, gamma = P (es §2.1 'gamma, or P in the algorithm'; Theorem 2 zh §3:
    error O(sqrt(log(N/delta)/L)))."""
    rng = np.random.default_rng(100 + P)
    N, d = 8, 4
    q = rng.standard_normal((N, d))
    k = rng.standard_normal((N, d))
    v = rng.standard_normal((N, d))
    ref, _ = bruteforce.angular_attention(q, k, v, P, causal)
    errs = []
    for L in (1000, 10000, 100000):
        W = rng.standard_normal((L, P, d))
        o, den = oracle.forward(q, k, v, W, 0.0, causal)
        # the mean collision count per table estimates sum_j (1-theta/pi)^P
        errs.append(np.abs(o - ref).max())
        if L == 100000:
            kern = bruteforce.angular_kernel(q, k, P)
            exp_den = (np.tril(kern) if causal else kern).sum(1) * L
            np.testing.assert_allclose(den / exp_den, 1.0, atol=0.03)
    assert errs[2] < 0.03, errs
    assert errs[2] < errs[0] / 3.0, errs


def test_soft_hash_error_falls_as_beta_grows():
    """Theorem 2's bias term O(P/beta): at fixed large L the soft estimator approaches the
    angular-kernel attention as beta = 1/tau grows."""
    rng = np.random.default_rng(7)
    N, d, P, L = 8, 4, 2, 60000
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    W = rng.standard_normal((L, P, d))
    ref, _ = bruteforce.angular_attention(q, k, v, P, False)
    errs = [np.abs(oracle.forward(q, k, v, W, tau, False)[0] - ref).max() for tau in (2.0, 0.2, 0.01)]
    assert errs[0] > errs[1] > errs[2], errs
    assert errs[2] < 0.03, errs


# ------------------------------------------------------------------------------------------
# Structure: causality, convexity, invariances
# ------------------------------------------------------------------------------------------

def test_causal_rows_ignore_later_tokens():
    q, k, v, W = _case(N=30, d=6, L=4, P=2, seed=8)
    o, den = oracle.forward(q, k, v, W, 0.5, True)
    np.testing.assert_allclose(o[0], v[0], rtol=1e-14, atol=1e-15)  # the only key is k_0
    for i in (0, 7, 19):
        k2, v2 = k.copy(), v.copy()
        k2[i + 1:] = RNG.standard_normal(k2[i + 1:].shape)
        v2[i + 1:] = RNG.standard_normal(v2[i + 1:].shape)
        o2, den2 = oracle.forward(q, k2, v2, W, 0.5, True)
        np.testing.assert_array_equal(o2[: i + 1], o[: i + 1])
        np.testing.assert_array_equal(den2[: i + 1], den[: i + 1])
        assert not np.allclose(o2[i + 1:], o[i + 1:])


@pytest.mark.parametrize("causal", [False, True])
def test_outputs_are_convex_combinations_of_values(causal):
    q, k, v, W = _case(N=60, d=5, L=5, P=3, seed=9)
    o, den = oracle.forward(q, k, v, W, 0.5, causal)
    assert np.all(den > 0)
    for i in range(60):
        vv = v[: i + 1] if causal else v
        assert np.all(o[i] >= vv.min(0) - 1e-12) and np.all(o[i] <= vv.max(0) + 1e-12)


def test_invariances():
    q, k, v, W = _case(N=25, d=6, L=4, P=3, seed=11)
    o, den = oracle.forward(q, k, v, W, 0.5, False)
    perm = RNG.permutation(25)
    o2, _ = oracle.forward(q, k[perm], v[perm], W, 0.5, False)
    np.testing.assert_allclose(o2, o, rtol=1e-12, atol=1e-13)
    s = RNG.uniform(0.1, 10.0, size=(25, 1))
    o3, _ = oracle.forward(q * s, k * s[::-1], v, W, 0.5, False)
    np.testing.assert_allclose(o3, o, rtol=1e-12, atol=1e-13)
    # identical keys: every query weighs every (admissible) value equally
    kk = np.repeat(k[:1], 25, axis=0)
    o4, _ = oracle.forward(q, kk, v, W, 0.5, False)
    np.testing.assert_allclose(o4, np.repeat(v.mean(0, keepdims=True), 25, 0), rtol=1e-12, atol=1e-13)
    o5, _ = oracle.forward(q, kk, v, W, 0.5, True)
    np.testing.assert_allclose(o5, np.cumsum(v, 0) / np.arange(1, 26)[:, None], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_row_subset_matches_full_run(causal):
    q, k, v, W = _case(N=5000, d=8, L=4, P=3, seed=12)
    o, den = oracle.forward(q, k, v, W, 0.5, causal)
    rows = np.array([0, 1, 2047, 2048, 2049, 4095, 4999])
    os_, dens = oracle.forward(q, k, v, W, 0.5, causal, rows=rows)
    np.testing.assert_array_equal(os_, o[rows])
    np.testing.assert_array_equal(dens, den[rows])


def test_zero_length_and_batch_layout():
    q, k, v, W = _case(N=0, d=4, L=2, P=2, seed=13)
    o, den = oracle.forward(q, k, v, W, 0.5, True)
    assert o.shape == (0, 4) and den.shape == (0,)
    rng = np.random.default_rng(14)
    qb, kb, vb = (rng.standard_normal((2, 3, 9, 4)) for _ in range(3))
    Wb = rng.standard_normal((2, 2, 4))
    ob, _ = oracle.forward(qb, kb, vb, Wb, 0.5, True)
    o12, _ = oracle.forward(qb[1, 2], kb[1, 2], vb[1, 2], Wb, 0.5, True)
    np.testing.assert_array_equal(ob[1, 2], o12)


# ------------------------------------------------------------------------------------------
# Backward: finite differences and identities
# ------------------------------------------------------------------------------------------

def _fd_grads(q, k, v, W, do, tau, causal, h=1e-6):
    def loss(q_, k_, v_):
        return float((oracle.forward(q_, k_, v_, W, tau, causal)[0] * do).sum())
    grads = []
    for which in range(3):
        base = [q, k, v]
        g = np.zeros_like(base[which])
        for idx in np.ndindex(g.shape):
            plus = [b.copy() for b in base]
            minus = [b.copy() for b in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        grads.append(g)
    return grads


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau", [0.5, 1.0])
def test_backward_matches_finite_differences(causal, tau):
    q, k, v, W = _case(N=8, d=4, L=2, P=2, seed=15)
    do = np.random.default_rng(16).standard_normal(q.shape)
    dq, dk, dv = oracle.backward(q, k, v, W, do, tau, causal)
    fq, fk, fv = _fd_grads(q, k, v, W, do, tau, causal)
    for a, b in ((dq, fq), (dk, fk), (dv, fv)):
        np.testing.assert_allclose(a, b, rtol=1e-6, atol=1e-8 * np.abs(b).max())


def test_features_backward_matches_finite_differences():
    q, _, _, W = _case(N=3, d=5, L=3, P=3, seed=17)
    g = np.random.default_rng(18).standard_normal((3, 24))
    dx = oracle.features_backward(q, W, 0.6, g)
    h = 1e-6
    for i in range(3):
        for c in range(5):
            a, b = q[i].copy(), q[i].copy()
            a[c] += h
            b[c] -= h
            fd = ((oracle.features(a, W, 0.6) - oracle.features(b, W, 0.6)) @ g[i]) / (2 * h)
            np.testing.assert_allclose(dx[i, c], fd, rtol=1e-6, atol=1e-9)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_identities(causal):
    """Each output row is a normalised average of values, so sum_j dv_j = sum_i dO_i; the
    output ignores the scale of q and k rows, so dq_i . q_i = 0 and dk_j . k_j = 0."""
    q, k, v, W = _case(N=300, d=8, L=4, P=3, seed=19, scale=3.0)
    do = np.random.default_rng(20).standard_normal(q.shape)
    dq, dk, dv = oracle.backward(q, k, v, W, do, 0.5, causal)
    np.testing.assert_allclose(dv.sum(0), do.sum(0), rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose((dq * q).sum(1), 0.0, atol=1e-12 * np.abs(dq).max() * 3)
    np.testing.assert_allclose((dk * k).sum(1), 0.0, atol=1e-12 * np.abs(dk).max() * 3)


def test_backward_spans_feature_blocks():
    """A causal run longer than the oracle's feature block walks the same sums."""
    q, k, v, W = _case(N=4500, d=4, L=2, P=2, seed=21)
    do = np.random.default_rng(22).standard_normal(q.shape)
    dq, dk, dv = oracle.backward(q, k, v, W, do, 0.5, True)
    # rows of the last block only see the tail of the suffix sums: recompute them on a
    # sequence whose first rows are the same and check the prefix-only quantity dq
    dq2, _, _ = oracle.backward(q[:2100], k[:2100], v[:2100], W, do[:2100], 0.5, True)
    np.testing.assert_allclose(dq[:2100], dq2, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dv.sum(0), do.sum(0), rtol=1e-9, atol=1e-9)


# ------------------------------------------------------------------------------------------
# Bucket statistics (zh §2.2): the state a streaming (decode-time) step continues from
# ------------------------------------------------------------------------------------------

def test_state_hard_hash_sums_values_per_bucket():
    """With hard hashing every key lands in one bucket per table, so each state row is the
    sum of [v_j, 1] over the keys whose sign-hash index picks that corner."""
    _, k, v, W = _case(N=200, d=6, L=3, P=3, seed=23)
    L, P = W.shape[0], W.shape[1]
    R = 1 << P
    H = oracle.state(k, v, W, 0.0)
    idx = oracle.hash_indices(k, W)
    want = np.zeros((L * R, k.shape[1] + 1))
    for j in range(k.shape[0]):
        for l in range(L):
            want[l * R + idx[j, l], :-1] += v[j]
            want[l * R + idx[j, l], -1] += 1.0
    np.testing.assert_allclose(H, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("tau", [0.25, 1.0])
def test_state_tables_split_every_key_once(tau):
    """A soft assignment is a distribution over each table's corners, so summed over the
    corners of any one table the state counts every key once: sum_r A_l[r] = N and
    sum_r B_l[r, :] = sum_j v_j."""
    _, k, v, W = _case(N=150, d=5, L=4, P=3, seed=24)
    L, P = W.shape[0], W.shape[1]
    H = oracle.state(k, v, W, tau).reshape(L, 1 << P, -1).sum(1)
    np.testing.assert_allclose(H[:, -1], k.shape[0], rtol=1e-12)
    np.testing.assert_allclose(H[:, :-1], np.broadcast_to(v.sum(0), (L, v.shape[1])), rtol=1e-11, atol=1e-11)


def test_state_is_additive_over_tokens():
    """The statistics are a sum over keys: a run across the oracle's feature blocks equals the
    sum of the states of its two parts."""
    _, k, v, W = _case(N=4500, d=4, L=2, P=2, seed=25)
    H = oracle.state(k, v, W, 0.5)
    H2 = oracle.state(k[:2100], v[:2100], W, 0.5) + oracle.state(k[2100:], v[2100:], W, 0.5)
    np.testing.assert_allclose(H, H2, rtol=1e-12, atol=1e-10)


def test_state_read_out_is_the_last_causal_row():
    """Algorithm 2 reads query i out of the statistics of keys 0..i: reading the last query
    out of the state of the whole prefix gives the causal forward's last row."""
    q, k, v, W = _case(N=40, d=6, L=3, P=2, seed=26)
    H = oracle.state(k, v, W, 0.5)
    y = oracle.features(q[-1], W, 0.5) @ H
    out, den = oracle.forward(q, k, v, W, 0.5, True, rows=[39])
    np.testing.assert_allclose(den[0], y[-1], rtol=1e-12)
    np.testing.assert_allclose(out[0], y[:-1] / y[-1], rtol=1e-12)


# ------------------------------------------------------------------------------------------
# Gradient with respect to the hyperplanes W (chain rule through p = W_l x^; the pages
# treat W as fixed random projections, zh §2.2, so this is the learnable-W variant)
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("tau", [0.5, 1.0])
def test_hyperplane_gradient_matches_finite_differences(causal, tau):
    q, k, v, W = _case(N=9, d=4, L=2, P=2, seed=27)
    do = np.random.default_rng(28).standard_normal(q.shape)
    dq, dk, dv, dW = oracle.backward(q, k, v, W, do, tau, causal, with_dw=True)
    h = 1e-6
    fd = np.zeros_like(W)
    for idx in np.ndindex(W.shape):
        Wp, Wm = W.copy(), W.copy()
        Wp[idx] += h
        Wm[idx] -= h
        lp = float((oracle.forward(q, k, v, Wp, tau, causal)[0] * do).sum())
        lm = float((oracle.forward(q, k, v, Wm, tau, causal)[0] * do).sum())
        fd[idx] = (lp - lm) / (2 * h)
    np.testing.assert_allclose(dW, fd, rtol=1e-6, atol=1e-8 * np.abs(fd).max())
    # the other gradients are unchanged by asking for dW
    for a, b in zip((dq, dk, dv), oracle.backward(q, k, v, W, do, tau, causal)):
        np.testing.assert_array_equal(a, b)


def test_hyperplane_gradient_sums_over_heads_and_blocks():
    """W is shared by every head, so the batch's dW is the sum of the heads' dW; a run longer
    than the oracle's feature block accumulates across blocks."""
    rng = np.random.default_rng(29)
    q, k, v, do = (rng.standard_normal((2, 2100, 4)) for _ in range(4))
    W = rng.standard_normal((2, 2, 4))
    dW = oracle.backward(q, k, v, W, do, 0.5, True, with_dw=True)[3]
    parts = [oracle.backward(q[h], k[h], v[h], W, do[h], 0.5, True, with_dw=True)[3] for h in range(2)]
    np.testing.assert_allclose(dW, parts[0] + parts[1], rtol=1e-12, atol=1e-12)


def test_hyperplane_gradient_of_a_scale_free_loss():
    """Scaling one hyperplane row W_lp by a > 0 changes p_lp = W_lp x^ by the same factor;
    the loss's derivative along that direction, sum_c W_lpc dW_lpc, must equal
    d/da L(a W_lp) at a = 1 (a directional check of every row at once)."""
    q, k, v, W = _case(N=20, d=5, L=3, P=2, seed=30)
    do = np.random.default_rng(31).standard_normal(q.shape)
    dW = oracle.backward(q, k, v, W, do, 0.5, True, with_dw=True)[3]
    h = 1e-6
    for l in range(W.shape[0]):
        for p in range(W.shape[1]):
            Wp, Wm = W.copy(), W.copy()
            Wp[l, p] *= 1 + h
            Wm[l, p] *= 1 - h
            lp = float((oracle.forward(q, k, v, Wp, 0.5, True)[0] * do).sum())
            lm = float((oracle.forward(q, k, v, Wm, 0.5, True)[0] * do).sum())
            np.testing.assert_allclose((W[l, p] * dW[l, p]).sum(), (lp - lm) / (2 * h), rtol=1e-6, atol=1e-9)
