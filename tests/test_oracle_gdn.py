"""Pins for the oracle's Gated DeltaNet recurrence and its chunked form.

The per-memory update is Gated DeltaNet's gate and update rule (the authors'
MoM blog post, experiments section; "MoM: Linear Sequence Modeling with
Mixture-of-Memories", Summary), S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T)
+ beta_t v_t k_t^T, o_t = S_t q_t.  The pins below do not re-type the
oracle's expression: they use exact rational arithmetic with the explicit
matrix product, closed forms, and properties of the delta rule
("Sparse Delta Memory ...", gated delta update: forget, then correct the
memory toward v).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import mom_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _frac_matmul(A, B):
    return [[sum(A[i][t] * B[t][j] for t in range(len(B))) for j in range(len(B[0]))] for i in range(len(A))]


def _frac_recurrence(q, k, v, beta, alpha, scale):
    """Explicit S (I - beta k k^T) with full matrix products, exact rationals."""
    dk, dv = len(k[0]), len(v[0])
    S = [[Fraction(0)] * dk for _ in range(dv)]
    outs = []
    for t in range(len(k)):
        P = [[(Fraction(1) if i == j else Fraction(0)) - beta[t] * k[t][i] * k[t][j] for j in range(dk)]
             for i in range(dk)]
        SP = _frac_matmul(S, P)
        S = [[alpha[t] * SP[i][j] + beta[t] * v[t][i] * k[t][j] for j in range(dk)] for i in range(dv)]
        outs.append([sum(S[i][j] * scale * q[t][j] for j in range(dk)) for i in range(dv)])
    return outs, S


def test_recurrence_matches_exact_rational_brute_force():
    rng = np.random.default_rng(0)
    T, dk, dv = 6, 3, 2
    # rational inputs (multiples of 1/8) so the brute force is exact
    q = [[Fraction(int(z), 8) for z in rng.integers(-8, 9, dk)] for _ in range(T)]
    k = [[Fraction(int(z), 8) for z in rng.integers(-8, 9, dk)] for _ in range(T)]
    v = [[Fraction(int(z), 4) for z in rng.integers(-8, 9, dv)] for _ in range(T)]
    beta = [Fraction(int(z), 8) for z in rng.integers(0, 9, T)]
    alpha = [Fraction(int(z), 8) for z in rng.integers(1, 9, T)]
    scale = Fraction(3, 4)
    o_ref, S_ref = _frac_recurrence(q, k, v, beta, alpha, scale)
    f = lambda a: np.array([[float(z) for z in row] for row in a])
    o, S = orc.gdn_recurrence(f(q)[:, None, :], f(k)[:, None, :], f(v)[:, None, :],
                              np.array([float(b) for b in beta])[:, None],
                              np.log(np.array([float(a) for a in alpha]))[:, None],
                              None, float(scale))
    assert np.allclose(o[:, 0, :], f(o_ref), rtol=0, atol=1e-12)
    assert np.allclose(S[0], f(S_ref), rtol=0, atol=1e-12)


def test_golden_scalar_worked_example():
    """Hand-worked scalar case, stored with its derivation."""
    with open(os.path.join(GOLDEN, "gdn_scalar_worked.json")) as fh:
        g = json.load(fh)
    T = len(g["v"])
    arr = lambda a: np.array(a, dtype=np.float64).reshape(T, 1, 1)
    o, S = orc.gdn_recurrence(arr(g["q"]), arr(g["k"]), arr(g["v"]),
                              np.array(g["beta"]).reshape(T, 1),
                              np.log(np.array(g["alpha"])).reshape(T, 1), None, 1.0)
    assert np.allclose(o.reshape(-1), g["o"], atol=1e-12)
    assert abs(S.reshape(-1)[0] - g["S_final"]) < 1e-12


def _rand_inputs(rng, T, H, dk, dv, strong_decay=False):
    q = orc.l2norm(rng.standard_normal((T, H, dk)))
    k = orc.l2norm(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    la = -np.exp(rng.uniform(0, 2.7, (T, H))) * np.logaddexp(0, rng.standard_normal((T, H)) + rng.uniform(-4, 0, (T, H)))
    if strong_decay:
        la[::5] = -20.0
    return q, k, v, beta, la


def test_beta_zero_zero_state_gives_zero():
    rng = np.random.default_rng(1)
    q, k, v, _, la = _rand_inputs(rng, 20, 2, 8, 8)
    o, S = orc.gdn_recurrence(q, k, v, np.zeros((20, 2)), la)
    assert np.all(o == 0) and np.all(S == 0)


def test_no_write_no_decay_reads_initial_state():
    rng = np.random.default_rng(2)
    T, H, d = 15, 2, 8
    q, k, v, _, _ = _rand_inputs(rng, T, H, d, d)
    h0 = rng.standard_normal((H, d, d))
    o, S = orc.gdn_recurrence(q, k, v, np.zeros((T, H)), np.zeros((T, H)), h0, scale=0.5)
    for t in range(T):
        for h in range(H):
            assert np.allclose(o[t, h], 0.5 * h0[h] @ q[t, h], atol=1e-13)
    assert np.allclose(S, h0, atol=0)


def test_decay_only_closed_form():
    rng = np.random.default_rng(3)
    T, H, d = 12, 1, 4
    q, k, v, _, la = _rand_inputs(rng, T, H, d, d)
    h0 = rng.standard_normal((H, d, d))
    o, S = orc.gdn_recurrence(q, k, v, np.zeros((T, H)), la, h0)
    cum = np.cumsum(la[:, 0])
    for t in range(T):
        assert np.allclose(o[t, 0], math.exp(cum[t]) * h0[0] @ q[t, 0], atol=1e-12)
    assert np.allclose(S[0], math.exp(cum[-1]) * h0[0], atol=1e-12)


def test_delta_rule_stores_value_exactly():
    """alpha=1, beta=1, |k|=1: after the write, S_t k_t = v_t."""
    rng = np.random.default_rng(4)
    T, H, d = 10, 2, 6
    q, k, v, _, _ = _rand_inputs(rng, T, H, d, d)
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    S = np.zeros((H, d, d))
    for t in range(T):
        _, S = orc.gdn_step(S, q[t], k[t], v[t], np.ones(H), np.zeros(H))
        for h in range(H):
            assert np.allclose(S[h] @ k[t, h], v[t, h], atol=1e-12)


def test_orthonormal_keys_form_associative_memory():
    """Writing d pairs with orthonormal keys (alpha=beta=1) gives S = V^T K,
    and reading with q = k_j returns v_j."""
    rng = np.random.default_rng(5)
    d = 5
    K, _ = np.linalg.qr(rng.standard_normal((d, d)))
    K = K.T                                   # rows orthonormal
    V = rng.standard_normal((d, d))
    o, S = orc.gdn_recurrence(K[:, None, :], K[:, None, :], V[:, None, :], np.ones((d, 1)), np.zeros((d, 1)))
    assert np.allclose(S[0], V.T @ K, atol=1e-12)
    for j in range(d):
        assert np.allclose(S[0] @ K[j], V[j], atol=1e-12)


def test_scale_is_linear_in_the_readout():
    rng = np.random.default_rng(6)
    q, k, v, b, la = _rand_inputs(rng, 9, 2, 4, 4)
    o1, S1 = orc.gdn_recurrence(q, k, v, b, la, scale=1.0)
    o2, S2 = orc.gdn_recurrence(q, k, v, b, la, scale=0.125)
    assert np.allclose(o2, 0.125 * o1, atol=1e-14) and np.array_equal(S1, S2)


@pytest.mark.parametrize("chunk", [1, 7, 64])
@pytest.mark.parametrize("with_h0", [False, True])
def test_chunked_form_equals_token_loop(chunk, with_h0):
    rng = np.random.default_rng(7 + chunk)
    T, H, dk, dv = 150, 2, 16, 12
    q, k, v, b, la = _rand_inputs(rng, T, H, dk, dv, strong_decay=True)
    h0 = rng.standard_normal((H, dv, dk)) if with_h0 else None
    o_r, S_r = orc.gdn_recurrence(q, k, v, b, la, h0, scale=0.7)
    o_c, S_c = orc.gdn_chunked(q, k, v, b, la, h0, scale=0.7, chunk=chunk)
    assert np.allclose(o_c, o_r, rtol=0, atol=1e-10)
    assert np.allclose(S_c, S_r, rtol=0, atol=1e-10)


def test_state_hand_off():
    rng = np.random.default_rng(8)
    T, H, d = 40, 2, 8
    q, k, v, b, la = _rand_inputs(rng, T, H, d, d)
    o, S = orc.gdn_recurrence(q, k, v, b, la)
    o1, S1 = orc.gdn_recurrence(q[:17], k[:17], v[:17], b[:17], la[:17])
    o2, S2 = orc.gdn_recurrence(q[17:], k[17:], v[17:], b[17:], la[17:], S1)
    assert np.allclose(np.concatenate([o1, o2]), o, atol=1e-13)
    assert np.allclose(S2, S, atol=1e-13)


def test_projection_closed_forms():
    """Zero gate weights give beta = 1/2 and log alpha = -exp(A) softplus(b_a);
    q and k come out with unit norm per head (up to the 1e-6 epsilon)."""
    rng = np.random.default_rng(9)
    N, D, H, d = 7, 16, 2, 4
    p = dict(w_q=rng.standard_normal((H * d, D)), w_k_sh=rng.standard_normal((H * d, D)),
             w_v_sh=rng.standard_normal((H * d, D)), w_beta=np.zeros((H, D)), w_a=np.zeros((H, D)),
             A=np.array([0.0, 1.0]), b_a=np.array([0.0, -2.0]))
    x = rng.standard_normal((N, D))
    q, k_sh, v_sh, beta, la = orc.shared_projections(x, p, H, d)
    assert np.allclose(beta, 0.5, atol=0)
    assert np.allclose(la[:, 0], -math.log(2.0), atol=1e-15)
    assert np.allclose(la[:, 1], -math.e * math.log1p(math.exp(-2.0)), atol=1e-15)
    nq = np.linalg.norm(q, axis=-1)
    assert np.all(np.abs(nq - 1) < 1e-6)
    # v is the plain projection: column c of head h is x . w_v_sh[h*d + c]
    for n in range(N):
        for h in range(H):
            for c in range(d):
                ref = sum(x[n, i] * p["w_v_sh"][h * d + c, i] for i in range(D))
                assert abs(v_sh[n, h, c] - ref) < 1e-12


def test_elementwise_helpers_against_math_module():
    # the gates' building blocks, checked against Python's math library one
    # value at a time, including inputs far outside the workloads' range
    import math
    for z in (-30.0, -5.0, -0.3, 0.0, 0.7, 5.0, 30.0):
        assert abs(orc.softplus(np.array(z)) - math.log1p(math.exp(z))) <= 1e-15 * max(1.0, abs(z))
        assert abs(orc.sigmoid(np.array(z)) - 1.0 / (1.0 + math.exp(-z))) <= 1e-16
        assert abs(orc.sigmoid(np.array(-z)) - (1.0 - orc.sigmoid(np.array(z)))) <= 1e-15
    assert orc.softplus(np.array(800.0)) == 800.0 and orc.softplus(np.array(-800.0)) == 0.0
    y = orc.l2norm(np.array([[3.0, 4.0], [0.0, 0.0]]))
    assert abs(y[0, 0] - 3.0 / math.sqrt(25.0 + orc.NORM_EPS)) <= 1e-16 and np.all(y[1] == 0.0)
    p = orc.softmax(np.array([1000.0, 1000.0, 998.0]))     # no overflow
    assert abs(p[0] - 1.0 / (2.0 + math.exp(-2.0))) <= 1e-15


def _check_memory_kv(fn):
    """Memory m's key/value projection against a pure-Python dot product per
    element (paper card, Summary: every memory has its own key and value
    projections): k is x . W_k^m row, then L2-normalised per head with the
    1e-6 epsilon; v is x . W_v^m row unnormalised.  Three memories with
    different weights, so that reading another memory's weights fails."""
    rng = np.random.default_rng(11)
    N, D, H, d, M = 4, 10, 2, 3, 3
    p = dict(w_k=rng.standard_normal((M, H * d, D)), w_v=rng.standard_normal((M, H * d, D)))
    x = rng.standard_normal((N, D))
    for m in range(M):
        k, v = fn(x, p, m, H, d)
        assert k.shape == (N, H, d) and v.shape == (N, H, d)
        for n in range(N):
            for h in range(H):
                raw = [sum(x[n, i] * p["w_k"][m][h * d + c][i] for i in range(D)) for c in range(d)]
                nrm = math.sqrt(sum(r * r for r in raw) + orc.NORM_EPS)
                for c in range(d):
                    assert abs(k[n, h, c] - raw[c] / nrm) < 1e-12, ("k", m, n, h, c)
                    ref_v = sum(x[n, i] * p["w_v"][m][h * d + c][i] for i in range(D))
                    assert abs(v[n, h, c] - ref_v) < 1e-12, ("v", m, n, h, c)
                # every head of k has unit norm (up to the epsilon)
                assert abs(math.sqrt(sum(float(kc) ** 2 for kc in k[n, h])) - 1.0) < 1e-6


def test_memory_kv_pure_python():
    _check_memory_kv(orc.memory_kv)


def _kv_swapped(x, p, m, H, d):
    n = x.shape[0]
    return (orc.l2norm((x @ p["w_v"][m].T).reshape(n, H, d)), (x @ p["w_k"][m].T).reshape(n, H, d))


def _kv_unnormalised(x, p, m, H, d):
    n = x.shape[0]
    return (x @ p["w_k"][m].T).reshape(n, H, d), (x @ p["w_v"][m].T).reshape(n, H, d)


def _kv_wrong_memory(x, p, m, H, d):
    return orc.memory_kv(x, p, (m + 1) % len(p["w_k"]), H, d)


def _kv_norm_over_all_heads(x, p, m, H, d):
    n = x.shape[0]
    k = orc.l2norm(x @ p["w_k"][m].T).reshape(n, H, d)
    return k, (x @ p["w_v"][m].T).reshape(n, H, d)


@pytest.mark.parametrize("planted", [_kv_swapped, _kv_unnormalised, _kv_wrong_memory, _kv_norm_over_all_heads])
def test_memory_kv_pin_catches_planted_mistakes(planted):
    # the pin above must fail for each plausible mistake in memory_kv
    with pytest.raises(AssertionError):
        _check_memory_kv(planted)
