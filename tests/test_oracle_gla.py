"""Pins of the oracle's second memory rule, the scalar-gated linear form
(the authors' MoM blog post, "Linear Recurrent Memory": linear attention,
RetNet and Mamba2-style memories written as S_t = alpha_t S_{t-1} +
beta_t v_t k_t^T, o_t = S_t (scale q_t)), against forms that do not run
its token loop:

* the closed form of the unrolled recurrence, summed term by term in pure
  Python: o_t = sum_{s<=t} e^(gamma_t - gamma_s) beta_s (scale q_t . k_s) v_s
  + e^(gamma_t) S_0 (scale q_t), S_T likewise (gamma the running sum of
  log alpha);
* causal linear attention (alpha = beta = 1, S_0 = 0), the textbook
  ((Q K^T) masked to s <= t) V;
* at the layer: the mixed-state form equals the output sum, one memory with
  top-1 is two plain recurrences, decode continues a prefill.

Planted mistakes in the step (decay after the write, no write strength,
read before the write) each fail the closed form.
"""
import math

import numpy as np
import pytest

from mixture_memories_layer_b200 import synth
from oracle import mom_oracle as orc


def _inputs(rng, T=9, H=2, dk=3, dv=2):
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    v = rng.standard_normal((T, H, dv))
    beta = rng.uniform(0.1, 0.9, (T, H))
    la = -rng.uniform(0.0, 1.5, (T, H))
    h0 = rng.standard_normal((H, dv, dk))
    return q, k, v, beta, la, h0


def _closed_form(q, k, v, beta, la, h0, scale):
    T, H, dk = k.shape
    dv = v.shape[-1]
    o = [[[0.0] * dv for _ in range(H)] for _ in range(T)]
    S = [[[0.0] * dk for _ in range(dv)] for _ in range(H)]
    for h in range(H):
        gam = []
        acc = 0.0
        for t in range(T):
            acc += la[t, h]
            gam.append(acc)
        for t in range(T):
            for i in range(dv):
                tot = math.exp(gam[t]) * sum(h0[h, i, j] * scale * q[t, h, j] for j in range(dk))
                for s in range(t + 1):
                    qk = sum(scale * q[t, h, j] * k[s, h, j] for j in range(dk))
                    tot += math.exp(gam[t] - gam[s]) * beta[s, h] * qk * v[s, h, i]
                o[t][h][i] = tot
        for i in range(dv):
            for j in range(dk):
                S[h][i][j] = math.exp(gam[-1]) * h0[h, i, j] + sum(
                    math.exp(gam[-1] - gam[s]) * beta[s, h] * v[s, h, i] * k[s, h, j] for s in range(T))
    return np.array(o), np.array(S)


def _check_step(step):
    rng = np.random.default_rng(21)
    q, k, v, beta, la, h0 = _inputs(rng)
    S = h0.copy()
    outs = []
    for t in range(len(q)):
        o, S = step(S, q[t], k[t], v[t], beta[t], la[t], 0.6)
        outs.append(o)
    o_ref, S_ref = _closed_form(q, k, v, beta, la, h0, 0.6)
    assert np.allclose(np.array(outs), o_ref, rtol=0, atol=1e-12)
    assert np.allclose(S, S_ref, rtol=0, atol=1e-12)


def test_gla_step_matches_the_closed_form():
    _check_step(orc.gla_step)
    rng = np.random.default_rng(22)
    q, k, v, beta, la, h0 = _inputs(rng)
    o, S = orc.gdn_recurrence(q, k, v, beta, la, h0, 0.6, rule="gated_linear")
    o_ref, S_ref = _closed_form(q, k, v, beta, la, h0, 0.6)
    assert np.allclose(o, o_ref, atol=1e-12) and np.allclose(S, S_ref, atol=1e-12)


def _decay_after_write(S, q_t, k_t, v_t, beta_t, la_t, scale=1.0):
    a = np.exp(la_t)[:, None, None]
    S = a * (S + beta_t[:, None, None] * v_t[:, :, None] * k_t[:, None, :])
    return np.einsum("hvk,hk->hv", S, scale * q_t), S


def _no_beta(S, q_t, k_t, v_t, beta_t, la_t, scale=1.0):
    S = np.exp(la_t)[:, None, None] * S + v_t[:, :, None] * k_t[:, None, :]
    return np.einsum("hvk,hk->hv", S, scale * q_t), S


def _read_before_write(S, q_t, k_t, v_t, beta_t, la_t, scale=1.0):
    o = np.einsum("hvk,hk->hv", S, scale * q_t)
    S = np.exp(la_t)[:, None, None] * S + beta_t[:, None, None] * v_t[:, :, None] * k_t[:, None, :]
    return o, S


@pytest.mark.parametrize("planted", [_decay_after_write, _no_beta, _read_before_write])
def test_closed_form_catches_planted_mistakes(planted):
    with pytest.raises(AssertionError):
        _check_step(planted)


def test_linear_attention_is_masked_qk_times_v():
    rng = np.random.default_rng(23)
    T, H, d = 12, 2, 5
    q, k, v = (rng.standard_normal((T, H, d)) for _ in range(3))
    ones, zeros = np.ones((T, H)), np.zeros((T, H))
    o, S = orc.gdn_recurrence(q, k, v, ones, zeros, None, 1.0, rule="gated_linear")
    for h in range(H):
        A = np.tril(q[:, h] @ k[:, h].T)
        assert np.allclose(o[:, h], A @ v[:, h], atol=1e-12)
        assert np.allclose(S[h], v[:, h].T @ k[:, h], atol=1e-12)


def _tiny(seed, M=4, k=2, N=24, varlen=False):
    w = synth.Workload("t", 1, N, 16, 2, 8, M, k, "f32", seed=seed)
    rng = np.random.default_rng(seed)
    p = synth.make_weights(w, rng)
    cu = np.array([0, 9, 9, 20, 31], np.int32) if varlen else np.array([0, N], np.int32)
    return w, p, synth.make_tokens(w, rng, int(cu[-1])), cu


@pytest.mark.parametrize("varlen", [False, True])
def test_gla_layer_mixed_state_equals_output_sum(varlen):
    w, p, x, cu = _tiny(31, varlen=varlen)
    r = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head, rule="gated_linear")
    mixed = orc.mom_forward_mixed_state(x, p, cu, w.top_k, w.heads, w.d_head, rule="gated_linear")
    assert np.allclose(r["out"], mixed, atol=1e-12)


def test_gla_layer_one_memory_top1_is_two_plain_recurrences():
    w, p, x, cu = _tiny(32, M=1, k=1)
    r = orc.mom_forward(x, p, cu, 1, w.heads, w.d_head, rule="gated_linear")
    q, k_sh, v_sh, b, la = orc.shared_projections(x, p, w.heads, w.d_head)
    k0, v0 = orc.memory_kv(x, p, 0, w.heads, w.d_head)
    o_sh, _ = _closed_form(q, k_sh, v_sh, b, la, np.zeros((w.heads, w.d_head, w.d_head)), 1.0)
    o_0, S0 = _closed_form(q, k0, v0, b, la, np.zeros((w.heads, w.d_head, w.d_head)), 1.0)
    assert np.allclose(r["out"], o_sh + o_0, atol=1e-11)
    assert np.allclose(r["h_mem"][0, 0], S0, atol=1e-11)


def test_gla_decode_continues_a_prefill():
    w, p, x, cu = _tiny(33, N=17)
    full = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head, rule="gated_linear")
    pre = orc.mom_forward(x[:16], p, np.array([0, 16]), w.top_k, w.heads, w.d_head, rule="gated_linear")
    st = orc.decode_state_from_prefill(pre["h_shared"], pre["h_mem"])
    out, new, idx, _, _ = orc.mom_decode_step(x[16:17], p, st, w.top_k, w.heads, w.d_head, rule="gated_linear")
    assert np.allclose(out[0], full["out"][16], atol=1e-12)
    assert np.allclose(new[0, w.n_mem], full["h_shared"][0], atol=1e-12)
