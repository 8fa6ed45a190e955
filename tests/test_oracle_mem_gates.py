"""Pins of the oracle's per-memory gates (each routed memory with its own
W_beta, W_a, A, b_a: the per-memory variant of the gates, "MoM: Linear
Sequence Modeling with Mixture-of-Memories", Summary: every memory has its
own recurrent update):

* memory_gates against pure-Python sums per element, three memories with
  different weights; planted mistakes (the shared gates, another memory's
  weights, sigmoid and softplus swapped) fail it;
* a layer whose per-memory gates all equal the shared ones is the layer
  without per-memory gates;
* the mixed-state form equals the output sum, and decode continues a
  prefill, with per-memory gates.
"""
import math

import numpy as np
import pytest

from mixture_memories_layer_b200 import synth
from oracle import mom_oracle as orc


def _sig(z):
    return 1.0 / (1.0 + math.exp(-z))


def _check_gates(fn):
    rng = np.random.default_rng(41)
    N, D, H, M = 3, 7, 2, 3
    p = dict(w_beta_mem=rng.standard_normal((M, H, D)), w_a_mem=rng.standard_normal((M, H, D)),
             A_mem=rng.uniform(0, 2.7, (M, H)), b_a_mem=rng.uniform(-4, 0, (M, H)),
             w_beta=rng.standard_normal((H, D)), w_a=rng.standard_normal((H, D)),
             A=rng.uniform(0, 2.7, H), b_a=rng.uniform(-4, 0, H))
    x = rng.standard_normal((N, D))
    for m in range(M):
        b, la = fn(x, p, m)
        for n in range(N):
            for h in range(H):
                zb = sum(x[n, i] * p["w_beta_mem"][m][h][i] for i in range(D))
                za = sum(x[n, i] * p["w_a_mem"][m][h][i] for i in range(D)) + p["b_a_mem"][m][h]
                assert abs(b[n, h] - _sig(zb)) < 1e-13, ("beta", m, n, h)
                ref = -math.exp(p["A_mem"][m][h]) * math.log1p(math.exp(za))
                assert abs(la[n, h] - ref) < 1e-12, ("log alpha", m, n, h)


def test_memory_gates_pure_python():
    _check_gates(orc.memory_gates)


def _shared_gates(x, p, m):
    b = orc.sigmoid(x @ p["w_beta"].T)
    return b, -np.exp(p["A"]) * orc.softplus(x @ p["w_a"].T + p["b_a"])


def _next_memory(x, p, m):
    return orc.memory_gates(x, p, (m + 1) % len(p["A_mem"]))


def _swapped_nonlinearities(x, p, m):
    b = orc.softplus(x @ p["w_beta_mem"][m].T)
    return b, -np.exp(p["A_mem"][m]) * orc.sigmoid(x @ p["w_a_mem"][m].T + p["b_a_mem"][m])


@pytest.mark.parametrize("planted", [_shared_gates, _next_memory, _swapped_nonlinearities])
def test_memory_gates_pin_catches_planted_mistakes(planted):
    with pytest.raises(AssertionError):
        _check_gates(planted)


def _tiny(seed=51, N=24, varlen=False, rule="gated_delta"):
    w = synth.Workload("t", 1, N, 16, 2, 8, 4, 2, "f32", seed=seed, mem_gates=True)
    rng = np.random.default_rng(seed)
    p = synth.make_weights(w, rng)
    cu = np.array([0, 9, 9, 20, 31], np.int32) if varlen else np.array([0, N], np.int32)
    return w, p, synth.make_tokens(w, rng, int(cu[-1])), cu


def test_equal_per_memory_gates_are_the_shared_gates():
    w, p, x, cu = _tiny()
    M = w.n_mem
    p["w_beta_mem"] = np.stack([p["w_beta"]] * M)
    p["w_a_mem"] = np.stack([p["w_a"]] * M)
    p["A_mem"] = np.stack([p["A"]] * M)
    p["b_a_mem"] = np.stack([p["b_a"]] * M)
    with_gates = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head)
    plain = {k: v for k, v in p.items() if not k.endswith("_mem")}
    without = orc.mom_forward(x, plain, cu, w.top_k, w.heads, w.d_head)
    assert np.allclose(with_gates["out"], without["out"], atol=1e-13)
    assert np.allclose(with_gates["h_mem"], without["h_mem"], atol=1e-13)


def test_per_memory_gates_change_the_routed_memories_only():
    w, p, x, cu = _tiny(seed=52)
    plain = {k: v for k, v in p.items() if not k.endswith("_mem")}
    a = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head)
    b = orc.mom_forward(x, plain, cu, w.top_k, w.heads, w.d_head)
    assert np.allclose(a["o_shared"], b["o_shared"], atol=0) and np.allclose(a["h_shared"], b["h_shared"], atol=0)
    assert not np.allclose(a["o_mem"], b["o_mem"], atol=1e-6)


@pytest.mark.parametrize("rule", ["gated_delta", "gated_linear"])
@pytest.mark.parametrize("varlen", [False, True])
def test_mixed_state_equals_output_sum_with_per_memory_gates(rule, varlen):
    w, p, x, cu = _tiny(seed=53, varlen=varlen)
    r = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head, rule=rule)
    mixed = orc.mom_forward_mixed_state(x, p, cu, w.top_k, w.heads, w.d_head, rule=rule)
    assert np.allclose(r["out"], mixed, atol=1e-12)


def test_decode_continues_a_prefill_with_per_memory_gates():
    w, p, x, cu = _tiny(seed=54, N=17)
    full = orc.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head)
    pre = orc.mom_forward(x[:16], p, np.array([0, 16]), w.top_k, w.heads, w.d_head)
    st = orc.decode_state_from_prefill(pre["h_shared"], pre["h_mem"])
    out, new, idx, _, _ = orc.mom_decode_step(x[16:17], p, st, w.top_k, w.heads, w.d_head)
    assert np.allclose(out[0], full["out"][16], atol=1e-12)
    for m in range(w.n_mem):
        assert np.allclose(new[0, m], full["h_mem"][m, 0], atol=1e-12)
