"""Pins of the reverse-pass oracle (oracle/mom_oracle_bwd.py).

Every gradient is checked against central finite differences of the forward
oracle in fp64, which is pinned on its own (test_oracle_*.py): a dropped
term, a wrong sign or a transposed operand in any adjoint moves some
derivative well past the difference quotient's error (~1e-9 here).  The
recurrence is tested with d_v != d_k so that a transpose cannot hide, and
against the closed form of the beta = 0 case (pure decay); its chunked form
(the one a blocked GPU reverse pass takes) must equal the token loop.
"""
import numpy as np
import pytest

from mixture_memories_layer_b200 import synth
from oracle import mom_oracle as fwd
from oracle import mom_oracle_bwd as bwd

EPS = 1e-6


def _fd(loss, arr, eps=EPS):
    """Central differences of loss() with respect to every element of arr
    (perturbed in place and restored)."""
    g = np.zeros_like(arr)
    it = np.nditer(arr, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        old = arr[i]
        arr[i] = old + eps
        lp = loss()
        arr[i] = old - eps
        lm = loss()
        arr[i] = old
        g[i] = (lp - lm) / (2 * eps)
    return g


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _gdn_case(T=6, H=2, dk=3, dv=4, seed=0, beta_zero=False):
    rng = np.random.default_rng(seed)
    c = dict(q=rng.normal(size=(T, H, dk)), k=rng.normal(size=(T, H, dk)) * 0.6, v=rng.normal(size=(T, H, dv)),
             beta=np.zeros((T, H)) if beta_zero else rng.uniform(0.1, 0.9, size=(T, H)),
             log_alpha=rng.uniform(-1.0, -0.05, size=(T, H)), h0=rng.normal(size=(H, dv, dk)))
    adj = dict(do=rng.normal(size=(T, H, dv)), dh=rng.normal(size=(H, dv, dk)))
    return c, adj


@pytest.mark.parametrize("rule", ["gated_delta", "gated_linear"])
@pytest.mark.parametrize("scale", [1.0, 0.7])
def test_gdn_recurrence_bwd_matches_finite_differences(scale, rule):
    c, adj = _gdn_case()

    def loss():
        o, S = fwd.gdn_recurrence(c["q"], c["k"], c["v"], c["beta"], c["log_alpha"], c["h0"], scale, rule)
        return float(np.sum(adj["do"] * o) + np.sum(adj["dh"] * S))

    g = bwd.gdn_recurrence_bwd(c["q"], c["k"], c["v"], c["beta"], c["log_alpha"], adj["do"], c["h0"], adj["dh"],
                               scale, rule)
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta"), ("log_alpha", "dlog_alpha"),
                      ("h0", "dh0")):
        e = _rel(g[key], _fd(loss, c[name]))
        assert e < 1e-7, (name, e)


def test_gdn_recurrence_bwd_pure_decay_closed_form():
    # beta = 0: S_t = (prod_{i<=t} alpha_i) h0, o_t = S_t (scale q_t), so
    # dh0 = sum_t (prod_{i<=t} alpha_i) scale do_t q_t^T (+ the final adjoint
    # times the whole product), dq_t = scale S_t^T do_t, dv = dk = 0
    c, adj = _gdn_case(beta_zero=True, seed=3)
    scale = 0.5
    g = bwd.gdn_recurrence_bwd(c["q"], c["k"], c["v"], c["beta"], c["log_alpha"], adj["do"], c["h0"], adj["dh"],
                               scale)
    decay = np.exp(np.cumsum(c["log_alpha"], axis=0))          # [T,H]
    dh0 = np.einsum("th,thv,thk->hvk", decay, adj["do"], scale * c["q"]) + decay[-1][:, None, None] * adj["dh"]
    assert _rel(g["dh0"], dh0) < 1e-12
    St = decay[:, :, None, None] * c["h0"][None]
    assert _rel(g["dq"], scale * np.einsum("thvk,thv->thk", St, adj["do"])) < 1e-12
    assert np.all(g["dv"] == 0) and np.all(g["dk"] == 0)


@pytest.mark.parametrize("chunk", [1, 3, 4, 64])
@pytest.mark.parametrize("with_states", [True, False])
def test_gdn_chunked_bwd_equals_token_loop(chunk, with_states):
    # T = 11 leaves a ragged last chunk for every chunk size above 1
    c, adj = _gdn_case(T=11, seed=5)
    h0, dh = (c["h0"], adj["dh"]) if with_states else (None, None)
    ref = bwd.gdn_recurrence_bwd(c["q"], c["k"], c["v"], c["beta"], c["log_alpha"], adj["do"], h0, dh, 0.7)
    got = bwd.gdn_chunked_bwd(c["q"], c["k"], c["v"], c["beta"], c["log_alpha"], adj["do"], h0, dh, 0.7,
                              chunk=chunk)
    for key in ref:
        assert _rel(got[key], ref[key]) < 1e-12, (key, chunk)


def _layer_case(lens=(4, 0, 3), D=5, H=2, d=3, M=3, k=2, seed=1, mem_gates=False):
    w = synth.Workload("bwd_tiny", 0, 0, D, H, d, M, k, "f32", seed=seed, mem_gates=mem_gates)
    rng = np.random.default_rng(seed)
    p = {key: np.array(val, np.float64) for key, val in synth.make_weights(w, rng).items()}
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x = np.array(synth.make_tokens(w, rng, int(cu[-1])), np.float64)
    S = len(lens)
    N = int(cu[-1])
    adj = dict(dout=rng.normal(size=(N, H, d)), dhs=rng.normal(size=(S, H, d, d)),
               dhm=rng.normal(size=(M, S, H, d, d)))
    h0s = rng.normal(size=(S, H, d, d)) * 0.3
    h0m = rng.normal(size=(M, S, H, d, d)) * 0.3
    return w, p, cu, x, adj, h0s, h0m


@pytest.mark.parametrize("rule", ["gated_delta", "gated_linear"])
def test_mom_backward_matches_finite_differences(rule):
    w, p, cu, x, adj, h0s, h0m = _layer_case()
    H, d, K = w.heads, w.d_head, w.top_k
    idx = fwd.router_topk(x, p["w_r"], p["b_r"], K)[0]       # routing held fixed
    scale = 0.8

    def loss():
        f = fwd.mom_forward(x, p, cu, K, H, d, scale, forced_idx=idx, h0_shared=h0s, h0_mem=h0m, rule=rule)
        return float(np.sum(adj["dout"] * f["out"]) + np.sum(adj["dhs"] * f["h_shared"])
                     + np.sum(adj["dhm"] * f["h_mem"]))

    g = bwd.mom_backward(x, p, cu, K, H, d, adj["dout"], scale, forced_idx=idx, h0_shared=h0s, h0_mem=h0m,
                         dh_shared=adj["dhs"], dh_mem=adj["dhm"], rule=rule)
    checks = [("dx", x)] + [("d" + name, p[name]) for name in
                            ("w_r", "b_r", "w_q", "w_k_sh", "w_v_sh", "w_beta", "w_a", "A", "b_a", "w_k", "w_v")]
    checks += [("dh0_shared", h0s), ("dh0_mem", h0m)]
    for key, arr in checks:
        e = _rel(g[key], _fd(loss, arr))
        assert e < 1e-6, (key, e)


def test_mom_backward_with_per_memory_gates_matches_finite_differences():
    """Per-memory gates ("MoM", Summary: each memory its own parameters; the
    gates' placement is a reading): every gradient, the memories' own gate
    weights included, against central differences of the forward."""
    w, p, cu, x, adj, h0s, h0m = _layer_case(seed=4, mem_gates=True)
    H, d, K = w.heads, w.d_head, w.top_k
    idx = fwd.router_topk(x, p["w_r"], p["b_r"], K)[0]

    def loss():
        f = fwd.mom_forward(x, p, cu, K, H, d, 1.0, forced_idx=idx, h0_shared=h0s, h0_mem=h0m)
        return float(np.sum(adj["dout"] * f["out"]) + np.sum(adj["dhs"] * f["h_shared"])
                     + np.sum(adj["dhm"] * f["h_mem"]))

    g = bwd.mom_backward(x, p, cu, K, H, d, adj["dout"], 1.0, forced_idx=idx, h0_shared=h0s, h0_mem=h0m,
                         dh_shared=adj["dhs"], dh_mem=adj["dhm"])
    checks = [("dx", x)] + [("d" + name, p[name]) for name in
                            ("w_beta", "w_a", "A", "b_a", "w_k", "w_v", "w_q", "w_beta_mem", "w_a_mem", "A_mem",
                             "b_a_mem")]
    for key, arr in checks:
        e = _rel(g[key], _fd(loss, arr))
        assert e < 1e-6, (key, e)


def test_mom_backward_gate_gradient_sums_to_zero_over_chosen_logits():
    # the renormalised gates sum to 1 whatever the logits, so a common shift of
    # the chosen logits changes nothing: their gradients sum to zero per token
    w, p, cu, x, adj, _, _ = _layer_case(lens=(6,), seed=4)
    f = fwd.mom_forward(x, p, cu, w.top_k, w.heads, w.d_head)
    dgate = np.einsum("nhd,njhd->nj", adj["dout"], f["o_mem"])
    dl = bwd.router_gates_bwd(f["logits"], f["idx"], dgate)
    assert np.max(np.abs(dl.sum(axis=1))) < 1e-12
    chosen = np.zeros_like(dl, dtype=bool)
    np.put_along_axis(chosen, f["idx"].astype(np.int64), True, axis=1)
    assert np.all(dl[~chosen] == 0)


def test_l2norm_bwd_matches_finite_differences():
    rng = np.random.default_rng(7)
    z = rng.normal(size=(4, 2, 5))
    dy = rng.normal(size=(4, 2, 5))

    def loss():
        return float(np.sum(dy * fwd.l2norm(z)))

    assert _rel(bwd.l2norm_bwd(z, dy), _fd(loss, z)) < 1e-8


def test_gdn_recurrence_bwd_rules_differ_and_linear_rule_planted_mistake_fails():
    """The two rules' gradients differ (the delta terms matter), and a
    planted mistake in the linear rule's adjoint -- the delta term left in --
    fails its finite differences."""
    c, adj = _gdn_case(seed=3)
    args = (c["q"], c["k"], c["v"], c["beta"], c["log_alpha"], adj["do"], c["h0"], adj["dh"], 1.0)
    gd = bwd.gdn_recurrence_bwd(*args, "gated_delta")
    gl = bwd.gdn_recurrence_bwd(*args, "gated_linear")
    assert _rel(gd["dk"], gl["dk"]) > 1e-2 and _rel(gd["dh0"], gl["dh0"]) > 1e-2

    def loss():
        o, S = fwd.gdn_recurrence(c["q"], c["k"], c["v"], c["beta"], c["log_alpha"], c["h0"], 1.0, "gated_linear")
        return float(np.sum(adj["do"] * o) + np.sum(adj["dh"] * S))

    # the delta rule's adjoints are the linear rule's with the delta terms kept: they must fail here
    assert _rel(gd["dk"], _fd(loss, c["k"])) > 1e-3


def test_per_memory_gate_pin_catches_the_shared_gates_mistake():
    """The pin above fails a backward that runs the routed rows' reverse pass
    on the shared gates (the per-memory gates dropped): planted by handing
    the backward the weights without the memories' own gates."""
    w, p, cu, x, adj, h0s, h0m = _layer_case(seed=4, mem_gates=True)
    H, d, K = w.heads, w.d_head, w.top_k
    idx = fwd.router_topk(x, p["w_r"], p["b_r"], K)[0]

    def loss():
        f = fwd.mom_forward(x, p, cu, K, H, d, 1.0, forced_idx=idx, h0_shared=h0s, h0_mem=h0m)
        return float(np.sum(adj["dout"] * f["out"]) + np.sum(adj["dhs"] * f["h_shared"])
                     + np.sum(adj["dhm"] * f["h_mem"]))

    p_wrong = {k: v for k, v in p.items() if not k.endswith("_mem")}
    g = bwd.mom_backward(x, p_wrong, cu, K, H, d, adj["dout"], 1.0, forced_idx=idx, h0_shared=h0s, h0_mem=h0m,
                         dh_shared=adj["dhs"], dh_mem=adj["dhm"])
    assert _rel(g["dx"], _fd(loss, x)) > 1e-3
    assert _rel(g["dw_k"], _fd(loss, p["w_k"])) > 1e-3
