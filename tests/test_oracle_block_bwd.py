"""Pins for the block's reverse pass (oracle/mom_block_bwd.py): central
finite differences of the block's forward (oracle/mom_block.py) in fp64 for
every gradient -- the tokens, every weight including the convolution
filters, the norm weight, the output gate and W_o, and the initial states --
on a tiny packed batch with an empty sequence, under both update rules;
the pieces (SiLU, the convolution, the gated RMS norm) on their own; and a
planted mistake (the convolution's adjoint run causally instead of
anti-causally) failing its pin.  Training is the pages' main workload
("MoM: Linear Sequence Modeling with Mixture-of-Memories", Key points); the
block's form is a reading (mom_block)."""
import numpy as np
import pytest

from mixture_memories_layer_b200 import synth
from oracle import mom_block as blk
from oracle import mom_block_bwd as bb
from oracle import mom_oracle as fwd

EPS = 1e-6


def _fd(loss, arr, eps=EPS):
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


def test_pieces_match_finite_differences():
    rng = np.random.default_rng(0)
    z = rng.normal(size=(9, 4)) * 2
    dy = rng.normal(size=(9, 4))
    assert _rel(bb.silu_bwd(z, dy), _fd(lambda: float(np.sum(dy * blk.silu(z))), z)) < 1e-8
    w = rng.uniform(-1, 1, size=(4, 3))
    bounds = [(0, 5), (5, 5), (5, 9)]
    dz, dw = bb.short_conv_bwd(z, w, bounds, dy)
    loss = lambda: float(np.sum(dy * blk.short_conv(z, w, bounds)))
    assert _rel(dz, _fd(loss, z)) < 1e-8 and _rel(dw, _fd(loss, w)) < 1e-8
    o = rng.normal(size=(5, 2, 4)) * np.array([0.05, 3.0])[None, :, None]
    g = rng.normal(size=(5, 2, 4))
    wn = rng.uniform(0.5, 1.5, size=4)
    dyo = rng.normal(size=(5, 2, 4))
    do, dwn, dg = bb.rms_norm_gated_bwd(o, wn, g, dyo)
    loss = lambda: float(np.sum(dyo * blk.rms_norm_gated(o, wn, g)))
    assert _rel(do, _fd(loss, o)) < 1e-7 and _rel(dwn, _fd(loss, wn)) < 1e-8 and _rel(dg, _fd(loss, g)) < 1e-8


def test_planted_mistake_in_the_convolution_adjoint_fails():
    rng = np.random.default_rng(1)
    z = rng.normal(size=(7, 3))
    w = rng.uniform(-1, 1, size=(3, 4))
    dc = rng.normal(size=(7, 3))

    def causal_adjoint(z, w, bounds, dc):          # the mistake: taps run forward in time
        W = w.shape[1]
        dz = np.zeros_like(z)
        for a, b in bounds:
            for t in range(a, b):
                for j in range(W):
                    if t + j < b:
                        dz[t + j] += w[:, W - 1 - j] * dc[t]
        return dz

    ref = _fd(lambda: float(np.sum(dc * blk.short_conv(z, w, [(0, 7)]))), z)
    assert _rel(bb.short_conv_bwd(z, w, [(0, 7)], dc)[0], ref) < 1e-8
    assert _rel(causal_adjoint(z, w, [(0, 7)], dc), ref) > 1e-2


def _case(lens=(4, 0, 3), D=5, H=2, d=3, M=3, k=2, seed=2, mem_gates=False):
    w = synth.Workload("bwd_tiny_block", 0, 0, D, H, d, M, k, "f32", seed=seed, block=True, mem_gates=mem_gates)
    rng = np.random.default_rng(seed)
    p = {key: np.array(val, np.float64) for key, val in synth.make_weights(w, rng).items()}
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x = np.array(synth.make_tokens(w, rng, int(cu[-1])), np.float64)
    S, N = len(lens), int(cu[-1])
    adj = dict(dy=rng.normal(size=(N, D)), dhs=rng.normal(size=(S, H, d, d)), dhm=rng.normal(size=(M, S, H, d, d)))
    h0s = rng.normal(size=(S, H, d, d)) * 0.3
    h0m = rng.normal(size=(M, S, H, d, d)) * 0.3
    return w, p, cu, x, adj, h0s, h0m


@pytest.mark.parametrize("rule", ["gated_delta", "gated_linear"])
def test_block_backward_matches_finite_differences(rule):
    w, p, cu, x, adj, h0s, h0m = _case(seed=2 if rule == "gated_delta" else 3)
    H, d, K = w.heads, w.d_head, w.top_k
    idx = fwd.router_topk(x, p["w_r"], p["b_r"], K)[0]
    scale = 0.8

    def loss():
        f = blk.block_forward(x, p, cu, K, H, d, scale, forced_idx=idx, h0_shared=h0s, h0_mem=h0m, rule=rule)
        return float(np.sum(adj["dy"] * f["y"]) + np.sum(adj["dhs"] * f["h_shared"]) + np.sum(adj["dhm"] * f["h_mem"]))

    g = bb.block_backward(x, p, cu, K, H, d, adj["dy"], scale, forced_idx=idx, h0_shared=h0s, h0_mem=h0m,
                          dh_shared=adj["dhs"], dh_mem=adj["dhm"], rule=rule)
    names = ("w_r", "b_r", "w_q", "w_k_sh", "w_v_sh", "w_g", "conv_q", "conv_k_sh", "conv_v_sh", "conv_k", "conv_v",
             "w_norm", "w_o", "w_beta", "w_a", "A", "b_a", "w_k", "w_v")
    checks = [("dx", x)] + [("d" + n, p[n]) for n in names] + [("dh0_shared", h0s), ("dh0_mem", h0m)]
    for key, arr in checks:
        e = _rel(g[key], _fd(loss, arr))
        assert e < 1e-6, (rule, key, e)


def test_block_backward_with_per_memory_gates_matches_finite_differences():
    """Per-memory gates inside the block: the memories' own gate weights and
    everything upstream of them against central differences."""
    w, p, cu, x, adj, h0s, h0m = _case(seed=6, mem_gates=True)
    H, d, K = w.heads, w.d_head, w.top_k
    idx = fwd.router_topk(x, p["w_r"], p["b_r"], K)[0]

    def loss():
        f = blk.block_forward(x, p, cu, K, H, d, 1.0, forced_idx=idx, h0_shared=h0s, h0_mem=h0m)
        return float(np.sum(adj["dy"] * f["y"]) + np.sum(adj["dhs"] * f["h_shared"]) + np.sum(adj["dhm"] * f["h_mem"]))

    g = bb.block_backward(x, p, cu, K, H, d, adj["dy"], 1.0, forced_idx=idx, h0_shared=h0s, h0_mem=h0m,
                          dh_shared=adj["dhs"], dh_mem=adj["dhm"])
    names = ("w_beta", "w_a", "A", "b_a", "w_k", "w_q", "conv_k", "w_beta_mem", "w_a_mem", "A_mem", "b_a_mem")
    for key, arr in [("dx", x)] + [("d" + n, p[n]) for n in names]:
        e = _rel(g[key], _fd(loss, arr))
        assert e < 1e-6, (key, e)
