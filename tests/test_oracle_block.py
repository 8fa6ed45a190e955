"""Pins for the block oracle (oracle/mom_block.py), the Gated DeltaNet block
around the MoM memories (the authors' blog post, experiments section: each
memory is a Gated DeltaNet mixer; the block's form is a reading, the pages
print none of it).

* The short convolution against numpy's convolution, per channel and per
  segment (an independent library routine), including segments of length
  1 and 0; causality and segment locality by perturbation; a delta filter
  as a row shift.
* SiLU and the gated RMS norm against torch's silu and rms_norm.
* A memory's convolution runs over the tokens routed to it, in token order
  (forced routing, against numpy's convolution of that subsequence).
* With the identity convolution and no activation the block's memories are
  the plain layer's (mom_oracle.mom_forward) and y is W_o applied to the
  gated norm of its output (pure-Python dot products).
* Planted mistakes in the convolution (a flipped filter, a window crossing
  the segment start) and in the norm (the mean over all heads) fail their pins.
* Decode (constant-cost inference through the block): the one-row window
  step reproduces the convolution, and a decode step after a prefill equals
  the forward over one more token.
"""
import numpy as np
import pytest
import torch

from mixture_memories_layer_b200 import synth
from oracle import mom_block as blk
from oracle import mom_oracle as orc


def _conv_case(seed=0, C=6, W=4):
    rng = np.random.default_rng(seed)
    bounds = [(0, 7), (7, 8), (8, 8), (8, 19)]
    z = rng.standard_normal((19, C))
    w = rng.uniform(-1, 1, size=(C, W))
    return z, w, bounds


def _check_conv_vs_numpy(conv):
    z, w, bounds = _conv_case()
    out = conv(z, w, bounds)
    for a, b in bounds:
        for c in range(z.shape[1]):
            ref = np.convolve(z[a:b, c], w[c, ::-1])[: b - a] if b > a else np.zeros(0)
            np.testing.assert_allclose(out[a:b, c], ref, rtol=0, atol=1e-13)


def _check_conv_local(conv):
    z, w, bounds = _conv_case(seed=1)
    base = conv(z, w, bounds)
    W = w.shape[1]
    for a, b in bounds:
        for r in range(a, b):
            z2 = z.copy()
            z2[r] += 1.0
            diff = np.abs(conv(z2, w, bounds) - base).max(axis=1) > 0
            changed = set(np.nonzero(diff)[0].tolist())
            assert changed <= set(range(r, min(r + W, b))), (r, changed)
            assert r in changed


def test_short_conv_matches_numpy_convolve():
    _check_conv_vs_numpy(blk.short_conv)


def test_short_conv_is_causal_and_segment_local():
    _check_conv_local(blk.short_conv)


def test_short_conv_delta_filter_is_a_shift():
    z, _, bounds = _conv_case(seed=2)
    C, W = z.shape[1], 4
    for lag in range(W):
        w = np.zeros((C, W))
        w[:, W - 1 - lag] = 1.0
        out = blk.short_conv(z, w, bounds)
        for a, b in bounds:
            for t in range(a, b):
                np.testing.assert_array_equal(out[t], z[t - lag] if t - lag >= a else 0.0)


def test_silu_and_gated_rms_norm_match_torch():
    rng = np.random.default_rng(3)
    o = rng.standard_normal((5, 3, 8)) * np.array([1e-3, 1.0, 40.0])[None, :, None]
    g = rng.standard_normal((5, 3, 8)) * 3
    w = rng.uniform(0.5, 1.5, size=8)
    np.testing.assert_allclose(blk.silu(g), torch.nn.functional.silu(torch.from_numpy(g)).numpy(), rtol=1e-14)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(o), (8,), torch.from_numpy(w), eps=blk.RMS_EPS)
    ref = ref * torch.nn.functional.silu(torch.from_numpy(g))
    np.testing.assert_allclose(blk.rms_norm_gated(o, w, g), ref.numpy(), rtol=1e-12, atol=1e-15)


def _block_problem(seed=0, M=4, k=2, H=2, d=8, D=16, cu=(0, 9, 9, 21, 30)):
    w = synth.Workload("t", 1, 1, D, H, d, M, k, "f32", seed=seed, block=True)
    rng = np.random.default_rng(seed)
    p = synth.make_weights(w, rng)
    cu = np.asarray(cu, np.int32)
    x = synth.make_tokens(w, rng, int(cu[-1]))
    return w, p, x, cu


def test_memory_convolution_runs_over_its_routed_tokens():
    w, p, x, cu = _block_problem(seed=4, cu=(0, 12))
    N, M, H, d = 12, w.n_mem, w.heads, w.d_head
    # memory 0 sees tokens 0, 3, 7, 8; the other slot cycles through memories 1..3
    forced = np.zeros((N, 2), np.int32)
    mine = {0, 3, 7, 8}
    for t in range(N):
        forced[t] = (0, 1 + t % 3) if t in mine else (1 + t % 3, 1 + (t + 1) % 3)
    r = blk.block_forward(x, p, cu, 2, H, d, forced_idx=forced)
    rows = sorted(mine)
    zk = x[rows].astype(np.float64) @ p["w_k"][0].astype(np.float64).T
    zv = x[rows].astype(np.float64) @ p["w_v"][0].astype(np.float64).T
    ck = np.stack([np.convolve(zk[:, c], p["conv_k"][0][c, ::-1])[: len(rows)] for c in range(H * d)], axis=1)
    cv = np.stack([np.convolve(zv[:, c], p["conv_v"][0][c, ::-1])[: len(rows)] for c in range(H * d)], axis=1)
    silu = lambda a: a / (1.0 + np.exp(-a))
    k_ref = silu(ck).reshape(len(rows), H, d)
    k_ref = k_ref / np.sqrt((k_ref ** 2).sum(-1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(r["k_mem"][rows, 0], k_ref, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(r["v_mem"][rows, 0], silu(cv).reshape(len(rows), H, d), rtol=1e-12, atol=1e-14)


def test_identity_block_reduces_to_the_layer():
    w, p, x, cu = _block_problem(seed=5)
    for name in ("conv_q", "conv_k_sh", "conv_v_sh", "conv_k", "conv_v"):
        c = np.zeros_like(p[name])
        c[..., -1] = 1.0
        p[name] = c
    H, d = w.heads, w.d_head
    r = blk.block_forward(x, p, cu, w.top_k, H, d, act=blk.identity)
    ref = orc.mom_forward(x, p, cu, w.top_k, H, d)
    np.testing.assert_allclose(r["out"], ref["out"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["h_mem"], ref["h_mem"], rtol=0, atol=1e-12)
    # y = W_o o~ with o~ the gated norm of out, by hand for a few entries
    xs = x.astype(np.float64)
    for t in (0, 13, 29):
        o = ref["out"][t]
        for hh in range(H):
            ms = sum(float(v) * float(v) for v in o[hh]) / d
            for c in range(d):
                gl = sum(float(p["w_g"][hh * d + c, i]) * float(xs[t, i]) for i in range(w.d_model))
                want = o[hh, c] / np.sqrt(ms + 1e-5) * float(p["w_norm"][c]) * gl / (1.0 + np.exp(-gl))
                assert abs(r["o_tilde"][t, hh, c] - want) < 1e-12
        for i in (0, 7, 15):
            want = sum(float(p["w_o"][i, c]) * r["o_tilde"][t].reshape(-1)[c] for c in range(H * d))
            assert abs(r["y"][t, i] - want) < 1e-12


def test_planted_mistakes_fail_their_pins():
    def flipped(z, w, bounds):
        return blk.short_conv(z, np.asarray(w)[:, ::-1], bounds)

    def leaky(z, w, bounds):
        return blk.short_conv(z, w, [(0, bounds[-1][1])])

    with pytest.raises(AssertionError):
        _check_conv_vs_numpy(flipped)
    with pytest.raises(AssertionError):
        _check_conv_local(leaky)
    rng = np.random.default_rng(6)
    o = rng.standard_normal((4, 3, 8)) * np.array([0.1, 1.0, 10.0])[None, :, None]
    g = rng.standard_normal((4, 3, 8))
    w = np.ones(8)
    whole = o / np.sqrt(np.mean(o * o, axis=(-2, -1), keepdims=True) + blk.RMS_EPS) * blk.silu(g)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(o), (8,), torch.from_numpy(w), eps=blk.RMS_EPS)
    ref = (ref * torch.nn.functional.silu(torch.from_numpy(g))).numpy()
    assert np.abs(whole - ref).max() > 1e-3
    assert np.abs(blk.rms_norm_gated(o, w, g) - ref).max() < 1e-12


def test_block_decode_continues_a_prefill():
    """Constant-cost inference through the block: the forward over T tokens,
    its final states and convolution windows, then one decode step per
    sequence, equals the forward over T + 1 tokens (the last token's y, every
    final state) -- the decode's window arithmetic is written apart from the
    forward's convolution."""
    w, p, _, _ = _block_problem(seed=7, cu=(0, 2))
    rng = np.random.default_rng(70)
    lens = (9, 1, 6)
    H, d, K = w.heads, w.d_head, w.top_k
    xs = [synth.make_tokens(w, rng, n + 1) for n in lens]
    pre = [blk.block_forward(xi[:-1], p, np.array([0, len(xi) - 1]), K, H, d) for xi in xs]
    full = [blk.block_forward(xi, p, np.array([0, len(xi)]), K, H, d) for xi in xs]
    state = np.stack([orc.decode_state_from_prefill(r["h_shared"], r["h_mem"])[0] for r in pre])
    conv = [blk.block_conv_state(xi[:-1], p, np.array([0, len(xi) - 1]), r["idx"], 4) for xi, r in zip(xs, pre)]
    conv_sh = np.stack([c[0][0] for c in conv])
    conv_mem = np.stack([c[1][0] for c in conv])
    x_new = np.stack([xi[-1] for xi in xs])
    forced = np.stack([f["idx"][-1] for f in full])
    y, new, _, _, _, _ = blk.block_decode_step(x_new, p, state, conv_sh, conv_mem, K, H, d, forced_idx=forced)
    for b, f in enumerate(full):
        np.testing.assert_allclose(y[b], f["y"][-1], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(new[b, w.n_mem], f["h_shared"][0], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(new[b, :w.n_mem], f["h_mem"][:, 0], rtol=1e-10, atol=1e-12)


def test_conv_window_step_is_the_convolution():
    """The decode's one-row window step, run row by row from a zero window,
    reproduces the forward's convolution (numpy-pinned above)."""
    z, w, _ = _conv_case(seed=8)
    win = np.zeros((w.shape[1] - 1, z.shape[1]))
    ref = blk.short_conv(z, w, [(0, len(z))])
    for t in range(len(z)):
        out, win = blk.conv_window_step(win, z[t], w, blk.identity)
        np.testing.assert_allclose(out, ref[t], rtol=0, atol=1e-13)
