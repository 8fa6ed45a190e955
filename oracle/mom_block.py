"""CPU oracle for the Gated DeltaNet block around the MoM memories: plain,
slow, fp64.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the test suite, the
smoke check in ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
reference leg of ``bench.py`` may import or call anything in this directory.
It shares no code with the CUDA path.

Sources: [blog] the authors' MoM blog post, experiments section ("實驗結果"):
every memory is a Gated DeltaNet token mixer (its gate and update rule);
[card] "MoM: Linear Sequence Modeling with Mixture-of-Memories", Summary
(shared q, per-memory key/value projections, router-weighted combine, an
always-on shared memory).  The pages print nothing of the block that wraps
the memories in a Gated DeltaNet layer.  The form taken here is the plain
Gated DeltaNet block, each choice a reading listed in the design notes:

* q, k and v (shared and per-memory) are projected without normalisation,
  pass through a causal depthwise convolution of width W (the conv weights'
  last axis; W = 4 in every workload) and then SiLU; q and k are then
  L2-normalised per head (x / sqrt(|x|^2 + 1e-6));
* the convolution runs along the rows its recurrence sees: the shared q, k,
  v along each sequence, memory m's k, v along the tokens of that sequence
  routed to m, in token order (a memory never sees the tokens it is not
  given); rows before a segment's start count as zero;
* a memory's own k and v have their own convolution weights, like their
  own projections;
* the combined output o (shared memory plus the router-weighted memories)
  is normalised per head by its root mean square (eps 1e-5) times a learned
  weight w_norm [d] shared by the heads, multiplied by SiLU of an output
  gate x W_g^T [Hd], and projected back by W_o [d_model, Hd].

The gates beta, log alpha, the router and the recurrences are those of
mom_oracle.  Parity pins: tests/test_oracle_block.py (numpy's convolution,
torch's RMS norm and SiLU, causality and segment locality of the
convolution, the routed-subsequence convolution, the reduction of the
block to mom_oracle.mom_forward when the convolution is the identity and
the activation is dropped, and the decode step continuing a prefill: the
forward over T tokens, its states and windows, then block_decode_step,
equals the forward over T + 1 tokens).
"""
from __future__ import annotations

import numpy as np

from . import mom_oracle as orc

F64 = np.float64
RMS_EPS = 1e-5


def silu(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, F64)
    return z * orc.sigmoid(z)


def identity(z: np.ndarray) -> np.ndarray:
    return np.asarray(z, F64)


def short_conv(z, w, bounds):
    """Causal depthwise convolution of the rows of z [n, C] inside each
    segment (a, b) of bounds: out[t] = sum_j w[:, W-1-j] * z[t-j] over the
    taps j = 0..W-1 with t-j >= a (tap W-1 is the current row).  Rows outside
    every segment stay zero.  w [C, W]."""
    z = np.asarray(z, F64)
    w = np.asarray(w, F64)
    W = w.shape[1]
    out = np.zeros_like(z)
    for a, b in bounds:
        for t in range(a, b):
            acc = np.zeros(z.shape[1], F64)
            for j in range(W):
                if t - j >= a:
                    acc += w[:, W - 1 - j] * z[t - j]
            out[t] = acc
    return out


def rms_norm_gated(o, w_norm, g, eps: float = RMS_EPS):
    """Per head: o / sqrt(mean(o^2) + eps) * w_norm * silu(g).  o, g [N, H, d];
    w_norm [d]."""
    o = np.asarray(o, F64)
    r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return o * r * np.asarray(w_norm, F64) * silu(g)


def _mixer_inputs(z_q, z_k, z_v, conv_q, conv_k, conv_v, bounds, H, d, act):
    """q (or None), k, v of one memory's rows from their raw projections."""
    n = z_k.shape[0]
    q = None
    if z_q is not None:
        q = orc.l2norm(act(short_conv(z_q, conv_q, bounds)).reshape(n, H, d))
    k = orc.l2norm(act(short_conv(z_k, conv_k, bounds)).reshape(n, H, d))
    v = act(short_conv(z_v, conv_v, bounds)).reshape(n, H, d)
    return q, k, v


def block_forward(x, p, cu_seqlens, top_k: int, H: int, d: int, scale: float = 1.0, forced_idx=None,
                  h0_shared=None, h0_mem=None, rule: str = "gated_delta", act=silu):
    """The block over a packed batch.  x [N, d_model]; p the layer weights
    plus w_g [Hd, d_model], w_o [d_model, Hd], conv_q, conv_k_sh, conv_v_sh
    [Hd, W], conv_k, conv_v [M, Hd, W], w_norm [d].  ``act`` is SiLU in the
    block; the identity is there for the reduction pin only.

    Returns a dict: y [N, d_model]; o_tilde [N, H, d] (normalised and gated,
    the input of W_o); out [N, H, d] (the combined memories); g [N, H, d]
    (the output gate's pre-activation); q, k_sh, v_sh [N, H, d]; k_mem, v_mem
    [N, k, H, d] (memory idx[t, j]'s key and value at t); o_shared, o_mem;
    idx, gate; h_shared [S, H, d, d]; h_mem [M, S, H, d, d]."""
    x = np.asarray(x, F64)
    cu = np.asarray(cu_seqlens, np.int64)
    N = x.shape[0]
    S = len(cu) - 1
    M = np.shape(p["w_r"])[0]
    lin = lambda a, w_: a @ np.asarray(w_, F64).T
    idx, gate, logits, near_tie = orc.router_topk(x, p["w_r"], p.get("b_r"), top_k)
    if forced_idx is not None:
        idx = np.asarray(forced_idx, np.int32)
        gate = orc.gates_for(logits, idx)
    # gates as in the layer (per token, or per memory)
    _, _, _, beta, log_alpha = orc.shared_projections(x, p, H, d)
    seqs = [(int(cu[s]), int(cu[s + 1])) for s in range(S)]
    q, k_sh, v_sh = _mixer_inputs(lin(x, p["w_q"]), lin(x, p["w_k_sh"]), lin(x, p["w_v_sh"]), p["conv_q"],
                                  p["conv_k_sh"], p["conv_v_sh"], seqs, H, d, act)
    o_shared = np.zeros((N, H, d), F64)
    o_mem = np.zeros((N, top_k, H, d), F64)
    k_mem = np.zeros((N, top_k, H, d), F64)
    v_mem = np.zeros((N, top_k, H, d), F64)
    h_shared = np.zeros((S, H, d, d), F64)
    h_mem = np.zeros((M, S, H, d, d), F64)
    for s, (t0, t1) in enumerate(seqs):
        h0 = None if h0_shared is None else h0_shared[s]
        o_shared[t0:t1], h_shared[s] = orc.gdn_recurrence(q[t0:t1], k_sh[t0:t1], v_sh[t0:t1], beta[t0:t1],
                                                          log_alpha[t0:t1], h0, scale, rule)
        for m in range(M):
            rows = t0 + np.nonzero((idx[t0:t1] == m).any(axis=1))[0]
            h0 = None if h0_mem is None else h0_mem[m, s]
            if len(rows) == 0:
                h_mem[m, s] = 0.0 if h0 is None else h0
                continue
            xr = x[rows]
            # memory m's rows of sequence s are one segment of its convolution
            _, k_m, v_m = _mixer_inputs(None, lin(xr, p["w_k"][m]), lin(xr, p["w_v"][m]), None, p["conv_k"][m],
                                        p["conv_v"][m], [(0, len(rows))], H, d, act)
            if orc.has_memory_gates(p):
                b_m, la_m = orc.memory_gates(xr, p, m)
            else:
                b_m, la_m = beta[rows], log_alpha[rows]
            o_m, h_mem[m, s] = orc.gdn_recurrence(q[rows], k_m, v_m, b_m, la_m, h0, scale, rule)
            slot = np.argmax(idx[rows] == m, axis=1)
            o_mem[rows, slot] = o_m
            k_mem[rows, slot] = k_m
            v_mem[rows, slot] = v_m
    out = o_shared + np.einsum("nj,njhd->nhd", gate, o_mem)
    g = lin(x, p["w_g"]).reshape(N, H, d)
    o_tilde = rms_norm_gated(out, p["w_norm"], g)
    y = lin(o_tilde.reshape(N, H * d), p["w_o"])
    return dict(y=y, o_tilde=o_tilde, out=out, g=g, q=q, k_sh=k_sh, v_sh=v_sh, k_mem=k_mem, v_mem=v_mem,
                o_shared=o_shared, o_mem=o_mem, idx=idx, gate=gate, logits=logits, near_tie=near_tie,
                h_shared=h_shared, h_mem=h_mem, beta=beta, log_alpha=log_alpha)


def conv_window_step(window, z, w, act):
    """One row of the causal convolution from the W-1 rows before it:
    window [W-1, C] (oldest first; zeros before the segment's start), z [C]
    the current row, w [C, W].  Returns (act(out) [C], the next window)."""
    rows = np.concatenate([np.asarray(window, F64), np.asarray(z, F64)[None]], axis=0)   # [W, C], oldest first
    out = np.einsum("wc,cw->c", rows, np.asarray(w, F64))
    return act(out), rows[1:]


def block_decode_step(x, p, state, conv_sh, conv_mem, top_k: int, H: int, d: int, scale: float = 1.0,
                      forced_idx=None, rule: str = "gated_delta", act=silu):
    """One new token per sequence through the block.  x [B, d_model]; state
    [B, M+1, H, d, d] (slot M = the shared memory), conv_sh [B, 3, W-1, Hd]
    (the raw q, k_sh, v_sh of the sequence's last W-1 tokens, oldest first,
    zero before its start) and conv_mem [B, M, 2, W-1, Hd] (the raw k, v of
    the last W-1 tokens routed to each memory); none is modified.  Each
    sequence updates only its k routed memories' states and windows and the
    shared ones.  Returns (y [B, d_model], new state, new conv_sh, new
    conv_mem, idx, parts) with parts = {"out": the combined output [B, H, d]
    before the gated norm, "g": the output gate's pre-activation}."""
    x = np.asarray(x, F64)
    Bn = x.shape[0]
    M = np.shape(p["w_r"])[0]
    lin = lambda a, w_: a @ np.asarray(w_, F64).T
    idx, gate, logits, _ = orc.router_topk(x, p["w_r"], p.get("b_r"), top_k)
    if forced_idx is not None:
        idx = np.asarray(forced_idx, np.int32)
        gate = orc.gates_for(logits, idx)
    _, _, _, beta, log_alpha = orc.shared_projections(x, p, H, d)
    raw_sh = [lin(x, p["w_q"]), lin(x, p["w_k_sh"]), lin(x, p["w_v_sh"])]
    filt_sh = [p["conv_q"], p["conv_k_sh"], p["conv_v_sh"]]
    g = lin(x, p["w_g"]).reshape(Bn, H, d)
    new = np.array(state, F64, copy=True)
    csh = np.array(conv_sh, F64, copy=True)
    cmem = np.array(conv_mem, F64, copy=True)
    out = np.zeros((Bn, H, d), F64)
    for b in range(Bn):
        qkv = []
        for i in range(3):
            c, csh[b, i] = conv_window_step(csh[b, i], raw_sh[i][b], filt_sh[i], act)
            qkv.append(c.reshape(H, d))
        q, k_sh, v_sh = orc.l2norm(qkv[0]), orc.l2norm(qkv[1]), qkv[2]
        out[b], new[b, M] = orc.RULES[rule](new[b, M], q, k_sh, v_sh, beta[b], log_alpha[b], scale)
        for j in range(top_k):
            m = int(idx[b, j])
            ck, cmem[b, m, 0] = conv_window_step(cmem[b, m, 0], lin(x[b], p["w_k"][m]), p["conv_k"][m], act)
            cv, cmem[b, m, 1] = conv_window_step(cmem[b, m, 1], lin(x[b], p["w_v"][m]), p["conv_v"][m], act)
            if orc.has_memory_gates(p):
                b_m, la_m = orc.memory_gates(x[b:b + 1], p, m)
                b_m, la_m = b_m[0], la_m[0]
            else:
                b_m, la_m = beta[b], log_alpha[b]
            o_m, new[b, m] = orc.RULES[rule](new[b, m], q, orc.l2norm(ck.reshape(H, d)), cv.reshape(H, d), b_m, la_m,
                                             scale)
            out[b] += gate[b, j] * o_m
    y = lin(rms_norm_gated(out, p["w_norm"], g).reshape(Bn, H * d), p["w_o"])
    return y, new, csh, cmem, idx, {"out": out, "g": g}


def block_conv_state(x, p, cu_seqlens, idx, W: int):
    """The convolution windows after a block forward over whole sequences:
    conv_sh [S, 3, W-1, Hd] (raw q, k_sh, v_sh of each sequence's last W-1
    tokens, oldest first, zero before its start) and conv_mem [S, M, 2, W-1,
    Hd] (raw k, v of the last W-1 tokens of each sequence routed to each
    memory).  idx [N, k] the routing the forward used."""
    x = np.asarray(x, F64)
    cu = np.asarray(cu_seqlens, np.int64)
    S = len(cu) - 1
    M = np.shape(p["w_r"])[0]
    Hd = np.shape(p["w_q"])[0]
    lin = lambda a, w_: a @ np.asarray(w_, F64).T
    csh = np.zeros((S, 3, W - 1, Hd), F64)
    cmem = np.zeros((S, M, 2, W - 1, Hd), F64)
    for s in range(S):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        last = np.arange(max(t0, t1 - (W - 1)), t1)
        for i, name in enumerate(("w_q", "w_k_sh", "w_v_sh")):
            if len(last):
                csh[s, i, W - 1 - len(last):] = lin(x[last], p[name])
        for m in range(M):
            rows = t0 + np.nonzero((idx[t0:t1] == m).any(axis=1))[0]
            rows = rows[max(0, len(rows) - (W - 1)):]
            if len(rows):
                cmem[s, m, 0, W - 1 - len(rows):] = lin(x[rows], p["w_k"][m])
                cmem[s, m, 1, W - 1 - len(rows):] = lin(x[rows], p["w_v"][m])
    return csh, cmem
