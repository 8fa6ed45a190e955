"""CPU oracle for the reverse pass of the Gated DeltaNet block around the
MoM memories (``mom_block.block_forward``): plain, slow, fp64.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  The same rules as the other
oracle modules: only the test suite may import it; it shares no code with
the CUDA path.

For the block's forward and the loss

    L = <dy, y> + sum_s <dh_shared[s], h_shared[s]> + sum_{m,s} <dh_mem[m,s], h_mem[m,s]>

the gradients with respect to the tokens x and every weight: the router,
the gates, the raw projections W_q, W_k_sh, W_v_sh, W_k^m, W_v^m, the
convolution filters, the output gate W_g, the norm weight and W_o, and the
initial states.  Each forward step is undone in reverse order by its
adjoint, written out by hand (no automatic differentiation); the
recurrences' reverse pass and the router's are those of mom_oracle_bwd.
Training is the pages' main workload ("MoM: Linear Sequence Modeling with
Mixture-of-Memories", Key points); the block's form is a reading (see
mom_block).  The routing is held fixed, as in the layer's backward.

Pinned by central finite differences of mom_block.block_forward
(tests/test_oracle_block_bwd.py).
"""
from __future__ import annotations

import numpy as np

from oracle import mom_block as blk
from oracle import mom_oracle as fwd
from oracle import mom_oracle_bwd as lbwd

F64 = np.float64


def silu_bwd(z, dy):
    """Adjoint of silu(z) = z sigmoid(z): dy sigmoid(z) (1 + z (1 - sigmoid(z)))."""
    z = np.asarray(z, F64)
    s = fwd.sigmoid(z)
    return np.asarray(dy, F64) * s * (1.0 + z * (1.0 - s))


def short_conv_bwd(z, w, bounds, dc):
    """Adjoint of c = blk.short_conv(z, w, bounds) for the output adjoint dc:
    dz[t] = sum_j w[:, W-1-j] dc[t+j] over the taps whose output row t+j is
    in t's segment, dw[:, W-1-j] = sum_t dc[t] z[t-j] over the rows with t-j
    in the segment.  Returns (dz, dw)."""
    z = np.asarray(z, F64)
    w = np.asarray(w, F64)
    dc = np.asarray(dc, F64)
    W = w.shape[1]
    dz = np.zeros_like(z)
    dw = np.zeros_like(w)
    for a, b in bounds:
        for t in range(a, b):
            for j in range(W):
                if t - j >= a:
                    dz[t - j] += w[:, W - 1 - j] * dc[t]
                    dw[:, W - 1 - j] += dc[t] * z[t - j]
    return dz, dw


def rms_norm_gated_bwd(o, w_norm, g, dy, eps: float = blk.RMS_EPS):
    """Adjoint of y = n w_norm silu(g), n = o / sqrt(mean(o^2) + eps) per
    head: do = r (dn - n mean(dn n)) with r the inverse RMS and dn = dy
    w_norm silu(g); dg = silu'(g) dy n w_norm; dw_norm = sum over tokens
    and heads of dy n silu(g).  o, g, dy [N, H, d]."""
    o = np.asarray(o, F64)
    dy = np.asarray(dy, F64)
    w = np.asarray(w_norm, F64)
    r = 1.0 / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    n = o * r
    s = blk.silu(g)
    dn = dy * w * s
    do = r * (dn - n * np.mean(dn * n, axis=-1, keepdims=True))
    dg = silu_bwd(g, dy * n * w)
    dw = np.sum(dy * n * s, axis=(0, 1))
    return do, dw, dg


def _mixer_bwd(x_rows, w_proj, w_conv, bounds, dy_out, H, d, l2):
    """The adjoint of one projected, convolved, activated (and normalised)
    input of a recurrence: out = [l2norm] silu(short_conv(x W^T)).  Returns
    (dx_rows, dW, dconv)."""
    n = x_rows.shape[0]
    z = x_rows @ np.asarray(w_proj, F64).T
    a = blk.short_conv(z, w_conv, bounds)
    c = blk.silu(a)
    dc = np.asarray(dy_out, F64).reshape(n, H * d)
    if l2:
        dc = lbwd.l2norm_bwd(c.reshape(n, H, d), dc.reshape(n, H, d)).reshape(n, H * d)
    da = silu_bwd(a, dc)
    dz, dconv = short_conv_bwd(z, w_conv, bounds, da)
    return dz @ np.asarray(w_proj, F64), dz.T @ x_rows, dconv


def block_backward(x, p, cu_seqlens, top_k: int, H: int, d: int, dy, scale: float = 1.0, forced_idx=None,
                   h0_shared=None, h0_mem=None, dh_shared=None, dh_mem=None, rule: str = "gated_delta"):
    """Gradients of L (module docstring) for one block forward over a packed
    batch; arguments as ``mom_block.block_forward`` plus the adjoints dy [N,
    d_model], dh_shared [S,H,d,d], dh_mem [M,S,H,d,d] (None: zero).

    Returns a dict: dx; dw_r, db_r; dw_q, dw_k_sh, dw_v_sh, dw_g; dconv_q,
    dconv_k_sh, dconv_v_sh [Hd, W], dconv_k, dconv_v [M, Hd, W]; dw_norm;
    dw_o; dw_beta, dw_a, dA, db_a; dw_k, dw_v [M, Hd, D]; dh0_shared,
    dh0_mem; and the forward's results under "fwd".  With per-memory gates
    (each memory's routed rows on its own beta and alpha, as in the forward)
    also dw_beta_mem, dw_a_mem [M, H, D], dA_mem, db_a_mem [M, H]."""
    mem_gates = fwd.has_memory_gates(p)
    x = np.asarray(x, F64)
    dy = np.asarray(dy, F64)
    cu = np.asarray(cu_seqlens, np.int64)
    N, D = x.shape
    S = len(cu) - 1
    M = np.shape(p["w_r"])[0]
    P = {k_: np.asarray(v_, F64) for k_, v_ in p.items() if k_ != "cu_seqlens" and k_ != "x"}
    f = blk.block_forward(x, p, cu, top_k, H, d, scale, forced_idx=forced_idx, h0_shared=h0_shared,
                          h0_mem=h0_mem, rule=rule)
    idx, gate = f["idx"], f["gate"]
    out = {}
    # y = o~ W_o^T
    dot = (dy @ P["w_o"]).reshape(N, H, d)
    out["dw_o"] = dy.T @ f["o_tilde"].reshape(N, H * d)
    # o~ = rmsnorm(o) w_norm silu(g), g = x W_g^T
    do, out["dw_norm"], dg = rms_norm_gated_bwd(f["out"], P["w_norm"], f["g"], dot)
    dg = dg.reshape(N, H * d)
    out["dw_g"] = dg.T @ x
    dx = dg @ P["w_g"]
    # combine: o = o_shared + sum_j gate_j o_mem[:, j]
    dgate = np.einsum("nhd,njhd->nj", do, f["o_mem"])
    dq = np.zeros((N, H, d), F64)
    dk_sh = np.zeros((N, H, d), F64)
    dv_sh = np.zeros((N, H, d), F64)
    dbeta = np.zeros((N, H), F64)
    dla = np.zeros((N, H), F64)
    dh0_shared = np.zeros((S, H, d, d), F64)
    dh0_mem = np.zeros((M, S, H, d, d), F64)
    for name in ("dw_k", "dw_v"):
        out[name] = np.zeros_like(P[name[1:]])
    out["dconv_k"] = np.zeros_like(P["conv_k"])
    out["dconv_v"] = np.zeros_like(P["conv_v"])
    if mem_gates:
        for name in ("w_beta_mem", "w_a_mem", "A_mem", "b_a_mem"):
            out["d" + name] = np.zeros_like(P[name])
    for s in range(S):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        dhf = None if dh_shared is None else dh_shared[s]
        if t1 > t0:
            h0 = None if h0_shared is None else h0_shared[s]
            r = lbwd.gdn_recurrence_bwd(f["q"][t0:t1], f["k_sh"][t0:t1], f["v_sh"][t0:t1], f["beta"][t0:t1],
                                        f["log_alpha"][t0:t1], do[t0:t1], h0, dhf, scale, rule)
            dq[t0:t1] += r["dq"]
            dk_sh[t0:t1] += r["dk"]
            dv_sh[t0:t1] += r["dv"]
            dbeta[t0:t1] += r["dbeta"]
            dla[t0:t1] += r["dlog_alpha"]
            dh0_shared[s] = r["dh0"]
        else:
            dh0_shared[s] = 0.0 if dhf is None else dhf
        for m in range(M):
            rows = t0 + np.nonzero((idx[t0:t1] == m).any(axis=1))[0]
            dhf = None if dh_mem is None else dh_mem[m, s]
            if len(rows) == 0:
                dh0_mem[m, s] = 0.0 if dhf is None else dhf
                continue
            slot = np.argmax(idx[rows] == m, axis=1)
            g_m = gate[rows, slot]
            k_m = f["k_mem"][rows, slot]
            v_m = f["v_mem"][rows, slot]
            h0 = None if h0_mem is None else h0_mem[m, s]
            if mem_gates:
                b_m, la_m = fwd.memory_gates(x[rows], p, m)
            else:
                b_m, la_m = f["beta"][rows], f["log_alpha"][rows]
            r = lbwd.gdn_recurrence_bwd(f["q"][rows], k_m, v_m, b_m, la_m, g_m[:, None, None] * do[rows], h0, dhf,
                                        scale, rule)
            dq[rows] += r["dq"]
            if mem_gates:
                # memory m's own gates (mom_oracle.memory_gates)
                dzb = r["dbeta"] * b_m * (1.0 - b_m)
                za = x[rows] @ P["w_a_mem"][m].T + P["b_a_mem"][m]
                dza = r["dlog_alpha"] * (-np.exp(P["A_mem"][m])) * fwd.sigmoid(za)
                out["dw_beta_mem"][m] += dzb.T @ x[rows]
                out["dw_a_mem"][m] += dza.T @ x[rows]
                out["dA_mem"][m] += np.sum(r["dlog_alpha"] * la_m, axis=0)
                out["db_a_mem"][m] += dza.sum(axis=0)
                dx[rows] += dzb @ P["w_beta_mem"][m] + dza @ P["w_a_mem"][m]
            else:
                dbeta[rows] += r["dbeta"]
                dla[rows] += r["dlog_alpha"]
            dh0_mem[m, s] = r["dh0"]
            seg = [(0, len(rows))]
            dxk, dwk, dck = _mixer_bwd(x[rows], P["w_k"][m], P["conv_k"][m], seg, r["dk"], H, d, True)
            dxv, dwv, dcv = _mixer_bwd(x[rows], P["w_v"][m], P["conv_v"][m], seg, r["dv"], H, d, False)
            dx[rows] += dxk + dxv
            out["dw_k"][m] += dwk
            out["dw_v"][m] += dwv
            out["dconv_k"][m] += dck
            out["dconv_v"][m] += dcv
    # the shared memory's q, k, v over whole sequences
    seqs = [(int(cu[s]), int(cu[s + 1])) for s in range(S)]
    for name, conv, dyo, l2 in (("q", "conv_q", dq, True), ("k_sh", "conv_k_sh", dk_sh, True),
                                ("v_sh", "conv_v_sh", dv_sh, False)):
        dxn, dwn, dcn = _mixer_bwd(x, P["w_" + name], P[conv], seqs, dyo, H, d, l2)
        dx += dxn
        out["dw_" + name] = dwn
        out["d" + conv] = dcn
    # gates and router, as in the layer
    beta = f["beta"]
    dz_beta = dbeta * beta * (1.0 - beta)
    z_a = x @ P["w_a"].T + P["b_a"]
    dz_a = dla * (-np.exp(P["A"])) * fwd.sigmoid(z_a)
    out["dA"] = np.sum(dla * f["log_alpha"], axis=0)
    out["db_a"] = dz_a.sum(axis=0)
    out["dw_beta"] = dz_beta.T @ x
    out["dw_a"] = dz_a.T @ x
    dx += dz_beta @ P["w_beta"] + dz_a @ P["w_a"]
    dl = lbwd.router_gates_bwd(f["logits"], idx, dgate)
    out["dw_r"] = dl.T @ x
    out["db_r"] = dl.sum(axis=0)
    dx += dl @ P["w_r"]
    out.update(dx=dx, dh0_shared=dh0_shared, dh0_mem=dh0_mem, fwd=f)
    return out
