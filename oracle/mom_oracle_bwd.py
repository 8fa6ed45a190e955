"""CPU oracle for the reverse pass of one Mixture-of-Memories (MoM) layer:
plain, slow, fp64.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  The same rules as
``mom_oracle``: only the test suite may import it; it shares no code with the
CUDA path.

What it computes.  For the forward of ``mom_oracle.mom_forward`` (the Gated
DeltaNet rule per memory, "MoM: Linear Sequence Modeling with
Mixture-of-Memories", Summary; the authors' blog post, "Mixture-of-Memories"
and the experiments section naming Gated DeltaNet's gate and update rule) and
a scalar loss

    L = <dout, out> + sum_s <dh_shared[s], h_shared[s]>
                    + sum_{m,s} <dh_mem[m,s], h_mem[m,s]>,

the gradients of L with respect to the tokens x, every weight (router W_r,
b_r; shared W_q, W_k_sh, W_v_sh, W_beta, W_a, A, b_a; per-memory W_k, W_v)
and the initial states.  Each forward step is undone in reverse order by its
adjoint, written out by hand below; no automatic differentiation.

Routing.  Which memories a token visits (the top-k of the logits) is
piecewise constant in the inputs, so no gradient flows through the choice;
gradients do flow through the renormalised gates g_j = exp(l_j) / sum_j'
exp(l_j') over the chosen logits ("MoM: Mixture-of-Memories Fixes Linear
Attention Recall", Router mechanics: softmax, top-k, renormalisation).

Pinned by central finite differences of the forward oracle in fp64
(tests/test_oracle_backward.py): every gradient of the recurrence and of the
whole layer, on tiny inputs.
"""
from __future__ import annotations

import numpy as np

from oracle import mom_oracle as fwd

F64 = np.float64


def l2norm_bwd(z, dy, eps: float = fwd.NORM_EPS):
    """Adjoint of y = z / n, n = sqrt(|z|^2 + eps) over the last axis:
    dz = dy / n - z (z . dy) / n^3."""
    z = np.asarray(z, F64)
    dy = np.asarray(dy, F64)
    n = np.sqrt(np.sum(z * z, axis=-1, keepdims=True) + eps)
    return dy / n - z * np.sum(z * dy, axis=-1, keepdims=True) / n ** 3


def gdn_recurrence_bwd(q, k, v, beta, log_alpha, do, h0=None, dh_final=None, scale: float = 1.0,
                       rule: str = "gated_delta"):
    """Reverse pass of ``mom_oracle.gdn_recurrence`` over one segment.

    Shapes as the forward: q,k [T,H,dk]; v, do [T,H,dv]; beta, log_alpha
    [T,H]; h0, dh_final [H,dv,dk] or None.  Returns a dict with dq, dk, dv,
    dbeta, dlog_alpha (the forward's shapes) and dh0 [H,dv,dk].

    With a = exp(log alpha_t), b = beta_t, y = S_{t-1} k_t, c = 1 for the
    Gated DeltaNet rule and 0 for the scalar-gated linear one, and
    S_t = a S_{t-1} - c a b y k^T + b v k^T,  o_t = S_t (scale q_t),
    and G the adjoint of S_t (do_t (scale q_t)^T plus what flows back from
    step t+1):
      dq_t = scale S_t^T do_t
      dv_t = b G k
      db_t = (v - c a y)^T G k
      da_t = <G, S_{t-1}> - c b y^T G k,       dlog_alpha_t = a da_t
      dk_t = b G^T v - c a b (S_{t-1}^T G k + G^T y)
      adjoint of S_{t-1} = a G - c a b (G k) k^T
    """
    if rule not in fwd.RULES:
        raise ValueError("rule must be one of %s" % sorted(fwd.RULES))
    c = 1.0 if rule == "gated_delta" else 0.0
    q = np.asarray(q, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    beta = np.asarray(beta, F64)
    log_alpha = np.asarray(log_alpha, F64)
    do = np.asarray(do, F64)
    T, H, dk = k.shape
    dv = v.shape[-1]
    # forward, keeping every state (S[t] = state after token t-1; S[0] = h0)
    S = np.zeros((T + 1, H, dv, dk), F64)
    if h0 is not None:
        S[0] = np.asarray(h0, F64)
    step = fwd.RULES[rule]
    for t in range(T):
        _, S[t + 1] = step(S[t], q[t], k[t], v[t], beta[t], log_alpha[t], scale)
    G = np.zeros((H, dv, dk), F64) if dh_final is None else np.array(dh_final, F64, copy=True)
    out = {name: np.zeros_like(a) for name, a in
           (("dq", q), ("dk", k), ("dv", v), ("dbeta", beta), ("dlog_alpha", log_alpha))}
    for t in range(T - 1, -1, -1):
        sq = scale * q[t]
        G = G + do[t][:, :, None] * sq[:, None, :]
        out["dq"][t] = scale * np.einsum("hvk,hv->hk", S[t + 1], do[t])
        a = np.exp(log_alpha[t])
        b = beta[t]
        kt, vt, Sp = k[t], v[t], S[t]
        y = np.einsum("hvk,hk->hv", Sp, kt)
        Gk = np.einsum("hvk,hk->hv", G, kt)
        out["dv"][t] = b[:, None] * Gk
        out["dbeta"][t] = np.einsum("hv,hv->h", vt - c * a[:, None] * y, Gk)
        da = np.einsum("hvk,hvk->h", G, Sp) - c * b * np.einsum("hv,hv->h", y, Gk)
        out["dlog_alpha"][t] = a * da
        GTv = np.einsum("hvk,hv->hk", G, vt)
        SGk = np.einsum("hvk,hv->hk", Sp, Gk)
        GTy = np.einsum("hvk,hv->hk", G, y)
        out["dk"][t] = b[:, None] * GTv - c * (a * b)[:, None] * (SGk + GTy)
        G = a[:, None, None] * G - c * (a * b)[:, None, None] * Gk[:, :, None] * kt[:, None, :]
    out["dh0"] = G
    return out


def gdn_chunked_bwd(q, k, v, beta, log_alpha, do, h0=None, dh_final=None, scale: float = 1.0,
                    chunk: int = 64):
    """The reverse pass in the chunked (UT / WY) form of
    ``mom_oracle.gdn_chunked``: a self-check of ``gdn_recurrence_bwd`` (the
    two must agree to rounding), not a separate definition.

    Per chunk, with H the state at its start, gamma the running sum of
    log alpha from the chunk start, D_rs = exp(gamma_r - gamma_s) (s <= r),
    Qs = scale Q, the forward is
      L = strict_lower(diag(beta) D o K K^T),  T = (I + L)^-1
      R = diag(beta) V - diag(beta e^gamma) K H^T,   U = T R
      O = diag(e^gamma) Qs H^T + (Qs K^T o D) U
      H' = e^gamma_C H + U^T diag(e^(gamma_C - gamma)) K
    and the adjoints are taken in the reverse order of those lines (dH' is the
    state adjoint carried back from the next chunk); the adjoint of gamma is
    turned into that of log alpha by a reversed running sum.
    """
    q = np.asarray(q, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    beta = np.asarray(beta, F64)
    log_alpha = np.asarray(log_alpha, F64)
    do = np.asarray(do, F64)
    T, Hn, dk = k.shape
    dv = v.shape[-1]
    out = {name: np.zeros_like(a) for name, a in
           (("dq", q), ("dk", k), ("dv", v), ("dbeta", beta), ("dlog_alpha", log_alpha))}
    out["dh0"] = np.zeros((Hn, dv, dk), F64)
    starts = list(range(0, T, chunk))
    for h in range(Hn):
        # forward: the state at every chunk start
        Hs = [np.zeros((dv, dk), F64) if h0 is None else np.array(h0[h], F64, copy=True)]
        parts = []
        for c0 in starts:
            c1 = min(c0 + chunk, T)
            n = c1 - c0
            Qs, K, V = scale * q[c0:c1, h], k[c0:c1, h], v[c0:c1, h]
            b = beta[c0:c1, h]
            g = np.cumsum(log_alpha[c0:c1, h])
            causal = np.tril(np.ones((n, n), dtype=bool))
            D = np.where(causal, np.exp(np.where(causal, g[:, None] - g[None, :], 0.0)), 0.0)
            strict = np.tril(np.ones((n, n), dtype=bool), -1)
            L = np.where(strict, b[:, None] * D * (K @ K.T), 0.0)
            Tm = np.linalg.inv(np.eye(n) + L)
            Kt = (b * np.exp(g))[:, None] * K
            R = b[:, None] * V - Kt @ Hs[-1].T
            U = Tm @ R
            E = np.exp(g[-1] - g)
            parts.append((c0, c1, Qs, K, V, b, g, D, causal, strict, L, Tm, Kt, R, U, E))
            Hs.append(np.exp(g[-1]) * Hs[-1] + U.T @ (E[:, None] * K))
        # reverse
        dH = np.zeros((dv, dk), F64) if dh_final is None else np.array(dh_final[h], F64, copy=True)
        for ci in range(len(starts) - 1, -1, -1):
            c0, c1, Qs, K, V, b, g, D, causal, strict, L, Tm, Kt, R, U, E = parts[ci]
            Hc = Hs[ci]
            dO = do[c0:c1, h]
            eg = np.exp(g)
            dg = np.zeros_like(g)
            # H' = e^gC H + U^T diag(E) K
            dHp = dH
            dH = np.exp(g[-1]) * dHp
            dg[-1] += np.exp(g[-1]) * np.sum(dHp * Hc)
            dU = E[:, None] * (K @ dHp.T)
            dK = E[:, None] * (U @ dHp)
            w_s = E * np.einsum("sv,vk,sk->s", U, dHp, K)      # d/dgamma of each E_s term
            dg[-1] += w_s.sum()
            dg -= w_s
            # O = diag(e^g) Qs H^T + (Qs K^T o D) U
            A = (Qs @ K.T) * D
            dU += A.T @ dO
            dA = np.where(causal, dO @ U.T, 0.0)
            dAD = dA * D
            dQs = eg[:, None] * (dO @ Hc) + dAD @ K
            dK += dAD.T @ Qs
            dH += (eg[:, None] * dO).T @ Qs
            dg += eg * np.einsum("rv,rv->r", dO, Qs @ Hc.T)
            wa = dA * A                                          # d/dgamma_r (+) and d/dgamma_s (-) of D
            dg += wa.sum(axis=1) - wa.sum(axis=0)
            # U = T R,  R = diag(b) V - Kt H^T,  Kt = diag(b e^g) K
            dT = dU @ R.T
            dR = Tm.T @ dU
            dV = b[:, None] * dR
            db = np.einsum("rv,rv->r", V, dR)
            dKt = -dR @ Hc
            dH += -dR.T @ Kt
            dK += (b * eg)[:, None] * dKt
            kd = np.einsum("rk,rk->r", K, dKt)
            db += eg * kd
            dg += b * eg * kd
            # T = (I + L)^-1,  L = strict(diag(b) D o K K^T)
            dL = np.where(strict, -Tm.T @ dT @ Tm.T, 0.0)
            KK = K @ K.T
            db += np.sum(dL * D * KK, axis=1)
            P = dL * b[:, None] * D
            dK += P @ K + P.T @ K
            wl = dL * L
            dg += wl.sum(axis=1) - wl.sum(axis=0)
            out["dq"][c0:c1, h] = scale * dQs
            out["dk"][c0:c1, h] = dK
            out["dv"][c0:c1, h] = dV
            out["dbeta"][c0:c1, h] = db
            out["dlog_alpha"][c0:c1, h] = np.cumsum(dg[::-1])[::-1]
        out["dh0"][h] = dH
    return out


def router_gates_bwd(logits, idx, dgate):
    """Adjoint of the renormalised top-k gates g = softmax(logits[idx]) with
    respect to all M logits (zero for memories not chosen)."""
    logits = np.asarray(logits, F64)
    idx = np.asarray(idx, np.int64)
    g = fwd.gates_for(logits, idx)
    dsel = g * (dgate - np.sum(g * dgate, axis=-1, keepdims=True))
    dl = np.zeros_like(logits)
    np.put_along_axis(dl, idx, dsel, axis=-1)
    return dl


def mom_backward(x, p, cu_seqlens, top_k: int, H: int, d: int, dout, scale: float = 1.0,
                 forced_idx=None, h0_shared=None, h0_mem=None, dh_shared=None, dh_mem=None,
                 rule: str = "gated_delta"):
    """Gradients of L (module docstring) for one layer forward over a packed
    batch; arguments as ``mom_oracle.mom_forward`` plus the adjoints dout
    [N,H,d], dh_shared [S,H,d,d] and dh_mem [M,S,H,d,d] (None: zero).

    Returns a dict: dx, dw_r, db_r, dw_q, dw_k_sh, dw_v_sh, dw_beta, dw_a,
    dA, db_a, dw_k [M,..], dw_v [M,..], dh0_shared [S,..], dh0_mem [M,S,..],
    and the forward's own results under "fwd".  With per-memory gates
    (mom_oracle.memory_gates: each memory's routed rows take that memory's
    beta and alpha) also dw_beta_mem, dw_a_mem [M,H,d_model], dA_mem,
    db_a_mem [M,H]; the shared gates then carry the shared memory's
    adjoints alone.
    """
    x = np.asarray(x, F64)
    dout = np.asarray(dout, F64)
    cu = np.asarray(cu_seqlens, np.int64)
    N, D = x.shape
    S = len(cu) - 1
    M = np.shape(p["w_r"])[0]
    W = {name: np.asarray(p[name], F64) for name in
         ("w_r", "w_q", "w_k_sh", "w_v_sh", "w_beta", "w_a", "A", "b_a", "w_k", "w_v")}
    f = fwd.mom_forward(x, p, cu, top_k, H, d, scale, forced_idx=forced_idx,
                        h0_shared=h0_shared, h0_mem=h0_mem, rule=rule)
    idx, gate = f["idx"], f["gate"]
    mem_gates = fwd.has_memory_gates(p)
    if mem_gates:
        WM = {name: np.asarray(p[name], F64) for name in ("w_beta_mem", "w_a_mem", "A_mem", "b_a_mem")}
        gm = {"d" + name: np.zeros_like(arr) for name, arr in WM.items()}

    # combine: out = o_shared + sum_j gate_j o_mem[:, j]
    dgate = np.einsum("nhd,njhd->nj", dout, f["o_mem"])
    do_shared = dout

    # recurrences: adjoints of the per-token quantities they consume
    dq = np.zeros((N, H, d), F64)
    dk_sh = np.zeros((N, H, d), F64)
    dv_sh = np.zeros((N, H, d), F64)
    dbeta = np.zeros((N, H), F64)
    dlog_alpha = np.zeros((N, H), F64)
    dx = np.zeros_like(x)
    dw_k = np.zeros_like(W["w_k"])
    dw_v = np.zeros_like(W["w_v"])
    dh0_shared = np.zeros((S, H, d, d), F64)
    dh0_mem = np.zeros((M, S, H, d, d), F64)
    for s in range(S):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        h0 = None if h0_shared is None else h0_shared[s]
        dhf = None if dh_shared is None else dh_shared[s]
        if t1 > t0:
            r = gdn_recurrence_bwd(f["q"][t0:t1], f["k_sh"][t0:t1], f["v_sh"][t0:t1], f["beta"][t0:t1],
                                   f["log_alpha"][t0:t1], do_shared[t0:t1], h0, dhf, scale, rule)
            dq[t0:t1] += r["dq"]
            dk_sh[t0:t1] += r["dk"]
            dv_sh[t0:t1] += r["dv"]
            dbeta[t0:t1] += r["dbeta"]
            dlog_alpha[t0:t1] += r["dlog_alpha"]
            dh0_shared[s] = r["dh0"]
        else:
            dh0_shared[s] = 0.0 if dhf is None else dhf
        for m in range(M):
            hit = idx[t0:t1] == m
            rows = t0 + np.nonzero(hit.any(axis=1))[0]
            dhf = None if dh_mem is None else dh_mem[m, s]
            if len(rows) == 0:
                dh0_mem[m, s] = 0.0 if dhf is None else dhf
                continue
            slot = np.argmax(idx[rows] == m, axis=1)
            g = gate[rows, slot]
            z_k = (x[rows] @ W["w_k"][m].T).reshape(len(rows), H, d)
            k_m = fwd.l2norm(z_k)
            v_m = (x[rows] @ W["w_v"][m].T).reshape(len(rows), H, d)
            h0 = None if h0_mem is None else h0_mem[m, s]
            if mem_gates:
                b_m, la_m = fwd.memory_gates(x[rows], p, m)
            else:
                b_m, la_m = f["beta"][rows], f["log_alpha"][rows]
            r = gdn_recurrence_bwd(f["q"][rows], k_m, v_m, b_m, la_m, g[:, None, None] * dout[rows], h0, dhf,
                                   scale, rule)
            dq[rows] += r["dq"]
            if mem_gates:
                # memory m's own gates: beta = sigmoid(x W_beta^m^T), log alpha =
                # -exp(A^m) softplus(x W_a^m^T + b_a^m)
                dzb = r["dbeta"] * b_m * (1.0 - b_m)
                za = x[rows] @ WM["w_a_mem"][m].T + WM["b_a_mem"][m]
                dza = r["dlog_alpha"] * (-np.exp(WM["A_mem"][m])) * fwd.sigmoid(za)
                gm["dw_beta_mem"][m] += dzb.T @ x[rows]
                gm["dw_a_mem"][m] += dza.T @ x[rows]
                gm["dA_mem"][m] += np.sum(r["dlog_alpha"] * la_m, axis=0)
                gm["db_a_mem"][m] += dza.sum(axis=0)
                dx[rows] += dzb @ WM["w_beta_mem"][m] + dza @ WM["w_a_mem"][m]
            else:
                dbeta[rows] += r["dbeta"]
                dlog_alpha[rows] += r["dlog_alpha"]
            dh0_mem[m, s] = r["dh0"]
            # memory m's projections of its rows
            dz_k = l2norm_bwd(z_k, r["dk"]).reshape(len(rows), H * d)
            dz_v = r["dv"].reshape(len(rows), H * d)
            dw_k[m] += dz_k.T @ x[rows]
            dw_v[m] += dz_v.T @ x[rows]
            dx[rows] += dz_k @ W["w_k"][m] + dz_v @ W["w_v"][m]

    # router: logits = x W_r^T + b_r, gates renormalised over the chosen ones
    dl = router_gates_bwd(f["logits"], idx, dgate)
    dw_r = dl.T @ x
    db_r = dl.sum(axis=0)
    dx += dl @ W["w_r"]

    # shared projections
    z_q = (x @ W["w_q"].T).reshape(N, H, d)
    z_k = (x @ W["w_k_sh"].T).reshape(N, H, d)
    dz_q = l2norm_bwd(z_q, dq).reshape(N, H * d)
    dz_k = l2norm_bwd(z_k, dk_sh).reshape(N, H * d)
    dz_v = dv_sh.reshape(N, H * d)
    beta = f["beta"]
    dz_beta = dbeta * beta * (1.0 - beta)
    z_a = x @ W["w_a"].T + W["b_a"]
    # log alpha = -exp(A) softplus(z_a): d/dz_a = -exp(A) sigmoid(z_a); d/dA = log alpha
    dz_a = dlog_alpha * (-np.exp(W["A"])) * fwd.sigmoid(z_a)
    dA = np.sum(dlog_alpha * f["log_alpha"], axis=0)
    db_a = dz_a.sum(axis=0)
    dx += dz_q @ W["w_q"] + dz_k @ W["w_k_sh"] + dz_v @ W["w_v_sh"] + dz_beta @ W["w_beta"] + dz_a @ W["w_a"]
    out = dict(dx=dx, dw_r=dw_r, db_r=db_r, dw_q=dz_q.T @ x, dw_k_sh=dz_k.T @ x, dw_v_sh=dz_v.T @ x,
               dw_beta=dz_beta.T @ x, dw_a=dz_a.T @ x, dA=dA, db_a=db_a, dw_k=dw_k, dw_v=dw_v,
               dh0_shared=dh0_shared, dh0_mem=dh0_mem, fwd=f)
    if mem_gates:
        out.update(gm)
    return out
