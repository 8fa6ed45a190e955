"""CPU oracle for one Mixture-of-Memories (MoM) layer: plain, slow, fp64.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the test suite, the
smoke check in ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
reference leg of ``bench.py`` may import or call anything in this directory.
It shares no code with the CUDA path (no kernels, headers, helpers or
constants); the two meet only in the seeded input generator, which holds
none of the layer's arithmetic.

Sources (page title, then section):

* [blog]      the authors' blog post on MoM (jxzklqfsx.com, article 809919):
              "Linear Recurrent Memory", "Mixture-of-Memories",
              "硬件高效實現" (hardware-efficient implementation) and the
              experiments section ("實驗結果"), which names Gated DeltaNet's
              gate and update rule as the per-memory recurrence and the
              4-memories / 2-active / 1-shared configuration.
* [card]      "MoM: Linear Sequence Modeling with Mixture-of-Memories"
              (Elamur Research paper card), Summary: a linear router sends
              each token to its top-k memories; every memory has its own
              key/value projections and recurrent update; outputs are
              combined with the router weights; a shared memory is always on.
* [explainer] "MoM: Mixture-of-Memories Fixes Linear Attention Recall",
              "Router mechanics, step by step" (one matmul, one softmax, one
              top-k, one renormalisation) and "Solving scatter-gather without
              new kernels" (routing becomes a reordering of tokens into
              contiguous per-memory segments).
* [sdm]       "Sparse Delta Memory: Scaling the State of Linear RNNs through
              Sparsity", gated delta update (forget by alpha, then correct the
              memory toward v with strength beta) -- a cross-check of the
              update's form only.

The formulas on [blog] were lost from the page; the recurrence used here is
the Gated DeltaNet rule those pages name,

    S_t = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
    o_t = S_t (scale * q_t),

with S the d_v x d_k state, read after the write at token t.  A second rule
of the family [blog] "Linear Recurrent Memory" lists (linear attention,
RetNet, Mamba2-style memories: the scalar-gated linear form, without the
delta correction) is available wherever the rule can be chosen:

    S_t = alpha_t * S_{t-1} + beta_t v_t k_t^T,      o_t = S_t (scale * q_t).

Readings where the pages are silent (each also listed in the design notes):
q, beta and alpha are shared by all memories (one W_q, W_beta, W_a) unless
the layer has per-memory gates (then each routed memory has its own W_beta,
W_a, A, b_a: memory_gates); every memory, the shared one included, has its
own W_k, W_v; a memory's state is
neither decayed nor updated on tokens not routed to it; the shared memory
enters the combine with weight 1; top-k is taken on logits with ties going
to the lower memory index; q and k are L2-normalised per head as
x / sqrt(|x|^2 + 1e-6); log alpha = -exp(A) * softplus(x W_a + b_a);
beta = sigmoid(x W_beta); there is no capacity limit and no token dropping.

Parity pins: every function here is checked by tests against brute force,
closed forms or invariants (tests/test_oracle_*.py).  Absolute values of the
full layer rest on the definition above: the pages print no worked example.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular

F64 = np.float64
NORM_EPS = 1e-6
TIE_GAP = 1e-4


# ----------------------------------------------------------------------------
# elementwise pieces
# ----------------------------------------------------------------------------

def l2norm(y: np.ndarray, eps: float = NORM_EPS) -> np.ndarray:
    """x / sqrt(sum x^2 + eps) over the last axis (one head)."""
    y = np.asarray(y, F64)
    return y / np.sqrt(np.sum(y * y, axis=-1, keepdims=True) + eps)


def softmax(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, F64)
    e = np.exp(z - z.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def sigmoid(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-np.asarray(z, F64)))


def softplus(z: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, np.asarray(z, F64))


# ----------------------------------------------------------------------------
# router  ([explainer] "Router mechanics, step by step"; [blog] Mixture-of-Memories)
# ----------------------------------------------------------------------------

def router_topk(x, w_r, b_r, top_k: int, tie_gap: float = TIE_GAP):
    """One matmul, one softmax, one top-k, one renormalisation.

    Returns (idx [N,k] in rank order, gate [N,k], logits [N,M], near_tie [N]).
    Ranking uses the logits, ties to the lower memory index.  ``near_tie``
    marks tokens whose k-th and (k+1)-th logits differ by less than
    ``tie_gap``: their choice can flip under rounding, so tests exclude them
    from exact index comparison.
    """
    x = np.asarray(x, F64)
    logits = x @ np.asarray(w_r, F64).T
    if b_r is not None:
        logits = logits + np.asarray(b_r, F64)
    probs = softmax(logits)
    N, M = logits.shape
    mem_index = np.broadcast_to(np.arange(M), (N, M))
    # primary key: descending logit; secondary key: ascending memory index
    order = np.lexsort((mem_index, -logits), axis=-1)
    idx = order[:, :top_k]
    sel = np.take_along_axis(probs, idx, axis=-1)
    gate = sel / sel.sum(axis=-1, keepdims=True)
    if top_k < M:
        ranked = np.take_along_axis(logits, order, axis=-1)
        near_tie = (ranked[:, top_k - 1] - ranked[:, top_k]) < tie_gap
    else:
        near_tie = np.zeros(N, dtype=bool)
    return idx.astype(np.int32), gate, logits, near_tie


def gates_for(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """Renormalised softmax weights of a given selection (used when the
    routing decision is imposed from outside, e.g. to follow a near-tie
    choice taken elsewhere)."""
    probs = softmax(logits)
    sel = np.take_along_axis(probs, np.asarray(idx, np.int64), axis=-1)
    return sel / sel.sum(axis=-1, keepdims=True)


# ----------------------------------------------------------------------------
# reordering  ([explainer] "Solving scatter-gather without new kernels")
# ----------------------------------------------------------------------------

def permute(idx: np.ndarray, n_mem: int, cu_seqlens: np.ndarray):
    """Stable counting sort of the (token, slot) pairs by memory.

    Pair r = t*k + j routes token t to memory idx[t, j].  Returns
      perm_token [N*k]   token of each reordered row,
      row_of     [N*k]   reordered row of pair t*k+j,
      mem_offset [M+1]   first row of each memory,
      seg_cu     [M*S+1] segment bounds, one segment per (memory, sequence),
                         memory-major; rows inside a segment keep token order.
    """
    idx = np.asarray(idx)
    N, k = idx.shape
    pair_mem = idx.reshape(-1).astype(np.int64)
    order = np.argsort(pair_mem, kind="stable")
    perm_token = (order // k).astype(np.int32)
    row_of = np.empty(N * k, dtype=np.int32)
    row_of[order] = np.arange(N * k, dtype=np.int32)
    counts = np.bincount(pair_mem, minlength=n_mem)
    mem_offset = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    cu = np.asarray(cu_seqlens, np.int64)
    S = len(cu) - 1
    seg_cu = np.empty(n_mem * S + 1, dtype=np.int32)
    for m in range(n_mem):
        toks = perm_token[mem_offset[m]:mem_offset[m + 1]]
        for s in range(S):
            # rows of memory m whose token lies before sequence s starts
            seg_cu[m * S + s] = mem_offset[m] + np.searchsorted(toks, cu[s], side="left")
    seg_cu[n_mem * S] = N * k
    return perm_token, row_of, mem_offset, seg_cu


# ----------------------------------------------------------------------------
# projections  ([card] Summary: shared q, per-memory key/value projections)
# ----------------------------------------------------------------------------

def shared_projections(x, p, H: int, d: int):
    """q, k_sh, v_sh [N,H,d]; beta, log_alpha [N,H]."""
    x = np.asarray(x, F64)
    N = x.shape[0]
    q = l2norm((x @ np.asarray(p["w_q"], F64).T).reshape(N, H, d))
    k_sh = l2norm((x @ np.asarray(p["w_k_sh"], F64).T).reshape(N, H, d))
    v_sh = (x @ np.asarray(p["w_v_sh"], F64).T).reshape(N, H, d)
    beta = sigmoid(x @ np.asarray(p["w_beta"], F64).T)
    a_in = x @ np.asarray(p["w_a"], F64).T + np.asarray(p["b_a"], F64)
    log_alpha = -np.exp(np.asarray(p["A"], F64)) * softplus(a_in)
    return q, k_sh, v_sh, beta, log_alpha


def memory_kv(x_rows, p, m: int, H: int, d: int):
    """Memory m's own key/value projection of the rows routed to it."""
    x_rows = np.asarray(x_rows, F64)
    n = x_rows.shape[0]
    k = l2norm((x_rows @ np.asarray(p["w_k"][m], F64).T).reshape(n, H, d))
    v = (x_rows @ np.asarray(p["w_v"][m], F64).T).reshape(n, H, d)
    return k, v


def memory_gates(x_rows, p, m: int):
    """Memory m's own gates of the rows routed to it, when the layer has
    per-memory gates (p holds w_beta_mem, w_a_mem [M,H,d_model], A_mem,
    b_a_mem [M,H]): beta = sigmoid(x W_beta^m), log alpha = -exp(A^m)
    softplus(x W_a^m + b_a^m).  Without them every memory uses the shared
    gates of shared_projections."""
    x_rows = np.asarray(x_rows, F64)
    beta = sigmoid(x_rows @ np.asarray(p["w_beta_mem"][m], F64).T)
    a_in = x_rows @ np.asarray(p["w_a_mem"][m], F64).T + np.asarray(p["b_a_mem"][m], F64)
    log_alpha = -np.exp(np.asarray(p["A_mem"][m], F64)) * softplus(a_in)
    return beta, log_alpha


def has_memory_gates(p) -> bool:
    return "w_beta_mem" in p


# ----------------------------------------------------------------------------
# Gated DeltaNet recurrence  ([blog] experiments: "Gated DeltaNet gate and
# update rule" per memory; [sdm] gated delta update as a form check)
# ----------------------------------------------------------------------------

def gdn_step(S, q_t, k_t, v_t, beta_t, log_alpha_t, scale: float = 1.0):
    """One token for all heads.  S [H,dv,dk]; q_t,k_t [H,dk]; v_t [H,dv];
    beta_t, log_alpha_t [H].  Returns (o_t [H,dv], S_t).

    S_t = alpha S (I - beta k k^T) + beta v k^T, written with the product
    S (I - beta k k^T) = S - beta (S k) k^T distributed out; o_t = S_t (scale q).
    """
    a = np.exp(np.asarray(log_alpha_t, F64))[:, None, None]
    b = np.asarray(beta_t, F64)[:, None, None]
    k_t = np.asarray(k_t, F64)
    Sk = np.einsum("hvk,hk->hv", S, k_t)
    S = a * (S - b * Sk[:, :, None] * k_t[:, None, :]) + b * np.asarray(v_t, F64)[:, :, None] * k_t[:, None, :]
    o = np.einsum("hvk,hk->hv", S, scale * np.asarray(q_t, F64))
    return o, S


def gla_step(S, q_t, k_t, v_t, beta_t, log_alpha_t, scale: float = 1.0):
    """One token of the scalar-gated linear rule (the linear-attention form of
    the update-rule family in [blog] "Linear Recurrent Memory": linear
    attention with alpha = beta = 1, RetNet with a fixed alpha per head,
    Mamba2-style memories with a data-dependent scalar alpha):

        S_t = alpha_t S_{t-1} + beta_t v_t k_t^T,     o_t = S_t (scale q_t)

    Shapes as gdn_step.  Returns (o_t [H,dv], S_t)."""
    a = np.exp(np.asarray(log_alpha_t, F64))[:, None, None]
    b = np.asarray(beta_t, F64)[:, None, None]
    S = a * S + b * np.asarray(v_t, F64)[:, :, None] * np.asarray(k_t, F64)[:, None, :]
    o = np.einsum("hvk,hk->hv", S, scale * np.asarray(q_t, F64))
    return o, S


RULES = {"gated_delta": gdn_step, "gated_linear": gla_step}


def gdn_recurrence(q, k, v, beta, log_alpha, h0=None, scale: float = 1.0, rule: str = "gated_delta"):
    """Token-by-token recurrence over one segment.  q,k [T,H,dk]; v [T,H,dv];
    beta, log_alpha [T,H]; h0 [H,dv,dk] or None (zeros); rule one of RULES
    (default the Gated DeltaNet step).  Returns (o [T,H,dv], S_final [H,dv,dk])."""
    T, H, dk = np.shape(k)
    dv = np.shape(v)[-1]
    S = np.zeros((H, dv, dk), F64) if h0 is None else np.array(h0, F64, copy=True)
    o = np.zeros((T, H, dv), F64)
    for t in range(T):
        o[t], S = RULES[rule](S, q[t], k[t], v[t], beta[t], log_alpha[t], scale)
    return o, S


def gdn_chunked(q, k, v, beta, log_alpha, h0=None, scale: float = 1.0, chunk: int = 64):
    """The same recurrence in chunked (UT / WY) form; a self-check of the
    token loop, not a separate definition.

    Within a chunk, with gamma_r the running sum of log alpha from the chunk
    start and H the state at the chunk start:
      L_rs = beta_r exp(gamma_r - gamma_s) k_r.k_s  (s < r),  T = (I + L)^-1
      W = T diag(beta exp(gamma)) K,   U = T diag(beta) V - W H^T
      O = diag(exp(gamma)) Q H^T + (Q K^T o [exp(gamma_r - gamma_s)]_{s<=r}) U
      H' = exp(gamma_C) H + U^T diag(exp(gamma_C - gamma)) K
    U's rows are u_r = beta_r (v_r - alpha_r S_{r-1} k_r), so that
    S_r = alpha_r S_{r-1} + u_r k_r^T.
    """
    q = np.asarray(q, F64) * scale
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    beta = np.asarray(beta, F64)
    log_alpha = np.asarray(log_alpha, F64)
    T, H, dk = k.shape
    dv = v.shape[-1]
    o = np.zeros((T, H, dv), F64)
    S_out = np.zeros((H, dv, dk), F64)
    for h in range(H):
        Hs = np.zeros((dv, dk), F64) if h0 is None else np.array(h0[h], F64, copy=True)
        for c0 in range(0, T, chunk):
            c1 = min(c0 + chunk, T)
            n = c1 - c0
            Q, K, V = q[c0:c1, h], k[c0:c1, h], v[c0:c1, h]
            b = beta[c0:c1, h]
            g = np.cumsum(log_alpha[c0:c1, h])
            diff = g[:, None] - g[None, :]
            causal = np.tril(np.ones((n, n), dtype=bool))
            D = np.where(causal, np.exp(np.where(causal, diff, 0.0)), 0.0)
            strict = np.tril(np.ones((n, n), dtype=bool), -1)
            L = np.where(strict, b[:, None] * D * (K @ K.T), 0.0)
            Tm = solve_triangular(np.eye(n) + L, np.eye(n), lower=True, unit_diagonal=True)
            W = Tm @ ((b * np.exp(g))[:, None] * K)
            U = Tm @ (b[:, None] * V) - W @ Hs.T
            o[c0:c1, h] = np.exp(g)[:, None] * (Q @ Hs.T) + ((Q @ K.T) * D) @ U
            Hs = np.exp(g[-1]) * Hs + U.T @ (np.exp(g[-1] - g)[:, None] * K)
        S_out[h] = Hs
    return o, S_out


# ----------------------------------------------------------------------------
# the layer  ([card] Summary; [blog] Mixture-of-Memories and the
# hardware-efficient implementation's output-sum form)
# ----------------------------------------------------------------------------

def mom_forward(x, p, cu_seqlens, top_k: int, H: int, d: int, scale: float = 1.0,
                forced_idx=None, h0_shared=None, h0_mem=None, rule: str = "gated_delta"):
    """One MoM layer forward over a packed batch.

    x [N,d_model]; p the weights (see the input generator for names and
    [out,in] layouts); cu_seqlens [S+1].  States restart at every sequence
    boundary (from h0_shared [S,H,d,d] / h0_mem [M,S,H,d,d] when given).

    Returns a dict: out [N,H,d]; idx, gate [N,k]; logits; near_tie [N];
    o_shared [N,H,d]; o_mem [N,k,H,d] (memory idx[t,j]'s output at t);
    h_shared [S,H,d,d]; h_mem [M,S,H,d,d]; and the projections.
    """
    x = np.asarray(x, F64)
    cu = np.asarray(cu_seqlens, np.int64)
    N = x.shape[0]
    S = len(cu) - 1
    M = np.shape(p["w_r"])[0]
    idx, gate, logits, near_tie = router_topk(x, p["w_r"], p.get("b_r"), top_k)
    if forced_idx is not None:
        idx = np.asarray(forced_idx, np.int32)
        gate = gates_for(logits, idx)
    q, k_sh, v_sh, beta, log_alpha = shared_projections(x, p, H, d)

    o_shared = np.zeros((N, H, d), F64)
    o_mem = np.zeros((N, top_k, H, d), F64)
    h_shared = np.zeros((S, H, d, d), F64)
    h_mem = np.zeros((M, S, H, d, d), F64)
    for s in range(S):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        h0 = None if h0_shared is None else h0_shared[s]
        o_shared[t0:t1], h_shared[s] = gdn_recurrence(
            q[t0:t1], k_sh[t0:t1], v_sh[t0:t1], beta[t0:t1], log_alpha[t0:t1], h0, scale, rule)
        for m in range(M):
            # the tokens of sequence s routed to memory m, in token order
            hit = idx[t0:t1] == m
            rows = t0 + np.nonzero(hit.any(axis=1))[0]
            h0 = None if h0_mem is None else h0_mem[m, s]
            if len(rows) == 0:
                h_mem[m, s] = 0.0 if h0 is None else h0
                continue
            k_m, v_m = memory_kv(x[rows], p, m, H, d)
            b_m, la_m = memory_gates(x[rows], p, m) if has_memory_gates(p) else (beta[rows], log_alpha[rows])
            o_m, h_mem[m, s] = gdn_recurrence(q[rows], k_m, v_m, b_m, la_m, h0, scale, rule)
            slot = np.argmax(idx[rows] == m, axis=1)
            o_mem[rows, slot] = o_m
    # combine: shared memory with weight 1 plus the router-weighted memories
    out = o_shared + np.einsum("nj,njhd->nhd", gate, o_mem)
    return dict(out=out, idx=idx, gate=gate, logits=logits, near_tie=near_tie,
                o_shared=o_shared, o_mem=o_mem, h_shared=h_shared, h_mem=h_mem,
                q=q, k_sh=k_sh, v_sh=v_sh, beta=beta, log_alpha=log_alpha)


def mom_forward_mixed_state(x, p, cu_seqlens, top_k: int, H: int, d: int, scale: float = 1.0,
                            forced_idx=None, rule: str = "gated_delta"):
    """The layer in its "mix the memories first, then read out" form
    ([blog] Mixture-of-Memories: the active memories are summed with their
    router weights into one mixed memory, which is then read with q).

    out_t = (S^sh_t + sum_j g_{t,j} S^{idx[t,j]}_t) (scale q_t), all states
    after their update at t.  Token loop over every memory state at once;
    tiny inputs only.
    """
    x = np.asarray(x, F64)
    cu = np.asarray(cu_seqlens, np.int64)
    N = x.shape[0]
    M = np.shape(p["w_r"])[0]
    idx, gate, logits, _ = router_topk(x, p["w_r"], p.get("b_r"), top_k)
    if forced_idx is not None:
        idx = np.asarray(forced_idx, np.int32)
        gate = gates_for(logits, idx)
    q, k_sh, v_sh, beta, log_alpha = shared_projections(x, p, H, d)
    out = np.zeros((N, H, d), F64)
    for s in range(len(cu) - 1):
        states = np.zeros((M + 1, H, d, d), F64)      # slot M is the shared memory
        for t in range(int(cu[s]), int(cu[s + 1])):
            _, states[M] = RULES[rule](states[M], q[t], k_sh[t], v_sh[t], beta[t], log_alpha[t])
            for j in range(top_k):
                m = int(idx[t, j])
                k_m, v_m = memory_kv(x[t:t + 1], p, m, H, d)
                b_m, la_m = memory_gates(x[t:t + 1], p, m) if has_memory_gates(p) else (beta[t:t + 1], log_alpha[t:t + 1])
                _, states[m] = RULES[rule](states[m], q[t], k_m[0], v_m[0], b_m[0], la_m[0])
            mixed = states[M] + sum(gate[t, j] * states[int(idx[t, j])] for j in range(top_k))
            out[t] = np.einsum("hvk,hk->hv", mixed, scale * q[t])
    return out


# ----------------------------------------------------------------------------
# recurrent decode  ([blog] constant-cost inference; [card] Summary)
# ----------------------------------------------------------------------------

def decode_state_from_prefill(h_shared, h_mem):
    """[S,H,d,d] + [M,S,H,d,d] -> decode layout [S, M+1, H, d, d] (slot M = shared)."""
    h_shared = np.asarray(h_shared, F64)
    h_mem = np.asarray(h_mem, F64)
    M = h_mem.shape[0]
    st = np.zeros((h_shared.shape[0], M + 1) + h_shared.shape[1:], F64)
    st[:, :M] = np.transpose(h_mem, (1, 0, 2, 3, 4))
    st[:, M] = h_shared
    return st


def mom_decode_step(x, p, state, top_k: int, H: int, d: int, scale: float = 1.0, forced_idx=None,
                    rule: str = "gated_delta"):
    """One new token per sequence.  x [B,d_model]; state [B,M+1,H,d,d]
    (slot M = shared), not modified.  Each sequence updates only its k routed
    states and the shared one.  Returns (out [B,H,d], new_state, idx, gate,
    near_tie)."""
    x = np.asarray(x, F64)
    B = x.shape[0]
    M = np.shape(p["w_r"])[0]
    idx, gate, logits, near_tie = router_topk(x, p["w_r"], p.get("b_r"), top_k)
    if forced_idx is not None:
        idx = np.asarray(forced_idx, np.int32)
        gate = gates_for(logits, idx)
    q, k_sh, v_sh, beta, log_alpha = shared_projections(x, p, H, d)
    new = np.array(state, F64, copy=True)
    out = np.zeros((B, H, d), F64)
    for b in range(B):
        o_sh, new[b, M] = RULES[rule](new[b, M], q[b], k_sh[b], v_sh[b], beta[b], log_alpha[b], scale)
        out[b] = o_sh
        for j in range(top_k):
            m = int(idx[b, j])
            k_m, v_m = memory_kv(x[b:b + 1], p, m, H, d)
            b_m, la_m = memory_gates(x[b:b + 1], p, m) if has_memory_gates(p) else (beta[b:b + 1], log_alpha[b:b + 1])
            o_m, new[b, m] = RULES[rule](new[b, m], q[b], k_m[0], v_m[0], b_m[0], la_m[0], scale)
            out[b] += gate[b, j] * o_m
    return out, new, idx, gate, near_tie
