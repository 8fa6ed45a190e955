"""Pins for the oracle's router and reordering, against brute force.

Router: "one matmul, one softmax, one top-k, one renormalisation"
("MoM: Mixture-of-Memories Fixes Linear Attention Recall", Router mechanics,
step by step).  Reordering: routed pairs become contiguous per-memory
segments in token order (same page, "Solving scatter-gather without new
kernels").
"""
import itertools
import math

import numpy as np
import pytest

from oracle import mom_oracle as orc


def _python_softmax(row):
    mx = max(row)
    e = [math.exp(z - mx) for z in row]
    s = sum(e)
    return [v / s for v in e]


@pytest.mark.parametrize("M,k", [(4, 1), (4, 2), (5, 3), (8, 2), (16, 4)])
def test_router_matches_subset_brute_force(M, k):
    rng = np.random.default_rng(10 + M * 7 + k)
    N, D = 40, 12
    x = rng.standard_normal((N, D))
    w_r = rng.standard_normal((M, D)) / np.sqrt(D)
    b_r = rng.standard_normal(M) * 0.1
    idx, gate, logits, near = orc.router_topk(x, w_r, b_r, k)
    for t in range(N):
        lg = [sum(float(x[t, c]) * float(w_r[m, c]) for c in range(D)) + float(b_r[m]) for m in range(M)]
        # the top-k set maximises the sum of logits over all k-subsets
        best = max(itertools.combinations(range(M), k), key=lambda c: sum(lg[i] for i in c))
        assert set(int(i) for i in idx[t]) == set(best)
        # rank order: descending logit
        ranked = sorted(best, key=lambda i: -lg[i])
        assert [int(i) for i in idx[t]] == ranked
        # softmax over all M, keep the chosen, renormalise
        p = _python_softmax(lg)
        tot = sum(p[i] for i in ranked)
        for j, i in enumerate(ranked):
            assert abs(gate[t, j] - p[i] / tot) < 1e-12
        assert abs(gate[t].sum() - 1.0) < 1e-12


def test_router_topk_equal_M_is_full_softmax():
    rng = np.random.default_rng(3)
    N, D, M = 20, 8, 6
    x = rng.standard_normal((N, D))
    w_r = rng.standard_normal((M, D))
    idx, gate, logits, near = orc.router_topk(x, w_r, None, M)
    assert not near.any()
    for t in range(N):
        lg = [float(v) for v in logits[t]]
        p = _python_softmax(lg)
        for j in range(M):
            assert abs(gate[t, j] - p[int(idx[t, j])]) < 1e-12
        assert sorted(int(i) for i in idx[t]) == list(range(M))


def test_router_ties_go_to_lower_index():
    # memories 1 and 3 have identical weights and the largest logits
    D = 4
    x = np.array([[1.0, 0.5, -0.25, 2.0]])
    w_r = np.array([[0.1, 0.0, 0.0, 0.0],
                    [1.0, 1.0, 1.0, 1.0],
                    [0.0, 0.2, 0.0, 0.0],
                    [1.0, 1.0, 1.0, 1.0]])
    idx, gate, _, near = orc.router_topk(x, w_r, None, 1)
    assert idx[0, 0] == 1
    assert near[0]          # gap 0 < 1e-4
    idx, gate, _, near = orc.router_topk(x, w_r, None, 2)
    assert list(idx[0]) == [1, 3]
    assert abs(gate[0, 0] - 0.5) < 1e-15 and abs(gate[0, 1] - 0.5) < 1e-15


def test_router_near_tie_flag():
    x = np.eye(3)
    # logits of token 0: (1.0, 1.0 - 5e-5, 0) -> near tie for top-1
    # logits of token 1: (0.3, 0.3 + 2e-4, 0) -> not a near tie
    w_r = np.array([[1.0, 0.3, 0.0], [1.0 - 5e-5, 0.3 + 2e-4, 0.0], [0.0, 0.0, 0.0]])
    _, _, _, near = orc.router_topk(x, w_r, None, 1)
    assert bool(near[0]) and not bool(near[1])


def test_router_bias_shift_invariance_and_skew():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((30, 8))
    w_r = rng.standard_normal((4, 8))
    i1, g1, _, _ = orc.router_topk(x, w_r, np.zeros(4), 2)
    i2, g2, _, _ = orc.router_topk(x, w_r, np.full(4, 7.5), 2)
    assert np.array_equal(i1, i2) and np.allclose(g1, g2, atol=1e-14)
    i3, _, _, _ = orc.router_topk(x, w_r, np.array([100.0, 0, 0, 0]), 2)
    assert (i3[:, 0] == 0).all()


def _loop_permute(idx, M, cu):
    N, k = len(idx), len(idx[0]) if len(idx) else 0
    perm, row_of = [], [None] * (N * k)
    offs, seg = [], []
    S = len(cu) - 1
    for m in range(M):
        offs.append(len(perm))
        for s in range(S):
            seg.append(len(perm))
            for t in range(cu[s], cu[s + 1]):
                for j in range(k):
                    if idx[t][j] == m:
                        row_of[t * k + j] = len(perm)
                        perm.append(t)
    offs.append(len(perm))
    seg.append(len(perm))
    return perm, row_of, offs, seg


@pytest.mark.parametrize("case", ["random", "one_memory", "empty_memory", "empty_sequence", "no_tokens"])
def test_permute_matches_loop_construction(case):
    rng = np.random.default_rng(11)
    M, k = 5, 2
    cu = [0, 7, 19, 19, 33]
    N = cu[-1]
    if case == "random":
        idx = np.array([rng.choice(M, k, replace=False) for _ in range(N)])
    elif case == "one_memory":
        k = 1
        idx = np.full((N, 1), 3)
    elif case == "empty_memory":
        idx = np.array([rng.choice([0, 1, 3, 4], k, replace=False) for _ in range(N)])
    elif case == "empty_sequence":
        cu = [0, 0, 10, 10, 33, 33]
        idx = np.array([rng.choice(M, k, replace=False) for _ in range(N)])
    else:
        cu = [0, 0]
        N = 0
        idx = np.zeros((0, k), dtype=np.int64)
    perm, row_of, offs, seg = orc.permute(idx, M, np.array(cu))
    e_perm, e_row, e_offs, e_seg = _loop_permute(idx.tolist(), M, cu)
    assert perm.tolist() == e_perm
    assert row_of.tolist() == e_row
    assert offs.tolist() == e_offs
    assert seg.tolist() == e_seg
    # bijection: every pair appears exactly once, and row_of inverts the order
    assert sorted(row_of.tolist()) == list(range(N * k))
    for t in range(N):
        for j in range(k):
            assert perm[row_of[t * k + j]] == t
    # each memory's segment length equals its routed count
    counts = np.bincount(idx.reshape(-1), minlength=M) if N else np.zeros(M, int)
    assert (np.diff(offs) == counts).all()
