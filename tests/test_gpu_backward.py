"""GPU parity of the recurrence's reverse pass (mom_memory_chunk_bwd) against
the oracle's reverse pass, itself pinned by finite differences of the
forward ("MoM: Linear Sequence Modeling with Mixture-of-Memories", Key
points: training; the update rules: the authors' MoM blog post).

Small ragged segments that cross the 8- and 64-token boundaries of the
kernel's recomputation (and an empty and a one-token segment), d in {64,
128, 256}, both rules, float32 and bf16 operands, with and without initial
states and final-state gradients, q and the gates read through a row index,
and gates given per row; then a 1024-token stretch (16 chunks) of a
sequence of the 380M layer's shared memory.  Gradients are float32 on both sides; the error
measure is max |gpu - ref| / max |ref| per tensor.
"""
import numpy as np
import pytest
import torch

from oracle import mom_oracle as orc
from oracle import mom_oracle_bwd as bwd
from tests.gpu_helpers import max_abs_rel

pytestmark = pytest.mark.gpu
TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _round(a, dtype):
    if dtype == "bf16":
        return torch.as_tensor(np.asarray(a, np.float32)).bfloat16().float().numpy().astype(np.float64)
    return np.asarray(a, np.float32).astype(np.float64)


def _case(lens, H, d, dtype, seed, qidx=False, with_states=True):
    rng = np.random.default_rng(seed)
    n = int(sum(lens))
    nq = n + 5 if qidx else n
    q = orc.l2norm(rng.standard_normal((nq, H, d)))
    k = orc.l2norm(rng.standard_normal((n, H, d)))
    v = rng.standard_normal((n, H, d))
    beta = rng.uniform(0.05, 0.95, size=(nq, H))
    la = -np.exp(rng.uniform(0.0, 1.0, size=(nq, H))) * np.log1p(np.exp(rng.uniform(-4, 0, size=(nq, H))))
    do = rng.standard_normal((n, H, d))
    S = len(lens)
    h0 = rng.standard_normal((S, H, d, d)) * 0.3 if with_states else None
    dh = rng.standard_normal((S, H, d, d)) * 0.3 if with_states else None
    idx = rng.permutation(nq)[:n].astype(np.int32) if qidx else None
    # gates of their own for every row (the per-row layout)
    beta_rows = rng.uniform(0.05, 0.95, size=(n, H))
    la_rows = -rng.uniform(0.01, 2.0, size=(n, H))
    c = dict(beta_rows=np.asarray(beta_rows, np.float32).astype(np.float64),
             la_rows=np.asarray(la_rows, np.float32).astype(np.float64),
             q=_round(q, dtype), k=_round(k, dtype), v=_round(v, dtype), do=_round(do, dtype),
             beta=np.asarray(beta, np.float32).astype(np.float64), la=np.asarray(la, np.float32).astype(np.float64),
             h0=None if h0 is None else np.asarray(h0, np.float32).astype(np.float64),
             dh=None if dh is None else np.asarray(dh, np.float32).astype(np.float64), idx=idx,
             cu=np.concatenate([[0], np.cumsum(lens)]).astype(np.int32))
    return c


def _oracle(c, rule, scale, gates_by_row):
    n, H, d = c["k"].shape
    S = len(c["cu"]) - 1
    out = dict(dq=np.zeros((n, H, d)), dk=np.zeros((n, H, d)), dv=np.zeros((n, H, d)), dbeta=np.zeros((n, H)),
               dlog_alpha=np.zeros((n, H)), dh0=np.zeros((S, H, d, d)))
    for s in range(S):
        a, b = int(c["cu"][s]), int(c["cu"][s + 1])
        rows = np.arange(a, b)
        qr = c["idx"][rows] if c["idx"] is not None else rows
        bsrc, lsrc, gr = (c["beta_rows"], c["la_rows"], rows) if gates_by_row else (c["beta"], c["la"], qr)
        g = bwd.gdn_recurrence_bwd(c["q"][qr], c["k"][rows], c["v"][rows], bsrc[gr], lsrc[gr], c["do"][rows],
                                   None if c["h0"] is None else c["h0"][s], None if c["dh"] is None else c["dh"][s],
                                   scale, rule)
        for key in ("dq", "dk", "dv", "dbeta", "dlog_alpha"):
            out[key][rows] = g[key]
        out["dh0"][s] = g["dh0"]
    return out


def _gpu(c, rule, scale, dtype, gates_by_row):
    from mixture_memories_layer_b200 import binding as B
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    t = lambda a, ty=dt: torch.as_tensor(np.asarray(a)).to("cuda", ty).contiguous()
    n, H, d = c["k"].shape
    S = len(c["cu"]) - 1
    beta, la = (c["beta_rows"], c["la_rows"]) if gates_by_row else (c["beta"], c["la"])
    f32 = torch.float32
    outs = dict(dq=torch.full((n, H, d), np.nan, device="cuda"), dk=torch.full((n, H, d), np.nan, device="cuda"),
                dv=torch.full((n, H, d), np.nan, device="cuda"), dbeta=torch.full((n, H), np.nan, device="cuda"),
                dlog_alpha=torch.full((n, H), np.nan, device="cuda"), dh0=torch.full((S, H, d, d), np.nan, device="cuda"))
    ws = B.new_workspace(B.mom_memory_chunk_bwd_workspace_size(n, S, H, d))
    B.mom_memory_chunk_bwd(t(c["q"]), None if c["idx"] is None else t(c["idx"], torch.int32), t(c["k"]), t(c["v"]),
                           t(beta, f32), t(la, f32), t(c["cu"], torch.int32), scale, B.RULES[rule],
                           None if c["h0"] is None else t(c["h0"], f32), t(c["do"]),
                           None if c["dh"] is None else t(c["dh"], f32), outs["dq"], outs["dk"], outs["dv"],
                           outs["dbeta"], outs["dlog_alpha"], outs["dh0"], ws,
                           gates=B.MOM_GATES_BY_ROW if gates_by_row else B.MOM_GATES_BY_TOKEN)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws)[0] == 0
    return {k: v.cpu().numpy() for k, v in outs.items()}


def _compare(c, rule, scale, dtype, gates_by_row=False):
    ref = _oracle(c, rule, scale, gates_by_row)
    got = _gpu(c, rule, scale, dtype, gates_by_row)
    for key in ref:
        assert not np.isnan(got[key]).any(), key
        e = max_abs_rel(got[key], ref[key])
        assert e < TOL, (key, e)


@pytest.mark.parametrize("rule", ["gated_delta", "gated_linear"])
@pytest.mark.parametrize("d,dtype", [(64, "f32"), (128, "bf16"), (256, "bf16"), (256, "f32")])
def test_recurrence_bwd_ragged_segments(d, dtype, rule):
    c = _case((137, 0, 1, 70, 9), H=2, d=d, dtype=dtype, seed=d + (rule == "gated_linear"))
    _compare(c, rule, 1.0, dtype)


def test_recurrence_bwd_without_states_and_with_scale():
    c = _case((65, 64, 3), H=1, d=128, dtype="f32", seed=7, with_states=False)
    _compare(c, "gated_delta", 0.7, "f32")


@pytest.mark.parametrize("gates_by_row", [False, True])
def test_recurrence_bwd_through_a_row_index(gates_by_row):
    c = _case((90, 33, 129), H=2, d=128, dtype="bf16", seed=11, qidx=True)
    _compare(c, "gated_delta", 1.0, "bf16", gates_by_row)


def test_recurrence_bwd_380m_shared_memory_long_segment():
    """The first 1024 tokens (16 chunks) of a sequence of the 380M layer's
    shared memory, on the layer's own q, k, v and gates, all four heads on
    the GPU; the oracle (which keeps every state) checks one head."""
    from mixture_memories_layer_b200 import binding as B
    from mixture_memories_layer_b200 import synth
    from tests.gpu_helpers import run_layer
    w = synth.WORKLOADS["mom380m"]
    p = synth.make_problem(w)
    lay, res = run_layer(w, p)
    seq, T, hh = 2, 1024, 1
    a = int(p["cu_seqlens"][seq])
    b = a + T
    rng = np.random.default_rng(5)
    f64 = lambda x: np.asarray(x, np.float64)
    c = dict(q=f64(res["q"][a:b]), k=f64(res["k_sh"][a:b]), v=f64(res["v_sh"][a:b]), beta=f64(res["beta"][a:b]),
             la=f64(res["log_alpha"][a:b]), do=_round(rng.standard_normal((T, w.heads, w.d_head)), "bf16"),
             h0=None, dh=np.asarray(rng.standard_normal((1, w.heads, w.d_head, w.d_head)) * 0.1, np.float32)
             .astype(np.float64), idx=None, cu=np.array([0, T], np.int32))
    got = _gpu(c, "gated_delta", 1.0, "bf16", False)
    one = {key: (c[key][:, hh:hh + 1] if c.get(key) is not None and key != "cu" and key != "idx" else c.get(key))
           for key in ("q", "k", "v", "beta", "la", "do")}
    g = bwd.gdn_recurrence_bwd(one["q"], one["k"], one["v"], one["beta"], one["la"], one["do"], None,
                               c["dh"][0][hh:hh + 1], 1.0, "gated_delta")
    for key, sl in (("dq", np.s_[:, hh:hh + 1]), ("dk", np.s_[:, hh:hh + 1]), ("dv", np.s_[:, hh:hh + 1]),
                    ("dbeta", np.s_[:, hh:hh + 1]), ("dlog_alpha", np.s_[:, hh:hh + 1])):
        e = max_abs_rel(got[key][sl], g[key])
        assert e < TOL, (key, e)
    assert max_abs_rel(got["dh0"][0, hh:hh + 1], g["dh0"]) < TOL
