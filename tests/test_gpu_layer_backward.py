"""GPU parity of the whole layer's backward (MoMLayer.backward: the
recurrences' reverse passes, the combine, router, norm and gate adjoints and
the projections' gradient GEMMs) against the oracle's layer backward, itself
pinned by finite differences of the forward ("MoM: Linear Sequence Modeling
with Mixture-of-Memories", Key points: training; explainer, Router
mechanics: the gradients flow through the renormalised gates, the top-k
choice held fixed).  The oracle runs with the GPU's routing.  float32 layers
within 1e-5 (measured ~1e-6), bf16 layers (operands rounded to bf16 in the
forward) within 2e-2 (measured 2e-4 .. 1.3e-2), per gradient tensor,
max |gpu - ref| / max |ref|.
"""
import numpy as np
import pytest
import torch

from mixture_memories_layer_b200 import synth
from oracle import mom_oracle_bwd as obwd
from tests.gpu_helpers import max_abs_rel

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _run(dtype, d, lens, M=4, K=2, H=2, D=256, seed=81, with_states=True, mem_gates=False, rule="gated_delta"):
    from mixture_memories_layer_b200 import layer as L
    w = synth.Workload("bwd", 0, 0, D, H, d, M, K, dtype, seed=seed, mem_gates=mem_gates)
    rng = np.random.default_rng(seed)
    p = synth.make_weights(w, rng)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x = synth.make_tokens(w, rng, int(cu[-1]))
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    lay = L.MoMLayer(L.pack_weights(p, dt), H, d, K, rule=rule)
    xt = torch.as_tensor(x).to("cuda", dt)
    cut = torch.as_tensor(cu).cuda()
    b = lay.forward(xt, cut)
    n, S = xt.shape[0], len(cu) - 1
    dout = synth._act(rng.standard_normal((n, H, d)).astype(np.float32), dtype)
    dh_sh = rng.standard_normal((S, H, d, d)).astype(np.float32) * 0.1 if with_states else None
    dh_m = rng.standard_normal((M, S, H, d, d)).astype(np.float32) * 0.1 if with_states else None
    t = lambda a, ty=torch.float32: None if a is None else torch.as_tensor(a).to("cuda", ty)
    g = lay.backward(xt, cut, t(dout, dt), dh_shared=t(dh_sh), dh_mem=t(dh_m))
    torch.cuda.synchronize()
    assert lay.device_errors() == {}
    got = {k: v.cpu().numpy().astype(np.float64) for k, v in g.items()}
    idx = b["idx"].cpu().numpy()
    ref = obwd.mom_backward(x, p, cu, K, H, d, dout, forced_idx=idx, dh_shared=dh_sh, dh_mem=dh_m, rule=rule)
    Hd = H * d
    pairs = {
        "dx": (got["dx"], ref["dx"]), "dw_r": (got["dw_r"], ref["dw_r"]), "db_r": (got["db_r"], ref["db_r"]),
        "dw_q": (got["dw_shared"][:Hd], ref["dw_q"]), "dw_k_sh": (got["dw_shared"][Hd:2 * Hd], ref["dw_k_sh"]),
        "dw_v_sh": (got["dw_shared"][2 * Hd:], ref["dw_v_sh"]), "dw_beta": (got["dw_gate"][:H], ref["dw_beta"]),
        "dw_a": (got["dw_gate"][H:], ref["dw_a"]), "dA": (got["dA"], ref["dA"]), "db_a": (got["db_a"], ref["db_a"]),
        "dw_k": (got["dw_kv"][:, :Hd], ref["dw_k"]), "dw_v": (got["dw_kv"][:, Hd:], ref["dw_v"]),
        "dh0_shared": (got["dh0_shared"], ref["dh0_shared"]), "dh0_mem": (got["dh0_mem"], ref["dh0_mem"]),
    }
    if mem_gates:
        pairs.update({"dw_beta_mem": (got["dw_gate_mem"][:, :H], ref["dw_beta_mem"]),
                      "dw_a_mem": (got["dw_gate_mem"][:, H:], ref["dw_a_mem"]),
                      "dA_mem": (got["dA_mem"], ref["dA_mem"]), "db_a_mem": (got["db_a_mem"], ref["db_a_mem"])})
    return {k: max_abs_rel(a, r) for k, (a, r) in pairs.items()}


@pytest.mark.parametrize("lens", [(130, 64, 65, 2), (77, 0, 200)])
def test_layer_backward_fp32(lens):
    errs = _run("f32", 64, lens)
    bad = {k: e for k, e in errs.items() if not e < 1e-5}
    assert not bad, bad


def test_layer_backward_bf16_tensor_core_forward():
    errs = _run("bf16", 128, (150, 61, 1), seed=82)
    bad = {k: e for k, e in errs.items() if not e < 2e-2}
    assert not bad, (bad, errs)


def test_layer_backward_without_state_gradients():
    errs = _run("f32", 64, (90, 33), M=5, K=3, seed=83, with_states=False)
    bad = {k: e for k, e in errs.items() if not e < 1e-5}
    assert not bad, bad


# ------------------------------------------------- the grouped GEMM alone --
def _gemm_case(trans_a, a_col, lda_pad, seed):
    """mom_gemm_grouped with bf16 B (the tf32 tensor-core kernel) against
    numpy in fp64: groups of ragged sizes (one empty), a ragged N, A read
    from column a_col of a wider matrix (a_col and the row pitch decide
    whether the 16-byte loads or the element loads run), the routed form's
    gathered B rows and per-group C, and accumulation into C."""
    from mixture_memories_layer_b200 import binding as B
    rng = np.random.default_rng(seed)
    sizes = [130, 0, 77, 256, 5]
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    rows, G = int(off[-1]), len(sizes)
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    bf = lambda a: torch.as_tensor(a, dtype=torch.float32).to("cuda", torch.bfloat16)
    if not trans_a:
        K, N = 96, 200
        A = rng.standard_normal((rows, K + lda_pad)).astype(np.float32)
        Bw = bf(rng.standard_normal((G, K, N)))
        gidx = rng.permutation(G).astype(np.int32)
        C0 = rng.standard_normal((rows, N)).astype(np.float32)
        C = torch.as_tensor(C0).cuda()
        B.mom_gemm_grouped(0, torch.as_tensor(A).cuda(), Bw, C, 0, N, K, torch.as_tensor(off).cuda(),
                           torch.as_tensor(gidx).cuda(), G, ws, a_col=a_col, total_rows=rows, b_group_stride=K * N,
                           accumulate=True)
        Bn = Bw.float().cpu().numpy().astype(np.float64)
        ref = C0.astype(np.float64).copy()
        for q in range(G):
            ref[off[q]:off[q + 1]] += A[off[q]:off[q + 1], a_col:a_col + K].astype(np.float64) @ Bn[gidx[q]]
    else:
        M, N, n_b = 72, 136, 700
        A = rng.standard_normal((rows, M + lda_pad)).astype(np.float32)
        Bx = bf(rng.standard_normal((n_b, N)))
        b_rows = rng.integers(0, n_b, rows).astype(np.int32)
        C = torch.zeros((G * M, N), device="cuda")
        B.mom_gemm_grouped(1, torch.as_tensor(A).cuda(), Bx, C, M, N, 0, torch.as_tensor(off).cuda(), None, G, ws,
                           a_col=a_col, b_rows=torch.as_tensor(b_rows).cuda(), c_group_stride=M * N)
        Bn = Bx.float().cpu().numpy().astype(np.float64)
        ref = np.zeros((G * M, N))
        for q in range(G):
            r = slice(off[q], off[q + 1])
            ref[q * M:(q + 1) * M] = A[r, a_col:a_col + M].astype(np.float64).T @ Bn[b_rows[r]]
    torch.cuda.synchronize()
    assert B.mom_get_error(ws)[0] == 0
    return max_abs_rel(C.cpu().numpy(), ref)


@pytest.mark.parametrize("trans_a", [0, 1])
@pytest.mark.parametrize("a_col,lda_pad", [(0, 0), (4, 8), (1, 3)])
def test_gemm_grouped_tf32(trans_a, a_col, lda_pad):
    """tf32 products (A rounded to a 10-bit mantissa, B exact, fp32 sums):
    within 2e-3 of the fp64 product per tensor."""
    assert _gemm_case(trans_a, a_col, lda_pad, seed=10 * trans_a + a_col) < 2e-3


@pytest.mark.parametrize("dtype,tol", [("f32", 1e-5), ("bf16", 2e-2)])
def test_layer_backward_per_memory_gates(dtype, tol):
    """Each memory's own gates (MOM_GATES_BY_ROW): the routed reverse pass on
    the rows' gates, their adjoints through mom_gates_bwd_by_group into the
    memories' gate weights, A_mem and b_a_mem."""
    errs = _run(dtype, 64, (120, 0, 77), M=4, K=2, seed=84, mem_gates=True)
    bad = {k: e for k, e in errs.items() if not e < tol}
    assert not bad, (bad, errs)


@pytest.mark.parametrize("dtype,tol", [("f32", 1e-5), ("bf16", 2e-2)])
def test_layer_backward_scalar_gated_linear_rule(dtype, tol):
    """The layer backward with the scalar-gated linear memories (MOM_RULE_GATED_LINEAR)."""
    errs = _run(dtype, 64, (100, 3, 60), seed=85, rule="gated_linear")
    bad = {k: e for k, e in errs.items() if not e < tol}
    assert not bad, (bad, errs)


def test_layer_backward_on_a_caller_stream():
    """Forward and backward launched on the caller's own stream (not torch's
    current one) give the gradients of the default-stream run: every table
    the calls read is made on the launching stream."""
    from mixture_memories_layer_b200 import layer as L
    w = synth.Workload("bwd", 0, 0, 256, 2, 64, 4, 2, "bf16", seed=86)
    rng = np.random.default_rng(86)
    p = synth.make_weights(w, rng)
    cu = torch.as_tensor(np.array([0, 90, 91, 200], np.int32)).cuda()
    x = torch.as_tensor(synth.make_tokens(w, rng, 200)).to("cuda", torch.bfloat16)
    dout = torch.as_tensor(rng.standard_normal((200, 2, 64)).astype(np.float32)).to("cuda", torch.bfloat16)
    grads = []
    for use_stream in (False, True):
        lay = L.MoMLayer(L.pack_weights(p, torch.bfloat16), 2, 64, 2)      # fresh tables each time
        s = torch.cuda.Stream() if use_stream else None
        if s is not None:
            s.wait_stream(torch.cuda.current_stream())
        lay.forward(x, cu, stream=s)
        g = lay.backward(x, cu, dout, stream=s)
        torch.cuda.synchronize()
        assert lay.device_errors() == {}
        grads.append({k: v.clone() for k, v in g.items()})
    for k in grads[0]:
        e = max_abs_rel(grads[1][k].cpu().numpy(), grads[0][k].cpu().numpy())
        assert e < 1e-5, (k, e)
