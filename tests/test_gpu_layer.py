"""GPU parity of the whole MoM layer and of each C-ABI entry point against
the fp64 oracle, on seeded inputs small enough for the oracle to finish in
seconds while still spanning several 64-row chunks, several GEMM tiles and
ragged tails.

Acceptance ("MoM: Linear Sequence Modeling with Mixture-of-Memories",
Summary, for what the layer computes): router indices and the permutation
bit-exact, with near-tie tokens (k-th vs (k+1)-th logit gap < 1e-4) counted
and excluded; outputs and final states within max-abs-rel 1e-4 (float32) or
2e-2 (bf16 inputs, float32 state).  The oracle is re-run with the GPU's
routing imposed, so that a near-tie choice does not change a whole memory's
downstream state.
"""
import numpy as np
import pytest
import torch

from mixture_memories_layer_b200 import synth
from oracle import mom_oracle as orc
from tests.gpu_helpers import TOL, max_abs_rel, run_layer, to_np, torch_dtype

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _small(d, dtype="bf16", lens=(300, 77, 1), M=4, k=2, H=2, D=256, seed=0, bias0=0.0):
    w = synth.Workload("small", 0, 0, D, H, d, M, k, dtype, seed=seed, router_bias0=bias0)
    rng = np.random.default_rng(seed)
    p = synth.make_weights(w, rng)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    p["cu_seqlens"] = cu
    p["x"] = synth.make_tokens(w, rng, int(cu[-1]))
    return w, p


def _check_layer(w, p, res, seqs=None, scale=1.0, tol=None, out_rows=None):
    tol = tol or TOL[w.dtype]
    cu = p["cu_seqlens"]
    S = len(cu) - 1
    seqs = range(S) if seqs is None else seqs
    for s in seqs:
        t0, t1 = int(cu[s]), int(cu[s + 1])
        if out_rows is not None:
            t1 = min(t1, t0 + out_rows)
        ref = orc.mom_forward(p["x"][t0:t1], p, np.array([0, t1 - t0]), w.top_k, w.heads, w.d_head,
                              scale=scale, forced_idx=res["idx"][t0:t1])
        # routing: bit-exact outside near ties
        keep = ~ref["near_tie"]
        nat = orc.router_topk(p["x"][t0:t1], p["w_r"], p["b_r"], w.top_k)[0]
        assert np.array_equal(res["idx"][t0:t1][keep], nat[keep]), "router indices differ"
        assert max_abs_rel(res["gate"][t0:t1], ref["gate"]) < 1e-5
        e_out = max_abs_rel(res["out"][t0:t1], ref["out"])
        assert e_out < tol, ("out", s, e_out)
        if out_rows is None or t1 == int(cu[s + 1]):
            e_hs = max_abs_rel(res["h_shared"][s], ref["h_shared"][0])
            e_hm = max_abs_rel(res["h_mem"][:, s], ref["h_mem"][:, 0])
            assert e_hs < tol and e_hm < tol, ("states", s, e_hs, e_hm)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_layer_small_bf16(d):
    w, p = _small(d)
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    _check_layer(w, p, res)


def test_layer_tiny_fp32_workload():
    w = synth.WORKLOADS["tiny_fp32"]
    p = synth.make_problem(w)
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    _check_layer(w, p, res)


@pytest.mark.parametrize("d", [64, 256])
def test_layer_small_fp32_ragged(d):
    w, p = _small(d, dtype="f32", lens=(130, 64, 65, 2))
    lay, res = run_layer(w, p, scale=0.5)
    _check_layer(w, p, res, scale=0.5)


def test_layer_skewed_routing_and_empty_segments():
    # +6 on memory 0 sends nearly every token there; memories 1-3 see few or none
    w, p = _small(128, lens=(200, 0, 90), bias0=6.0)
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    _check_layer(w, p, res)


def test_layer_all_tokens_one_memory_top1_M1():
    w, p = _small(64, M=1, k=1, lens=(150,))
    lay, res = run_layer(w, p)
    assert np.all(res["idx"] == 0) and np.allclose(res["gate"], 1.0)
    _check_layer(w, p, res)


def test_layer_many_memories_top4():
    w, p = _small(64, M=16, k=4, lens=(257, 31), H=3, D=192)
    lay, res = run_layer(w, p)
    _check_layer(w, p, res)


def test_layer_top_k_equals_memories():
    # every token reaches every memory: the gates are the whole softmax over M
    w, p = _small(128, M=4, k=4, lens=(130, 3))
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    assert np.all(np.sort(res["idx"], axis=1) == np.arange(4))
    _check_layer(w, p, res)


def test_layer_single_token():
    w, p = _small(256, lens=(1,))
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    _check_layer(w, p, res)


def test_layer_many_tiny_sequences():
    # 48 sequences of 0-5 tokens: nearly every (memory, sequence) segment
    # holds 0-3 rows, many chunks are both first and last
    lens = tuple(int(v) for v in np.random.default_rng(5).integers(0, 6, size=48))
    w, p = _small(64, lens=lens, seed=5)
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    _check_layer(w, p, res)


@pytest.mark.parametrize("with_h0", [False, True])
def test_layer_no_tokens(with_h0):
    # two empty sequences: no output rows; every final state is its initial
    # state (zeros without one)
    from mixture_memories_layer_b200 import layer as L
    w, p = _small(256, lens=(0, 0))
    dt = torch.bfloat16
    lay = L.MoMLayer(L.pack_weights(p, dt), w.heads, w.d_head, w.top_k)
    x = torch.empty((0, w.d_model), dtype=dt, device="cuda")
    cu = torch.zeros(3, dtype=torch.int32, device="cuda")
    H, d, M = w.heads, w.d_head, w.n_mem
    h0s = torch.randn((2, H, d, d), device="cuda") if with_h0 else None
    h0m = torch.randn((M, 2, H, d, d), device="cuda") if with_h0 else None
    b = lay.forward(x, cu, h0_shared=h0s, h0_mem=h0m)
    torch.cuda.synchronize()
    assert lay.device_errors() == {}
    assert tuple(b["out"].shape) == (0, H, d)
    assert torch.equal(b["h_shared"], h0s if with_h0 else torch.zeros_like(b["h_shared"]))
    assert torch.equal(b["h_mem"], h0m if with_h0 else torch.zeros_like(b["h_mem"]))
    assert tuple(b["seg_cu"].cpu().tolist()) == (0,) * (M * 2 + 1)


def test_binding_refuses_strided_views():
    from mixture_memories_layer_b200 import binding as B
    x = torch.zeros((64, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="non-contiguous"):
        B._p(x.t())
    assert B._p(x).value == x.data_ptr()


def test_layer_h0_hand_off():
    """Forward over [0, T) equals [0, T/2) then [T/2, T) seeded with the
    first call's final states."""
    w, p = _small(128, lens=(160,))
    _, full = run_layer(w, p)
    x = p["x"]
    pa = dict(p, x=x[:70], cu_seqlens=np.array([0, 70], np.int32))
    pb = dict(p, x=x[70:], cu_seqlens=np.array([0, 90], np.int32))
    _, ra = run_layer(w, pa)
    h0s = torch.as_tensor(ra["h_shared"]).cuda()
    h0m = torch.as_tensor(ra["h_mem"]).cuda()
    _, rb = run_layer(w, pb, h0_shared=h0s, h0_mem=h0m)
    tol = TOL[w.dtype]
    assert max_abs_rel(rb["out"], full["out"][70:]) < tol
    assert max_abs_rel(rb["h_mem"], full["h_mem"]) < tol
    assert max_abs_rel(rb["h_shared"], full["h_shared"]) < tol


def test_permute_bit_exact():
    w, p = _small(64, M=8, k=2, lens=(500, 3, 0, 260))
    lay, res = run_layer(w, p)
    perm, row_of, offs, seg = orc.permute(res["idx"], w.n_mem, p["cu_seqlens"])
    n = int(offs[-1])
    assert np.array_equal(res["perm"][:n], perm)
    assert np.array_equal(res["row_of"], row_of)
    assert np.array_equal(res["mem_offset"], offs)
    assert np.array_equal(res["seg_cu"], seg)


def test_projections_match_oracle():
    w, p = _small(128, lens=(200, 57))
    lay, res = run_layer(w, p)
    q, k_sh, v_sh, beta, la = orc.shared_projections(p["x"], p, w.heads, w.d_head)
    tol = TOL[w.dtype]
    for name, ref in (("q", q), ("k_sh", k_sh), ("v_sh", v_sh)):
        assert max_abs_rel(res[name], ref) < tol, name
    assert max_abs_rel(res["beta"], beta) < 1e-5
    assert max_abs_rel(res["log_alpha"], la) < 1e-5
    perm, _, offs, _ = orc.permute(res["idx"], w.n_mem, p["cu_seqlens"])
    for m in range(w.n_mem):
        rows = slice(offs[m], offs[m + 1])
        km, vm = orc.memory_kv(p["x"][perm[rows]], p, m, w.heads, w.d_head)
        assert max_abs_rel(res["k_p"][rows], km) < tol
        assert max_abs_rel(res["v_p"][rows], vm) < tol


def test_projections_with_gates_equal_separate_gate_call():
    """mom_kv_proj_grouped given beta / log_alpha writes exactly what the
    layer's separate mom_gate_proj call (beside the router) writes, and the
    same k / v."""
    from mixture_memories_layer_b200 import binding as B
    w, p = _small(128, lens=(200, 57))
    lay, res = run_layer(w, p)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    wt = lay.w
    x = torch.as_tensor(p["x"]).to("cuda", dt)
    g = lambda a, t=torch.int32: torch.as_tensor(a).to("cuda", t)
    n, H, d, K = x.shape[0], w.heads, w.d_head, w.top_k
    outs = {k: torch.empty((n, H, d), dtype=dt, device="cuda") for k in ("q", "k_sh", "v_sh")}
    kp = torch.empty((n * K, H, d), dtype=dt, device="cuda")
    vp = torch.empty_like(kp)
    beta = torch.empty((n, H), dtype=torch.float32, device="cuda")
    la = torch.empty_like(beta)
    ws = B.new_workspace(B.mom_kv_proj_workspace_size(n, w.d_model, H, d, w.n_mem, K))
    B.mom_kv_proj_grouped(x, g(res["perm"]), g(res["mem_offset"]), wt["w_shared"], wt["w_gate"], wt["A"], wt["b_a"],
                          wt["w_kv"], H, d, K, outs["q"], outs["k_sh"], outs["v_sh"], beta, la, kp, vp, ws)
    torch.cuda.synchronize()
    assert np.array_equal(beta.cpu().numpy(), res["beta"])
    assert np.array_equal(la.cpu().numpy(), res["log_alpha"])
    for k in ("q", "k_sh", "v_sh"):
        assert np.array_equal(outs[k].float().cpu().numpy(), res[k])
    rows = int(res["mem_offset"][-1])
    assert np.array_equal(kp[:rows].float().cpu().numpy(), res["k_p"][:rows])
