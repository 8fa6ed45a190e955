"""GPU parity of the per-memory gates (every routed memory with its own
W_beta^m, W_a^m, A^m, b_a^m: "MoM: Linear Sequence Modeling with
Mixture-of-Memories", Summary, every memory keeps its own recurrent update)
against the oracle with the GPU's routing imposed:

* mom_mem_gate_proj alone, row by row, on the tensor-core path (2H = 4 .. 32
  columns) and the CUDA-core path (float32, d_model not a multiple of 64),
  on the layer's routing and on a hand-made one whose tiny memories make
  16-row tiles straddle several memories; a bad token index is recorded and
  its row zeroed;
* the memory calls with per-row gates equal to the token gates gathered
  through the index give the default call's output bit for bit;
* whole layers with per-memory gates (tensor-core, token-serial and float32
  GDN, both update rules, skewed routing with empty segments, the 380M
  shape at full size) and decode continuing a prefill.
"""
import dataclasses

import numpy as np
import pytest
import torch

from mixture_memories_layer_b200 import synth
from oracle import mom_oracle as orc
from tests.gpu_helpers import TOL, max_abs_rel, run_layer

pytestmark = pytest.mark.gpu
GATE_TOL = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _small(d, dtype="bf16", lens=(300, 77, 1), M=4, k=2, H=2, D=256, seed=21, bias0=0.0):
    w = synth.Workload("small_mg", 0, 0, D, H, d, M, k, dtype, seed=seed, router_bias0=bias0, mem_gates=True)
    rng = np.random.default_rng(seed)
    p = synth.make_weights(w, rng)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    p["cu_seqlens"] = cu
    p["x"] = synth.make_tokens(w, rng, int(cu[-1]))
    return w, p


def _check_gates(p, x, perm, offs, beta_p, la_p):
    for m in range(len(offs) - 1):
        rows = slice(int(offs[m]), int(offs[m + 1]))
        if rows.start == rows.stop:
            continue
        b, la = orc.memory_gates(x[perm[rows]], p, m)
        assert max_abs_rel(beta_p[rows], b) < GATE_TOL, ("beta", m)
        assert max_abs_rel(la_p[rows], la) < GATE_TOL, ("log alpha", m)


def _check_layer(w, p, res, rule, seqs=None):
    tol = TOL[w.dtype]
    cu = p["cu_seqlens"]
    for s in (range(len(cu) - 1) if seqs is None else seqs):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        ref = orc.mom_forward(p["x"][t0:t1], p, np.array([0, t1 - t0]), w.top_k, w.heads, w.d_head,
                              forced_idx=res["idx"][t0:t1], rule=rule)
        e = max_abs_rel(res["out"][t0:t1], ref["out"])
        assert e < tol, ("out", s, e)
        e_hs = max_abs_rel(res["h_shared"][s], ref["h_shared"][0])
        e_hm = max_abs_rel(res["h_mem"][:, s], ref["h_mem"][:, 0])
        assert e_hs < tol and e_hm < tol, ("states", s, e_hs, e_hm)


# ------------------------------------------------------------ gate kernel
@pytest.mark.parametrize("H,D,dtype", [(2, 256, "bf16"), (4, 1024, "bf16"), (8, 512, "bf16"), (16, 256, "bf16"),
                                       (3, 256, "bf16"), (4, 256, "f32")])
def test_mem_gate_proj_on_layer_routing(H, D, dtype):
    w, p = _small(64, dtype=dtype, H=H, D=D, M=5, lens=(333, 70))
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    _check_gates(p, p["x"], res["perm"], res["mem_offset"], res["beta_p"], res["log_alpha_p"])


@pytest.mark.parametrize("H,D,dtype", [(4, 256, "bf16"), (4, 200, "bf16"), (5, 104, "f32")])
def test_mem_gate_proj_tiles_straddling_tiny_memories(H, D, dtype):
    from mixture_memories_layer_b200 import binding as B
    from mixture_memories_layer_b200 import layer as L
    M, K, n_tok = 12, 2, 100
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    w = synth.Workload("straddle", 0, 0, D, H, 64, M, K, dtype, seed=23, mem_gates=True)
    rng = np.random.default_rng(23)
    p = synth.make_weights(w, rng)
    x = synth.make_tokens(w, rng, n_tok)
    # memories of 0, 1, 2, 3, ... rows (several per 16-row tile), the rest to the last
    sizes = [0, 1, 2, 3, 5, 0, 7, 16, 17, 1, 30]
    sizes.append(n_tok * K - sum(sizes))
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    perm = rng.integers(0, n_tok, size=n_tok * K).astype(np.int32)
    wt = L.pack_weights(p, dt)
    g = lambda a: torch.as_tensor(a).cuda()
    bp = torch.full((n_tok * K, H), float("nan"), device="cuda")
    lp = torch.full_like(bp, float("nan"))
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    B.mom_mem_gate_proj(g(x).to(dt), g(perm), g(offs), wt["w_gate_mem"], wt["A_mem"], wt["b_a_mem"], K,
                        bp, lp, ws)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws)[0] == 0
    _check_gates(p, x, perm, offs, bp.cpu().numpy(), lp.cpu().numpy())
    # a token index out of range: recorded, its row zeroed, the others intact
    bad = perm.copy()
    bad[37] = n_tok
    bp.fill_(float("nan"))
    B.mom_mem_gate_proj(g(x).to(dt), g(bad), g(offs), wt["w_gate_mem"], wt["A_mem"], wt["b_a_mem"], K,
                        bp, lp, ws)
    torch.cuda.synchronize()
    code, info = B.mom_get_error(ws)
    assert (code, info) == (B.MOM_DEVERR_ROW_INDEX, 37)
    b = bp.cpu().numpy()
    assert np.all(b[37] == 0) and not np.isnan(b).any()


# -------------------------------------------------- per-row gate layout
@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (256, "bf16"), (64, "bf16"), (64, "f32")])
def test_gates_by_row_equal_to_token_gates_is_the_default_call(d, dtype):
    from mixture_memories_layer_b200 import binding as B
    w, p = _small(d, dtype=dtype, lens=(200, 131))
    p = {k: v for k, v in p.items() if not k.endswith("_mem")}
    lay, res = run_layer(w, p)
    b = lay.buffers(int(p["cu_seqlens"][-1]), len(p["cu_seqlens"]) - 1)
    perm = b["perm"].long()
    beta_p = b["beta"][perm].contiguous()
    la_p = b["log_alpha"][perm].contiguous()
    o1, o2 = torch.empty_like(b["o_p"]), torch.empty_like(b["o_p"])
    h1, h2 = torch.empty_like(b["h_mem"]), torch.empty_like(b["h_mem"])
    for rule in (B.MOM_RULE_GATED_DELTA, B.MOM_RULE_GATED_LINEAR):
        B.mom_memory_chunk_fwd(b["q"], b["perm"], b["k_p"], b["v_p"], b["beta"], b["log_alpha"], b["seg_cu"], 1.0,
                               rule, None, h1, o1, b["ws_gdn_p"])
        B.mom_memory_chunk_fwd(b["q"], b["perm"], b["k_p"], b["v_p"], beta_p, la_p, b["seg_cu"], 1.0,
                               rule, None, h2, o2, b["ws_gdn_p"], gates=B.MOM_GATES_BY_ROW)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(h1, h2), rule


# ------------------------------------------------------------- the layer
@pytest.mark.parametrize("rule", ["gated_delta", "gated_linear"])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_layer_with_per_memory_gates_small_bf16(d, rule):
    w, p = _small(d)
    lay, res = run_layer(w, p, rule=rule)
    assert lay.device_errors() == {}
    _check_layer(w, p, res, rule)


def test_layer_with_per_memory_gates_fp32():
    w, p = _small(64, dtype="f32", lens=(130, 64, 65, 2))
    lay, res = run_layer(w, p)
    _check_layer(w, p, res, "gated_delta")


def test_layer_with_per_memory_gates_skewed_routing_and_empty_segments():
    w, p = _small(128, lens=(200, 0, 90), bias0=6.0)
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    _check_layer(w, p, res, "gated_delta")


def test_layer_with_per_memory_gates_mom380m_full_size():
    w = dataclasses.replace(synth.WORKLOADS["mom380m"], mem_gates=True)
    p = synth.make_problem(w)
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    _check_gates(p, p["x"], res["perm"], res["mem_offset"], res["beta_p"], res["log_alpha_p"])
    _check_layer(w, p, res, "gated_delta", seqs=[5])


def test_decode_with_per_memory_gates_continues_prefill():
    from mixture_memories_layer_b200 import layer as L
    w = synth.Workload("dec_mg", 8, 0, 256, 2, 128, 4, 2, "bf16", seed=25, decode_steps=3, prefill_len=70,
                       mem_gates=True)
    p = synth.make_decode_problem(w, steps=3)
    lay = L.MoMLayer(L.pack_weights(p, torch.bfloat16), w.heads, w.d_head, w.top_k)
    assert lay.mem_gates
    Lp = w.prefill_len
    b = lay.forward(torch.as_tensor(p["x_prefill"]).to("cuda", torch.bfloat16), torch.as_tensor(p["cu_prefill"]).cuda())
    state = torch.empty((w.batch, w.n_mem + 1, w.heads, w.d_head, w.d_head), dtype=torch.float32, device="cuda")
    state[:, :w.n_mem] = b["h_mem"].permute(1, 0, 2, 3, 4)
    state[:, w.n_mem] = b["h_shared"]
    pre_idx = b["idx"].cpu().numpy()
    xs = torch.as_tensor(p["x_steps"]).to("cuda", torch.bfloat16)
    outs, idxs = [], []
    for s in range(3):
        o, i = lay.decode_step(xs[s], state)
        outs.append(o.float().cpu().numpy())
        idxs.append(i.cpu().numpy())
    torch.cuda.synchronize()
    assert lay.device_errors() == {}
    final = state.cpu().numpy()
    tol = TOL["bf16"]
    for bsq in range(w.batch):
        ref = orc.mom_forward(p["x_prefill"][bsq * Lp:(bsq + 1) * Lp], p, np.array([0, Lp]), w.top_k, w.heads,
                              w.d_head, forced_idx=pre_idx[bsq * Lp:(bsq + 1) * Lp])
        st = orc.decode_state_from_prefill(ref["h_shared"], ref["h_mem"])
        for s in range(3):
            o_ref, st, _, _, _ = orc.mom_decode_step(p["x_steps"][s][bsq:bsq + 1], p, st, w.top_k, w.heads,
                                                     w.d_head, forced_idx=idxs[s][bsq:bsq + 1])
            assert max_abs_rel(outs[s][bsq:bsq + 1], o_ref) < tol, ("decode out", bsq, s)
        assert max_abs_rel(final[bsq:bsq + 1], st) < tol
