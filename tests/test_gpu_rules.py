"""GPU parity of the second memory rule, the scalar-gated linear form
S_t = alpha_t S_{t-1} + beta_t v_t k_t^T (the authors' MoM blog post,
"Linear Recurrent Memory": linear attention, RetNet, Mamba2-style memories),
against the oracle run with the same rule and the GPU's routing imposed:
small ragged layers on the tensor-core path (d = 128, 256), the token-serial
path (d = 64) and float32, skewed routing with empty segments, the
380M-shape layer at full size (one whole sequence with its final states),
and decode continuing a prefill.  Also: the rule-taking GDN entry point with
the Gated DeltaNet rule is the default call, bit for bit.
"""
import numpy as np
import pytest
import torch

from mixture_memories_layer_b200 import synth
from oracle import mom_oracle as orc
from tests.gpu_helpers import TOL, max_abs_rel, run_layer

pytestmark = pytest.mark.gpu
RULE = "gated_linear"


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _small(d, dtype="bf16", lens=(300, 77, 1), M=4, k=2, H=2, D=256, seed=5, bias0=0.0):
    w = synth.Workload("small", 0, 0, D, H, d, M, k, dtype, seed=seed, router_bias0=bias0)
    rng = np.random.default_rng(seed)
    p = synth.make_weights(w, rng)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    p["cu_seqlens"] = cu
    p["x"] = synth.make_tokens(w, rng, int(cu[-1]))
    return w, p


def _check(w, p, res, seqs=None):
    tol = TOL[w.dtype]
    cu = p["cu_seqlens"]
    for s in (range(len(cu) - 1) if seqs is None else seqs):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        ref = orc.mom_forward(p["x"][t0:t1], p, np.array([0, t1 - t0]), w.top_k, w.heads, w.d_head,
                              forced_idx=res["idx"][t0:t1], rule=RULE)
        e = max_abs_rel(res["out"][t0:t1], ref["out"])
        assert e < tol, ("out", s, e)
        e_hs = max_abs_rel(res["h_shared"][s], ref["h_shared"][0])
        e_hm = max_abs_rel(res["h_mem"][:, s], ref["h_mem"][:, 0])
        assert e_hs < tol and e_hm < tol, ("states", s, e_hs, e_hm)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_gated_linear_layer_small_bf16(d):
    w, p = _small(d)
    lay, res = run_layer(w, p, rule=RULE)
    assert lay.device_errors() == {}
    _check(w, p, res)


def test_gated_linear_layer_small_fp32():
    w, p = _small(64, dtype="f32", lens=(130, 64, 65, 2))
    lay, res = run_layer(w, p, rule=RULE)
    _check(w, p, res)


def test_gated_linear_skewed_routing_and_empty_segments():
    w, p = _small(128, lens=(200, 0, 90), bias0=6.0)
    lay, res = run_layer(w, p, rule=RULE)
    assert lay.device_errors() == {}
    _check(w, p, res)


def test_gated_linear_mom380m_full_size():
    w = synth.WORKLOADS["mom380m"]
    p = synth.make_problem(w)
    lay, res = run_layer(w, p, rule=RULE)
    assert lay.device_errors() == {}
    _check(w, p, res, seqs=[3])


def test_gated_linear_decode_continues_prefill():
    from mixture_memories_layer_b200 import layer as L
    w = synth.Workload("dec_gla", 8, 0, 256, 2, 128, 4, 2, "bf16", seed=12, decode_steps=3, prefill_len=70)
    p = synth.make_decode_problem(w, steps=3)
    lay = L.MoMLayer(L.pack_weights(p, torch.bfloat16), w.heads, w.d_head, w.top_k, rule=RULE)
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
    final = state.cpu().numpy()
    tol = TOL["bf16"]
    for bsq in range(w.batch):
        ref = orc.mom_forward(p["x_prefill"][bsq * Lp:(bsq + 1) * Lp], p, np.array([0, Lp]), w.top_k, w.heads,
                              w.d_head, forced_idx=pre_idx[bsq * Lp:(bsq + 1) * Lp], rule=RULE)
        st = orc.decode_state_from_prefill(ref["h_shared"], ref["h_mem"])
        for s in range(3):
            o_ref, st, _, _, _ = orc.mom_decode_step(p["x_steps"][s][bsq:bsq + 1], p, st, w.top_k, w.heads,
                                                     w.d_head, forced_idx=idxs[s][bsq:bsq + 1], rule=RULE)
            assert max_abs_rel(outs[s][bsq:bsq + 1], o_ref) < tol, ("decode out", bsq, s)
        assert max_abs_rel(final[bsq:bsq + 1], st) < tol


def test_rule_entry_with_gated_delta_is_the_default_call():
    from mixture_memories_layer_b200 import binding as B
    w, p = _small(256, lens=(200, 131))
    lay, res = run_layer(w, p)
    b = lay.buffers(int(p["cu_seqlens"][-1]), len(p["cu_seqlens"]) - 1)
    cu = torch.as_tensor(p["cu_seqlens"]).cuda()
    o1, o2 = torch.empty_like(b["o_sh"]), torch.empty_like(b["o_sh"])
    h1, h2 = torch.empty_like(b["h_shared"]), torch.empty_like(b["h_shared"])
    args = (b["q"], None, b["k_sh"], b["v_sh"], b["beta"], b["log_alpha"], cu, 1.0)
    B.mom_gdn_chunk_fwd(*args, None, h1, o1, b["ws_gdn_sh"])
    B.mom_memory_chunk_fwd(*args, B.MOM_RULE_GATED_DELTA, None, h2, o2, b["ws_gdn_sh"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(h1, h2)
