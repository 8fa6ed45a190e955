"""GPU parity of mom_gdn_chunk_fwd called directly (edge cases of the
segment list) and of mom_decode_step against the oracle's Gated DeltaNet
token loop and decode step (constant-cost inference: the authors' MoM blog
post, introduction; "MoM: Linear Sequence Modeling with Mixture-of-Memories",
Summary), plus the device error record on bad indices.
"""
import numpy as np
import pytest
import torch

from mixture_memories_layer_b200 import binding as B
from mixture_memories_layer_b200 import synth
from oracle import mom_oracle as orc
from tests.gpu_helpers import TOL, max_abs_rel, run_layer, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _gdn_inputs(rng, n_rows, n_q, H, d, strong_decay=True):
    q = orc.l2norm(rng.standard_normal((n_q, H, d)))
    k = orc.l2norm(rng.standard_normal((n_rows, H, d)))
    v = rng.standard_normal((n_rows, H, d))
    beta = 1 / (1 + np.exp(-rng.standard_normal((n_q, H))))
    la = -np.exp(rng.uniform(0, 2.7, (n_q, H))) * np.logaddexp(0, rng.standard_normal((n_q, H)) + rng.uniform(-4, 0, (n_q, H)))
    if strong_decay:
        la[::7] = -20.0
    return q, k, v, beta, la


@pytest.mark.parametrize("dt", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 256])
def test_gdn_segments_edge_cases(dt, d):
    """Empty segments, length-1 segments, ragged lengths (not multiples of
    64), an initial state, and a row -> query index map."""
    rng = np.random.default_rng(d)
    H = 2
    seg_lens = [0, 1, 65, 130, 0, 64, 7]
    seg_cu = np.concatenate([[0], np.cumsum(seg_lens)]).astype(np.int32)
    n_rows = int(seg_cu[-1])
    n_q = n_rows + 5
    q, k, v, beta, la = _gdn_inputs(rng, n_rows, n_q, H, d)
    qidx = rng.permutation(n_q)[:n_rows].astype(np.int32)
    h0 = rng.standard_normal((len(seg_lens), H, d, d)) * 0.1
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    # the kernels read bf16 values: give the oracle the same rounded inputs
    rnd = (lambda a: synth.bf16_round(a)) if dt == "bf16" else (lambda a: a.astype(np.float32))
    q, k, v = rnd(q), rnd(k), rnd(v)
    beta, la, h0 = (a.astype(np.float32).astype(np.float64) for a in (beta, la, h0))
    g = lambda a, t=tdt: torch.as_tensor(np.ascontiguousarray(a)).to("cuda", t)
    o = torch.zeros((n_rows, H, d), dtype=tdt, device="cuda")
    hf = torch.zeros((len(seg_lens), H, d, d), dtype=torch.float32, device="cuda")
    ws = B.new_workspace(B.mom_gdn_workspace_size(n_rows, len(seg_lens), H, d, B.dtype_code(tdt)))
    B.mom_gdn_chunk_fwd(g(q), g(qidx, torch.int32), g(k), g(v), g(beta, torch.float32), g(la, torch.float32),
                        g(seg_cu, torch.int32), 0.8, g(h0, torch.float32), hf, o, ws)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws) == (0, 0)
    o, hf = to_np(o), to_np(hf)
    tol = TOL[dt]
    for s, L in enumerate(seg_lens):
        a, b = seg_cu[s], seg_cu[s + 1]
        rq = qidx[a:b]
        ro, rS = orc.gdn_recurrence(q[rq], k[a:b], v[a:b], beta[rq], la[rq], h0[s], scale=0.8)
        assert max_abs_rel(hf[s], rS) < tol, ("state", s, L)
        if L:
            assert max_abs_rel(o[a:b], ro) < tol, ("o", s, L)


@pytest.mark.parametrize("d", [128, 256])
def test_gdn_prep_then_state_equals_fwd(d):
    """mom_gdn_chunk_prep followed by mom_gdn_chunk_state (here on two
    streams ordered by an event, with another problem's prep in between)
    writes exactly what mom_gdn_chunk_fwd writes."""
    rng = np.random.default_rng(5 + d)
    H = 2
    seg_lens = [130, 0, 64, 200, 3]
    seg_cu = np.concatenate([[0], np.cumsum(seg_lens)]).astype(np.int32)
    n_rows = int(seg_cu[-1])
    q, k, v, beta, la = _gdn_inputs(rng, n_rows, n_rows, H, d)
    h0 = rng.standard_normal((len(seg_lens), H, d, d)) * 0.1
    g = lambda a, t=torch.bfloat16: torch.as_tensor(np.ascontiguousarray(a)).to("cuda", t)
    args = [g(q), None, g(k), g(v), g(beta, torch.float32), g(la, torch.float32), g(seg_cu, torch.int32), 1.0,
            g(h0, torch.float32)]
    code = B.dtype_code(torch.bfloat16)
    outs = []
    for split in (False, True):
        o = torch.zeros((n_rows, H, d), dtype=torch.bfloat16, device="cuda")
        hf = torch.zeros((len(seg_lens), H, d, d), dtype=torch.float32, device="cuda")
        ws = B.new_workspace(B.mom_gdn_workspace_size(n_rows, len(seg_lens), H, d, code))
        if split:
            other_o = torch.zeros_like(o)
            other_ws = B.new_workspace(B.mom_gdn_workspace_size(n_rows, len(seg_lens), H, d, code))
            B.mom_gdn_chunk_prep(*args, hf, o, ws)
            B.mom_gdn_chunk_prep(*args[:8], None, None, other_o, other_ws)
            side = torch.cuda.Stream()
            ev = torch.cuda.Event()
            ev.record(torch.cuda.current_stream())
            side.wait_event(ev)
            B.mom_gdn_chunk_state(*args, hf, o, ws, stream=side)
            B.mom_gdn_chunk_state(*args[:8], None, None, other_o, other_ws)
            torch.cuda.synchronize()
        else:
            B.mom_gdn_chunk_fwd(*args, hf, o, ws)
            torch.cuda.synchronize()
        assert B.mom_get_error(ws) == (0, 0)
        outs.append((to_np(o), to_np(hf)))
    assert np.array_equal(outs[0][0], outs[1][0])
    assert np.array_equal(outs[0][1], outs[1][1])


def test_device_error_record_on_bad_memory_index():
    """A memory index >= M is recorded and dropped, never read out of bounds."""
    n_tok, K, M = 300, 2, 4
    idx = torch.randint(0, M, (n_tok, K), dtype=torch.int32, device="cuda")
    idx[:, 1] = (idx[:, 0] + 1) % M
    idx[123, 1] = 9
    cu = torch.tensor([0, n_tok], dtype=torch.int32, device="cuda")
    perm = torch.full((n_tok * K,), -7, dtype=torch.int32, device="cuda")
    row_of = torch.empty(n_tok * K, dtype=torch.int32, device="cuda")
    offs = torch.empty(M + 1, dtype=torch.int32, device="cuda")
    seg = torch.empty(M + 1, dtype=torch.int32, device="cuda")
    ws = B.new_workspace(B.mom_permute_workspace_size(n_tok, K, M, 1))
    B.mom_permute(idx, M, cu, perm, row_of, offs, seg, ws)
    code, info = B.mom_get_error(ws)
    assert code == B.MOM_DEVERR_MEM_INDEX and info == 123
    assert int(offs[-1]) == n_tok * K - 1
    assert int(row_of[123 * K + 1]) == -1
    B.mom_clear_error(ws)
    assert B.mom_get_error(ws) == (0, 0)


def _decode_case(w, steps, check_seqs, prefill_len):
    """GPU: prefill forward -> decode layout -> `steps` decode steps.
    Oracle: the same for the sequences in check_seqs, routing imposed."""
    from mixture_memories_layer_b200 import layer as L
    p = synth.make_decode_problem(w, steps=steps)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    lay = L.MoMLayer(L.pack_weights(p, dt), w.heads, w.d_head, w.top_k)
    xg = torch.as_tensor(p["x_prefill"]).to("cuda", dt)
    cu = torch.as_tensor(p["cu_prefill"]).to("cuda")
    b = lay.forward(xg, cu)
    state = torch.empty((w.batch, w.n_mem + 1, w.heads, w.d_head, w.d_head), dtype=torch.float32, device="cuda")
    state[:, :w.n_mem] = b["h_mem"].permute(1, 0, 2, 3, 4)
    state[:, w.n_mem] = b["h_shared"]
    pre_idx = b["idx"].cpu().numpy()
    outs, idxs = [], []
    for s in range(steps):
        out, idx = lay.decode_step(torch.as_tensor(p["x_steps"][s]).to("cuda", dt), state)
        outs.append(to_np(out))
        idxs.append(idx.cpu().numpy())
    torch.cuda.synchronize()
    assert lay.device_errors() == {}
    final = state.cpu().numpy()
    tol = TOL[w.dtype]
    Lp = prefill_len
    for bsq in check_seqs:
        xs = p["x_prefill"][bsq * Lp:(bsq + 1) * Lp]
        ref = orc.mom_forward(xs, p, np.array([0, Lp]), w.top_k, w.heads, w.d_head,
                              forced_idx=pre_idx[bsq * Lp:(bsq + 1) * Lp])
        st = orc.decode_state_from_prefill(ref["h_shared"], ref["h_mem"])
        for s in range(steps):
            o_ref, st, _, _, _ = orc.mom_decode_step(p["x_steps"][s][bsq:bsq + 1], p, st, w.top_k, w.heads,
                                                     w.d_head, forced_idx=idxs[s][bsq:bsq + 1])
            e = max_abs_rel(outs[s][bsq:bsq + 1], o_ref)
            assert e < tol, ("decode out", bsq, s, e)
        assert max_abs_rel(final[bsq:bsq + 1], st) < tol


@pytest.mark.parametrize("d,dtype", [(64, "f32"), (256, "bf16")])
def test_decode_small(d, dtype):
    w = synth.Workload("dec_small", 16, 0, 256, 2, d, 8, 2, dtype, seed=9, decode_steps=3, prefill_len=40)
    _decode_case(w, steps=3, check_seqs=range(16), prefill_len=40)


def test_decode_one_sequence_every_memory():
    # a batch of one, top-k = M: the step updates all M + 1 states of the sequence
    w = synth.Workload("dec_one", 1, 0, 256, 2, 64, 4, 4, "f32", seed=11, decode_steps=2, prefill_len=8)
    _decode_case(w, steps=2, check_seqs=range(1), prefill_len=8)


def test_decode_empty_batch():
    from mixture_memories_layer_b200 import layer as L
    w = synth.Workload("dec_empty", 4, 0, 256, 2, 64, 4, 2, "bf16", seed=3, decode_steps=1, prefill_len=8)
    p = synth.make_decode_problem(w, steps=1)
    lay = L.MoMLayer(L.pack_weights(p, torch.bfloat16), w.heads, w.d_head, w.top_k)
    x = torch.empty((0, w.d_model), dtype=torch.bfloat16, device="cuda")
    state = torch.empty((0, w.n_mem + 1, w.heads, w.d_head, w.d_head), dtype=torch.float32, device="cuda")
    out, idx = lay.decode_step(x, state)
    torch.cuda.synchronize()
    assert tuple(out.shape) == (0, w.heads, w.d_head) and tuple(idx.shape) == (0, w.top_k)
    assert lay.device_errors() == {}
