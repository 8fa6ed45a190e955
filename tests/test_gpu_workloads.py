"""Parity at full workload sizes, in the launch configuration the benchmark
times: the 380M-shape layer (8 x 2048 tokens), its skewed-routing varlen
variant, the 1.3B-shape 16-memory layer, and the 256-sequence decode.

The GPU runs the whole batch.  What the oracle checks:
* routing and the reordering on every token (cheap on the CPU), bit-exact
  outside near ties;
* projections on a seeded sample of tokens and reordered rows;
* layer outputs and final states on whole sampled sequences (sequences are
  independent, so the oracle runs one of them alone with the GPU's routing
  imposed): for the skewed varlen batch, the sequence holding memory 0's
  longest routed segment and the clipped last one; for the 1.3B shape, one
  whole 4096-token sequence (64 chunks, 16 memories).

Tokens whose k-th and (k+1)-th router logits lie within 1e-4 of each other
(near ties: rounding may flip their choice) are counted, printed and left
out of the exact index comparison; the output comparison imposes the GPU's
routing on the oracle, so they are still covered there.
"""
import numpy as np
import pytest
import torch

from mixture_memories_layer_b200 import synth
from oracle import mom_oracle as orc
from tests.gpu_helpers import TOL, max_abs_rel, run_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _routing_and_permute(w, p, res):
    idx, gate, logits, near = orc.router_topk(p["x"], p["w_r"], p["b_r"], w.top_k)
    keep = ~near
    n_near = int(near.sum())
    print("%s: %d near-tie tokens of %d excluded from the exact index check" % (w.name, n_near, w.n_tokens))
    assert np.array_equal(res["idx"][keep], idx[keep]), ("routing", w.name, "near ties excluded", n_near)
    assert max_abs_rel(res["gate"][keep], gate[keep]) < 1e-5
    perm, row_of, offs, seg = orc.permute(res["idx"], w.n_mem, p["cu_seqlens"])
    assert np.array_equal(res["perm"][:offs[-1]], perm)
    assert np.array_equal(res["row_of"], row_of)
    assert np.array_equal(res["seg_cu"], seg)
    return int(near.sum())


def _projections_sampled(w, p, res, n=256, seed=0):
    rng = np.random.default_rng(seed)
    toks = np.sort(rng.choice(w.n_tokens, n, replace=False))
    q, k_sh, v_sh, beta, la = orc.shared_projections(p["x"][toks], p, w.heads, w.d_head)
    tol = TOL[w.dtype]
    assert max_abs_rel(res["q"][toks], q) < tol
    assert max_abs_rel(res["k_sh"][toks], k_sh) < tol
    assert max_abs_rel(res["v_sh"][toks], v_sh) < tol
    assert max_abs_rel(res["beta"][toks], beta) < 1e-5
    assert max_abs_rel(res["log_alpha"][toks], la) < 1e-5
    offs = res["mem_offset"]
    rows = np.sort(rng.choice(int(offs[-1]), n, replace=False))
    mem = np.searchsorted(offs, rows, side="right") - 1
    for m in np.unique(mem):
        r = rows[mem == m]
        km, vm = orc.memory_kv(p["x"][res["perm"][r]], p, int(m), w.heads, w.d_head)
        assert max_abs_rel(res["k_p"][r], km) < tol
        assert max_abs_rel(res["v_p"][r], vm) < tol


def _sequence(w, p, res, s, max_tokens=None):
    cu = p["cu_seqlens"]
    t0, t1 = int(cu[s]), int(cu[s + 1])
    full = max_tokens is None or t1 - t0 <= max_tokens
    if not full:
        t1 = t0 + max_tokens
    ref = orc.mom_forward(p["x"][t0:t1], p, np.array([0, t1 - t0]), w.top_k, w.heads, w.d_head,
                          forced_idx=res["idx"][t0:t1])
    tol = TOL[w.dtype]
    e = max_abs_rel(res["out"][t0:t1], ref["out"])
    assert e < tol, ("out", s, e)
    if full:
        assert max_abs_rel(res["h_shared"][s], ref["h_shared"][0]) < tol
        assert max_abs_rel(res["h_mem"][:, s], ref["h_mem"][:, 0]) < tol


def test_mom380m_full_size():
    w = synth.WORKLOADS["mom380m"]
    p = synth.make_problem(w)
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    _routing_and_permute(w, p, res)
    _projections_sampled(w, p, res)
    _sequence(w, p, res, s=5)


def test_mom380m_skewed_varlen_full_size():
    w = synth.WORKLOADS["mom380m_skew_varlen"]
    p = synth.make_problem(w)
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    _routing_and_permute(w, p, res)
    # skewed routing: memory 0 carries far more rows than the others
    counts = np.diff(res["mem_offset"])
    assert counts[0] > 2 * counts[1:].max()
    _projections_sampled(w, p, res, seed=1)
    S = len(p["cu_seqlens"]) - 1
    # the sequence holding memory 0's longest routed segment (the longest
    # chain of the routed walks), with its final states, then the last
    # (clipped, shortest) sequence
    seg = res["seg_cu"]
    longest = int(np.argmax(np.diff(seg[:S + 1])))
    assert seg[longest + 1] - seg[longest] > 1000
    _sequence(w, p, res, s=longest)
    if longest != S - 1:
        _sequence(w, p, res, s=S - 1)


def test_mom1p3b_m16_full_size():
    w = synth.WORKLOADS["mom1p3b_m16"]
    p = synth.make_problem(w)
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    _routing_and_permute(w, p, res)
    _projections_sampled(w, p, res, n=128, seed=2)
    _sequence(w, p, res, s=2)          # one whole 4096-token sequence with its final states


def test_no_wait_runs_to_its_limit():
    """Every wait inside the kernels is bounded (about two seconds) and a wait
    that gives up while tearing down leaves no error record: a layer forward
    far below that bound shows that none of them ran out."""
    from mixture_memories_layer_b200 import layer as L
    w = synth.WORKLOADS["mom380m"]
    p = synth.make_problem(w)
    lay = L.MoMLayer(L.pack_weights(p, torch.bfloat16), w.heads, w.d_head, w.top_k)
    x = torch.as_tensor(p["x"]).cuda().bfloat16()
    cu = torch.as_tensor(p["cu_seqlens"]).cuda()
    lay.forward(x, cu)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(3):
        lay.forward(x, cu)
    e1.record()
    torch.cuda.synchronize()
    assert e0.elapsed_time(e1) < 200.0, e0.elapsed_time(e1)
    assert lay.device_errors() == {}


def test_decode_b256_full_size():
    """The decode workload as the benchmark runs it (256 sequences, d_model
    1024, H=4, d=256, M=8 top-2 + shared, 256-token prefill, 512 steps):
    the GPU steps the whole batch; the oracle follows 8 sequences over the
    first 16 steps and 2 sequences over all 512 (outputs and final states),
    with the GPU's routing imposed, and checks each step's routing outside
    near ties."""
    from mixture_memories_layer_b200 import layer as L
    w = synth.WORKLOADS["decode_b256"]
    steps, short_steps = w.decode_steps, 16
    short_seqs, long_seqs = [0, 37, 74, 111, 148, 185, 222, 255], [5, 200]
    p = synth.make_decode_problem(w, steps=steps)
    dt = torch.bfloat16
    lay = L.MoMLayer(L.pack_weights(p, dt), w.heads, w.d_head, w.top_k)
    b = lay.forward(torch.as_tensor(p["x_prefill"]).to("cuda", dt), torch.as_tensor(p["cu_prefill"]).to("cuda"))
    state = torch.empty((w.batch, w.n_mem + 1, w.heads, w.d_head, w.d_head), dtype=torch.float32, device="cuda")
    state[:, :w.n_mem] = b["h_mem"].permute(1, 0, 2, 3, 4)
    state[:, w.n_mem] = b["h_shared"]
    pre_idx = b["idx"].cpu().numpy()
    xs = torch.as_tensor(p["x_steps"]).to("cuda", dt)
    outs, idxs = [], []
    for s in range(steps):
        out, idx = lay.decode_step(xs[s], state)
        idxs.append(idx.cpu().numpy())
        if s < short_steps:
            outs.append(out.float().cpu().numpy())
        elif s == steps - 1:
            last_out = out.float().cpu().numpy()
    torch.cuda.synchronize()
    assert lay.device_errors() == {}
    final = state[long_seqs].cpu().numpy()
    tol = TOL[w.dtype]
    Lp = w.prefill_len
    for bsq in short_seqs + long_seqs:
        n_steps = steps if bsq in long_seqs else short_steps
        xs_pre = p["x_prefill"][bsq * Lp:(bsq + 1) * Lp]
        ref = orc.mom_forward(xs_pre, p, np.array([0, Lp]), w.top_k, w.heads, w.d_head,
                              forced_idx=pre_idx[bsq * Lp:(bsq + 1) * Lp])
        st = orc.decode_state_from_prefill(ref["h_shared"], ref["h_mem"])
        for s in range(n_steps):
            x1 = p["x_steps"][s][bsq:bsq + 1]
            nat, _, _, near = orc.router_topk(x1, p["w_r"], p["b_r"], w.top_k)
            if not near[0]:
                assert np.array_equal(idxs[s][bsq], nat[0]), ("decode routing", bsq, s)
            o_ref, st, _, _, _ = orc.mom_decode_step(x1, p, st, w.top_k, w.heads, w.d_head,
                                                     forced_idx=idxs[s][bsq:bsq + 1])
            if s < short_steps:
                e = max_abs_rel(outs[s][bsq:bsq + 1], o_ref)
                assert e < tol, ("decode out", bsq, s, e)
            elif s == steps - 1:
                e = max_abs_rel(last_out[bsq:bsq + 1], o_ref)
                assert e < tol, ("decode out, last step", bsq, e)
        if bsq in long_seqs:
            e = max_abs_rel(final[long_seqs.index(bsq)], st[0])
            assert e < tol, ("decode final state", bsq, e)
