"""GPU parity of the Gated DeltaNet block around the memories against the
block oracle (oracle/mom_block.py; the authors' MoM blog post, experiments
section: every memory is a Gated DeltaNet mixer -- the block's form is a
reading, the pages print none of it).

Each C-ABI call on its own -- mom_short_conv (1 to 4 taps, groups of
segments, empty and one-row segments, rows outside every segment left
alone, with and without the per-head L2 norm), mom_combine_norm_gate
(top-k 1, 2 and 4, d 64 to 256), mom_linear (ragged rows) -- then the whole
block (MoMBlock) on small ragged batches with an empty and a one-token
sequence, and one whole sequence of the 380M-shape block with its final
states.  Error measure: max |gpu - ref| / max |ref| per tensor, 2e-2 (bf16
operands, float32 state and accumulation) for everything before the
per-head RMS norm; after it (o~, y), an element-wise bound carried from
that 2e-2 through the norm and W_o (_check_normalised): the norm rescales
every (token, head) to unit RMS, so a head whose output is small against
the sequence's largest sees its share of the combine's rounding enlarged.
"""
import numpy as np
import pytest
import torch

from mixture_memories_layer_b200 import synth
from oracle import mom_block as blk
from oracle import mom_oracle as orc
from tests.gpu_helpers import TOL, max_abs_rel, to_np

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _bf(a):
    return torch.as_tensor(np.asarray(a, np.float32)).to("cuda", BF)


def _rounded(a):
    return torch.as_tensor(np.asarray(a, np.float32)).bfloat16().double().numpy()


@pytest.mark.parametrize("width", [1, 2, 3, 4])
@pytest.mark.parametrize("d,l2", [(64, True), (128, True), (256, True), (128, False)])
def test_short_conv_segments(width, d, l2):
    from mixture_memories_layer_b200 import binding as B
    rng = np.random.default_rng(10 * width + d + l2)
    H = 2
    C = H * d
    lens = [0, 1, 5, 64, 0, 37, 3, 90]          # 8 segments, 4 groups of 2
    lead, tail = 2, 3                            # rows outside every segment
    seg_cu = np.concatenate([[lead], lead + np.cumsum(lens)]).astype(np.int32)
    n_rows = int(seg_cu[-1]) + tail
    z = _rounded(rng.standard_normal((n_rows, C)))
    w = rng.uniform(-0.5, 0.5, size=(4, C, width)).astype(np.float32)
    out = torch.full((n_rows, C), float("nan"), device="cuda", dtype=BF)
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    w_taps = torch.as_tensor(np.ascontiguousarray(np.swapaxes(w, 1, 2))).cuda()     # [groups, width, C]
    B.mom_short_conv(_bf(z), torch.as_tensor(seg_cu).cuda(), w_taps, out, ws, seg_per_group=2, head_dim=d, l2norm=l2)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws)[0] == 0
    got = to_np(out)
    assert np.isnan(got[:lead]).all() and np.isnan(got[int(seg_cu[-1]):]).all()
    for s in range(len(lens)):
        a, b = int(seg_cu[s]), int(seg_cu[s + 1])
        if a == b:
            continue
        ref = blk.silu(blk.short_conv(z[a:b], w[s // 2], [(0, b - a)]))
        if l2:
            ref = orc.l2norm(ref.reshape(b - a, H, d)).reshape(b - a, C)
        e = max_abs_rel(got[a:b], ref)
        assert e < 1e-2, (s, e)


def test_short_conv_batch_of_problems():
    """Three convolutions in one launch: different row counts, segment tables,
    filter groups and norms, each against its own oracle."""
    from mixture_memories_layer_b200 import binding as B
    rng = np.random.default_rng(11)
    d, H, width = 128, 2, 4
    C = H * d
    cases = [((0, 70, 1, 0, 9), 1, True), ((200,), 1, False), ((3, 0, 64, 65, 2, 17), 3, True)]
    probs, refs = [], []
    for lens, spg, l2 in cases:
        seg_cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        n = int(seg_cu[-1])
        n_groups = -(-len(lens) // spg)
        z = _rounded(rng.standard_normal((n, C)))
        w = rng.uniform(-0.5, 0.5, size=(n_groups, C, width)).astype(np.float32)
        out = torch.full((n, C), float("nan"), device="cuda", dtype=BF)
        w_taps = torch.as_tensor(np.ascontiguousarray(np.swapaxes(w, 1, 2))).cuda()
        probs.append(dict(z=_bf(z), out=out, seg_cu=torch.as_tensor(seg_cu).cuda(), w=w_taps,
                          seg_per_group=spg, l2norm=l2))
        ref = np.zeros((n, C))
        for s_ in range(len(lens)):
            a, b = int(seg_cu[s_]), int(seg_cu[s_ + 1])
            if a < b:
                r = blk.silu(blk.short_conv(z[a:b], w[s_ // spg], [(0, b - a)]))
                ref[a:b] = orc.l2norm(r.reshape(b - a, H, d)).reshape(b - a, C) if l2 else r
        refs.append(ref)
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    B.mom_short_conv_batch(probs, d, ws)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws)[0] == 0
    for q, ref in zip(probs, refs):
        assert max_abs_rel(to_np(q["out"]), ref) < 1e-2


@pytest.mark.parametrize("K", [1, 2, 4])
@pytest.mark.parametrize("d", [64, 128, 256])
def test_combine_norm_gate(K, d):
    from mixture_memories_layer_b200 import binding as B
    rng = np.random.default_rng(K * 1000 + d)
    H = 512 // d
    n = 150
    o_sh = _rounded(rng.standard_normal((n, H, d)))
    o_p = _rounded(rng.standard_normal((n * K, H, d)) * 2)
    g = _rounded(rng.standard_normal((n, H, d)) * 2)
    gate = rng.dirichlet(np.ones(K), size=n).astype(np.float32)
    row_of = rng.permutation(n * K).astype(np.int32)
    w_norm = rng.uniform(0.5, 1.5, size=d).astype(np.float32)
    out = torch.empty((n, H, d), device="cuda", dtype=BF)
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    B.mom_combine_norm_gate(_bf(o_sh), _bf(o_p), torch.as_tensor(row_of).cuda(), torch.as_tensor(gate).cuda(),
                            _bf(g), torch.as_tensor(w_norm).cuda(), 1e-5, out, ws)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws)[0] == 0
    o = o_sh + np.einsum("nj,njhd->nhd", gate.astype(np.float64), o_p[row_of.reshape(n, K)])
    ref = blk.rms_norm_gated(o, w_norm, g, 1e-5)
    assert max_abs_rel(to_np(out), ref) < 1e-2


def test_linear_ragged_rows():
    from mixture_memories_layer_b200 import binding as B
    rng = np.random.default_rng(7)
    n, k_in, n_out = 300, 192, 512
    x = _rounded(rng.standard_normal((n, k_in)))
    w = _rounded(rng.standard_normal((n_out, k_in)) / np.sqrt(k_in))
    y = torch.empty((n, n_out), device="cuda", dtype=BF)
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    B.mom_linear(_bf(x), _bf(w), y, ws)
    torch.cuda.synchronize()
    assert max_abs_rel(to_np(y), x @ w.T) < 1e-2


def _block_problem(d, lens, H, M=4, k=2, D=256, seed=0, bias0=0.0):
    w = synth.Workload("small_block", 0, 0, D, H, d, M, k, "bf16", seed=seed, router_bias0=bias0, block=True)
    rng = np.random.default_rng(seed)
    p = synth.make_weights(w, rng)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    p["cu_seqlens"] = cu
    p["x"] = synth.make_tokens(w, rng, int(cu[-1]))
    return w, p


def run_block(w, p):
    from mixture_memories_layer_b200 import block as BL
    blk_gpu = BL.MoMBlock(BL.pack_block_weights(p, BF), w.heads, w.d_head, w.top_k)
    x = torch.as_tensor(p["x"]).to("cuda", BF)
    cu = torch.as_tensor(p["cu_seqlens"]).to("cuda", torch.int32)
    b = blk_gpu.forward(x, cu)
    torch.cuda.synchronize()
    res = {k: (to_np(v) if v.dtype != torch.int32 else v.cpu().numpy()) for k, v in b.items()
           if not k.startswith("ws")}
    return blk_gpu, res


def _check_normalised(p, ref, res, tag):
    """o~ and y against a bound derived from the layer's bar: the combined
    output o is held to 2e-2 of its maximum (absolute error e = 2e-2 max|o|);
    the per-head RMS norm maps that to at most 2 e / rms(o[t, h]) |w_norm
    SiLU(g)| per element of o~ (the numerator's error and the RMS's), plus the
    bf16 roundings of g and o~ (4e-3 of max|o~|); W_o carries it to y by
    |W_o| (plus 4e-3 of max|y| for y's own rounding).  ref: whole-batch
    tensors out, g, o_tilde, y."""
    o = ref["out"]
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + blk.RMS_EPS)
    gain = np.abs(np.asarray(p["w_norm"], np.float64) * blk.silu(ref["g"])) / rms
    b_ot = 2 * TOL["bf16"] * np.abs(o).max() * gain + 4e-3 * np.abs(ref["o_tilde"]).max()
    err_ot = np.abs(res["o_tilde"] - ref["o_tilde"])
    assert np.all(err_ot <= b_ot), (tag, "o_tilde", float((err_ot / b_ot).max()))
    n = o.shape[0]
    b_y = b_ot.reshape(n, -1) @ np.abs(np.asarray(p["w_o"], np.float64)).T + 4e-3 * np.abs(ref["y"]).max()
    err_y = np.abs(res["y"] - ref["y"])
    assert np.all(err_y <= b_y), (tag, "y", float((err_y / b_y).max()))


def _block_refs(w, p, res, seqs, rule="gated_delta"):
    """The oracle's block run per sequence (under the GPU's routing) and laid
    out as the GPU's tensors over the chosen sequences: per-token tensors
    concatenated, the routed rows in the GPU's row order."""
    cu = p["cu_seqlens"]
    K = w.top_k
    keys = ("q", "k_sh", "v_sh", "o_shared", "out", "g", "o_tilde", "y")
    ref = {k: [] for k in keys}
    got = {k: [] for k in ("q", "k_sh", "v_sh", "o_sh", "o_tilde", "y", "k_p", "v_p", "o_p")}
    ref.update(k_mem=[], v_mem=[], o_mem=[], states=[])
    for s in seqs:
        t0, t1 = int(cu[s]), int(cu[s + 1])
        if t0 == t1:
            assert not np.any(res["h_shared"][s]) and not np.any(res["h_mem"][:, s])
            continue
        r = blk.block_forward(p["x"][t0:t1], p, np.array([0, t1 - t0]), K, w.heads, w.d_head,
                              forced_idx=res["idx"][t0:t1], rule=rule)
        keep = ~r["near_tie"]
        nat = orc.router_topk(p["x"][t0:t1], p["w_r"], p["b_r"], K)[0]
        assert np.array_equal(res["idx"][t0:t1][keep], nat[keep]), "router indices differ"
        for k in keys:
            ref[k].append(r[k])
        rows = res["row_of"][t0 * K:t1 * K].reshape(t1 - t0, K)
        for k in ("k_mem", "v_mem", "o_mem"):
            ref[k].append(r[k])
        for k in ("q", "k_sh", "v_sh", "o_sh", "o_tilde", "y"):
            got[k].append(res[k][t0:t1])
        for k in ("k_p", "v_p", "o_p"):
            got[k].append(res[k][rows])
        ref["states"].append((s, r["h_shared"][0], r["h_mem"][:, 0]))
    cat = lambda xs: np.concatenate(xs, axis=0)
    return ({k: (cat(v) if k != "states" else v) for k, v in ref.items()}, {k: cat(v) for k, v in got.items()})


def _check_block(w, p, res, seqs=None, rule="gated_delta"):
    """Whole-tensor errors (the acceptance measure: max-abs-rel per output
    tensor) over the chosen sequences."""
    tol = TOL["bf16"]
    seqs = range(len(p["cu_seqlens"]) - 1) if seqs is None else seqs
    ref, got = _block_refs(w, p, res, seqs, rule)
    for key, mine in (("q", "q"), ("k_sh", "k_sh"), ("v_sh", "v_sh"), ("o_sh", "o_shared"), ("k_p", "k_mem"),
                      ("v_p", "v_mem"), ("o_p", "o_mem")):
        e = max_abs_rel(got[key], ref[mine])
        assert e < tol, (key, e)
    _check_normalised(p, ref, got, "block")
    hs = np.stack([h for _, h, _ in ref["states"]])
    hm = np.stack([m for _, _, m in ref["states"]], axis=1)
    idx = [s for s, _, _ in ref["states"]]
    e_hs = max_abs_rel(res["h_shared"][idx], hs)
    e_hm = max_abs_rel(res["h_mem"][:, idx], hm)
    assert e_hs < tol and e_hm < tol, ("states", e_hs, e_hm)


@pytest.mark.parametrize("rule,mem_gates", [("gated_linear", False), ("gated_delta", True)])
def test_block_other_rule_and_per_memory_gates(rule, mem_gates):
    """The block around memories with the scalar-gated linear rule, and around
    memories with their own gates."""
    import dataclasses
    from mixture_memories_layer_b200 import block as BL
    w, p = _block_problem(128, (150, 1, 70), 2, seed=9)
    if mem_gates:
        w = dataclasses.replace(w, mem_gates=True)
        rng = np.random.default_rng(9)
        p.update({k: v for k, v in synth.make_weights(w, rng).items() if k.endswith("_mem")})
    blk_gpu = BL.MoMBlock(BL.pack_block_weights(p, BF), w.heads, w.d_head, w.top_k, rule=rule)
    b = blk_gpu.forward(torch.as_tensor(p["x"]).to("cuda", BF), torch.as_tensor(p["cu_seqlens"]).cuda())
    torch.cuda.synchronize()
    assert blk_gpu.device_errors() == {}
    res = {k: (to_np(v) if v.dtype != torch.int32 else v.cpu().numpy()) for k, v in b.items() if not k.startswith("ws")}
    _check_block(w, p, res, rule=rule)


@pytest.mark.parametrize("d,H", [(64, 4), (128, 2), (256, 1)])
def test_block_small_ragged(d, H):
    w, p = _block_problem(d, (190, 0, 77, 1), H, seed=d)
    b, res = run_block(w, p)
    assert b.device_errors() == {}
    _check_block(w, p, res)


def test_block_skewed_routing_top1_of_2():
    w, p = _block_problem(128, (140, 65), 2, M=2, k=1, seed=5, bias0=2.0)
    b, res = run_block(w, p)
    assert b.device_errors() == {}
    _check_block(w, p, res)


def test_block_380m_shape_one_sequence_with_states():
    """The mom380m_block workload (8 x 2048 tokens, d_model 1024, 4 heads of
    256, 4 memories top-2 + shared) on the GPU; the oracle checks the whole
    of its third sequence: y, the gated norm, the convolved q, k, v and the
    final states of every memory."""
    w = synth.WORKLOADS["mom380m_block"]
    p = synth.make_problem(w)
    b, res = run_block(w, p)
    assert b.device_errors() == {}
    _check_block(w, p, res, seqs=[2])
