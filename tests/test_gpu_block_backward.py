"""GPU parity of the block's reverse pass against the block oracle's
(oracle/mom_block_bwd.py, itself pinned by finite differences of the
block's forward; training is the pages' main workload: "MoM: Linear
Sequence Modeling with Mixture-of-Memories", Key points; the block's form
is a reading, the pages print none of it).

Each new C-ABI call on its own -- mom_norm_gate_bwd (top-k 0, 1, 2 and 5,
d 64 to 256, its g adjoint written into a column slice of a wider matrix),
mom_short_conv_bwd (1 to 4 taps, groups of segments, empty and one-row
segments, rows and columns outside the problem left alone, with and
without the per-head L2 norm, two problems in one call), mom_convert --
then the whole MoMBlock.backward on small ragged batches (both update
rules, with and without state adjoints) and on the 380M-shape block with
the output adjoint on one sequence.  The oracle runs with the GPU's
routing.  Error measure: max |gpu - ref| / max |ref| per gradient tensor;
the single calls within 1e-3 (float32 arithmetic on bf16 operands; 1e-2
for the bf16 do).  The whole block's gradients are sensitive to rounding
alone at about the layer's 2e-2 bar: the exact oracle, fed tokens x scaled
by 1 + u 2^-8 (u uniform in [-1, 1]: half a bf16 ulp), moves by up to
3.3e-2 (dA) on these cases, the filters' gradients (sums over a channel's
tokens only) by up to 1.8e-2.  So each block gradient is held to max(2e-2,
2 x that spread), the spread measured by the test on the same case and
routing (_tolerances); a wrong index, sign or dropped term still shows as
an O(1) error.
"""
import numpy as np
import pytest
import torch

from mixture_memories_layer_b200 import synth
from oracle import mom_block as blk
from oracle import mom_block_bwd as bbwd
from oracle import mom_oracle_bwd as lbwd
from tests.gpu_helpers import max_abs_rel, to_np

pytestmark = pytest.mark.gpu
BF = torch.bfloat16


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _bf(a):
    return torch.as_tensor(np.asarray(a, np.float32)).to("cuda", BF)


def _f32(a):
    return torch.as_tensor(np.asarray(a, np.float32)).cuda()


def _rounded(a):
    return torch.as_tensor(np.asarray(a, np.float32)).bfloat16().double().numpy()


@pytest.mark.parametrize("K,d,H", [(0, 64, 4), (1, 128, 2), (2, 256, 1), (5, 64, 2)])
def test_norm_gate_bwd(K, d, H):
    from mixture_memories_layer_b200 import binding as B
    rng = np.random.default_rng(K * 7 + d)
    n = 203
    Hd = H * d
    R = n * K
    o_sh = _rounded(rng.standard_normal((n, H, d)))
    o_p = _rounded(rng.standard_normal((max(R, 1), H, d)))
    row_of = rng.permutation(R).astype(np.int32)
    gate = rng.dirichlet(np.ones(max(K, 1)), size=n).astype(np.float32)[:, :K]
    g = _rounded(rng.standard_normal((n, H, d)) * 2)
    w_norm = rng.uniform(0.5, 1.5, d).astype(np.float32)
    dy = _rounded(rng.standard_normal((n, H, d)))
    o = o_sh.copy()
    for j in range(K):
        o += gate[:, j, None, None].astype(np.float64) * o_p[row_of.reshape(n, K)[:, j]]
    do_ref, dw_ref, dg_ref = bbwd.rms_norm_gated_bwd(o, w_norm, g, dy, blk.RMS_EPS)
    # dg into columns 8 .. 8 + Hd of a wider matrix whose other columns stay
    wide = torch.full((n, Hd + 16), float("nan"), device="cuda")
    d_o = torch.empty((n, H, d), device="cuda", dtype=BF)
    dw = torch.full((d,), float("nan"), device="cuda")
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    B.mom_norm_gate_bwd(_bf(o_sh), _bf(o_p) if K else None, torch.as_tensor(row_of).cuda() if K else None,
                        _f32(gate) if K else None, _bf(g), _f32(w_norm), blk.RMS_EPS, _bf(dy), d_o, wide[:, 8:8 + Hd],
                        dw, ws)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws)[0] == 0
    got = to_np(wide)
    assert np.isnan(got[:, :8]).all() and np.isnan(got[:, 8 + Hd:]).all()
    assert max_abs_rel(to_np(d_o), do_ref) < 1e-2
    assert max_abs_rel(got[:, 8:8 + Hd], dg_ref.reshape(n, Hd)) < 1e-3
    assert max_abs_rel(to_np(dw), dw_ref) < 1e-3


def _conv_ref(z, w_taps, seg_cu, spg, dout, H, d, l2):
    """Per segment: out = [l2norm] SiLU(conv(z)), the adjoints of z and of
    the group's filters (tap-major [G, W, C])."""
    C = z.shape[1]
    dz = np.zeros_like(z)
    dw = np.zeros(w_taps.shape)
    for s in range(len(seg_cu) - 1):
        a, b = int(seg_cu[s]), int(seg_cu[s + 1])
        if a == b:
            continue
        wg = np.swapaxes(w_taps[s // spg], 0, 1).astype(np.float64)        # [C, W]
        pre = blk.short_conv(z[a:b], wg, [(0, b - a)])
        c = blk.silu(pre)
        dc = dout[a:b]
        if l2:
            dc = lbwd.l2norm_bwd(c.reshape(b - a, H, d), dc.reshape(b - a, H, d)).reshape(b - a, C)
        da = bbwd.silu_bwd(pre, dc)
        dzs, dws = bbwd.short_conv_bwd(z[a:b], wg, [(0, b - a)], da)
        dz[a:b] = dzs
        dw[s // spg] += np.swapaxes(dws, 0, 1)
    return dz, dw


@pytest.mark.parametrize("width", [1, 2, 3, 4])
@pytest.mark.parametrize("d,l2", [(64, True), (256, True), (128, False)])
def test_short_conv_bwd_segments(width, d, l2):
    from mixture_memories_layer_b200 import binding as B
    rng = np.random.default_rng(10 * width + d + l2)
    H = 2
    C = H * d
    lens = [0, 1, 5, 64, 0, 37, 3, 90]          # 8 segments, 4 groups of 2
    lead, tail = 2, 3                            # rows outside every segment
    seg_cu = np.concatenate([[lead], lead + np.cumsum(lens)]).astype(np.int32)
    n_rows = int(seg_cu[-1]) + tail
    z = _rounded(rng.standard_normal((n_rows, C)))
    w = rng.uniform(-0.5, 0.5, size=(4, width, C)).astype(np.float32)
    dout = rng.standard_normal((n_rows, C)).astype(np.float32)
    dz = torch.full((n_rows, C + 12), float("nan"), device="cuda")
    dwt = torch.full((4, width, C), float("nan"), device="cuda")
    da = torch.empty((n_rows, C), device="cuda")
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    B.mom_short_conv_bwd([dict(z=_bf(z), dout=_f32(dout), da=da, dz=dz[:, 4:4 + C],
                               seg_cu=torch.as_tensor(seg_cu).cuda(), seg_per_group=2, w=_f32(w), dw=dwt,
                               l2norm=l2)], d, ws)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws)[0] == 0
    got = to_np(dz)
    a, b = lead, int(seg_cu[-1])
    assert np.isnan(got[:a]).all() and np.isnan(got[b:]).all()
    assert np.isnan(got[:, :4]).all() and np.isnan(got[:, 4 + C:]).all()
    dz_ref, dw_ref = _conv_ref(z, w, seg_cu, 2, dout, H, d, l2)
    assert max_abs_rel(got[a:b, 4:4 + C], dz_ref[a:b]) < 1e-3
    assert max_abs_rel(to_np(dwt), dw_ref) < 1e-3


def test_short_conv_bwd_two_problems_in_place():
    """Two problems in one call, each with its own rows, segment table, filter
    groups and norm; the second's da overwrites its own dout."""
    from mixture_memories_layer_b200 import binding as B
    rng = np.random.default_rng(4)
    H, d, W = 4, 64, 4
    C = H * d
    probs, refs = [], []
    for lens, spg, l2 in (([120, 0, 33], 3, True), ([7, 70, 1, 40], 2, False)):
        seg_cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        n = int(seg_cu[-1])
        G = (len(lens) + spg - 1) // spg
        z = _rounded(rng.standard_normal((n, C)))
        w = rng.uniform(-0.5, 0.5, size=(G, W, C)).astype(np.float32)
        dout = rng.standard_normal((n, C)).astype(np.float32)
        dout_t = _f32(dout)
        probs.append(dict(z=_bf(z), dout=dout_t, da=torch.empty_like(dout_t) if l2 else dout_t,
                          dz=torch.empty((n, C), device="cuda"), seg_cu=torch.as_tensor(seg_cu).cuda(),
                          seg_per_group=spg, w=_f32(w), dw=torch.empty((G, W, C), device="cuda"), l2norm=l2))
        refs.append(_conv_ref(z, w, seg_cu, spg, dout, H, d, l2))
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    B.mom_short_conv_bwd(probs, d, ws)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws)[0] == 0
    for q, (dz_ref, dw_ref) in zip(probs, refs):
        assert max_abs_rel(to_np(q["dz"]), dz_ref) < 1e-3
        assert max_abs_rel(to_np(q["dw"]), dw_ref) < 1e-3


def test_convert_round_trip():
    from mixture_memories_layer_b200 import binding as B
    a = torch.randn(100003, device="cuda") * 3
    h = torch.empty(100003, device="cuda", dtype=BF)
    B.mom_convert(a, h)
    back = torch.empty_like(a)
    B.mom_convert(h, back)
    torch.cuda.synchronize()
    assert torch.equal(h, a.to(BF))
    assert torch.equal(back, h.float())


# ------------------------------------------------------------ whole block --
def _problem(d, lens, H, M=4, k=2, D=256, seed=0):
    w = synth.Workload("small_block", 0, 0, D, H, d, M, k, "bf16", seed=seed, block=True)
    rng = np.random.default_rng(seed)
    p = synth.make_weights(w, rng)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    p["cu_seqlens"] = cu
    p["x"] = synth.make_tokens(w, rng, int(cu[-1]))
    return w, p


def _pairs(got, ref, H, d):
    Hd = H * d
    sw = got["dw_shared4"]
    return {
        "dx": (got["dx"], ref["dx"]), "dw_o": (got["dw_o"], ref["dw_o"]), "dw_norm": (got["dw_norm"], ref["dw_norm"]),
        "dw_q": (sw[:Hd], ref["dw_q"]), "dw_k_sh": (sw[Hd:2 * Hd], ref["dw_k_sh"]),
        "dw_v_sh": (sw[2 * Hd:3 * Hd], ref["dw_v_sh"]), "dw_g": (sw[3 * Hd:], ref["dw_g"]),
        "dw_beta": (got["dw_gate"][:H], ref["dw_beta"]), "dw_a": (got["dw_gate"][H:], ref["dw_a"]),
        "dA": (got["dA"], ref["dA"]), "db_a": (got["db_a"], ref["db_a"]),
        "dw_r": (got["dw_r"], ref["dw_r"]), "db_r": (got["db_r"], ref["db_r"]),
        "dw_k": (got["dw_kv"][:, :Hd], ref["dw_k"]), "dw_v": (got["dw_kv"][:, Hd:], ref["dw_v"]),
        "dconv_q": (got["dconv_q"][0].T, ref["dconv_q"]), "dconv_k_sh": (got["dconv_k_sh"][0].T, ref["dconv_k_sh"]),
        "dconv_v_sh": (got["dconv_v_sh"][0].T, ref["dconv_v_sh"]),
        "dconv_k": (np.swapaxes(got["dconv_k"], 1, 2), ref["dconv_k"]),
        "dconv_v": (np.swapaxes(got["dconv_v"], 1, 2), ref["dconv_v"]),
        "dh0_shared": (got["dh0_shared"], ref["dh0_shared"]), "dh0_mem": (got["dh0_mem"], ref["dh0_mem"]),
    } | ({"dw_beta_mem": (got["dw_gate_mem"][:, :H], ref["dw_beta_mem"]),
          "dw_a_mem": (got["dw_gate_mem"][:, H:], ref["dw_a_mem"]),
          "dA_mem": (got["dA_mem"], ref["dA_mem"]), "db_a_mem": (got["db_a_mem"], ref["db_a_mem"])}
         if "dw_gate_mem" in got else {})


def _run_block_bwd(w, p, rule="gated_delta", with_states=True, dy_rows=None, seqs=None):
    """The GPU block's forward and backward on p; the oracle's backward with
    the GPU's routing over the sequences ``seqs`` (all by default; dy and the
    state adjoints are zero elsewhere, so the weights' gradients are theirs
    alone).  Returns the per-tensor errors."""
    from mixture_memories_layer_b200 import block as BL
    H, d, M, K = w.heads, w.d_head, w.n_mem, w.top_k
    cu = p["cu_seqlens"]
    S = len(cu) - 1
    seqs = list(range(S)) if seqs is None else seqs
    rng = np.random.default_rng(w.seed + 100)
    n = int(cu[-1])
    dy = synth._act(rng.standard_normal((n, w.d_model)).astype(np.float32), "bf16")
    keep = np.zeros(n, bool)
    for s in seqs:
        keep[cu[s]:cu[s + 1]] = True
    dy[~keep] = 0.0
    dh_sh = dh_m = None
    if with_states:
        dh_sh = (rng.standard_normal((S, H, d, d)) * 0.1).astype(np.float32)
        dh_m = (rng.standard_normal((M, S, H, d, d)) * 0.1).astype(np.float32)
        off = [s for s in range(S) if s not in seqs]
        dh_sh[off] = 0.0
        dh_m[:, off] = 0.0
    blk_gpu = BL.MoMBlock(BL.pack_block_weights(p, BF), H, d, K, rule=rule)
    xt = torch.as_tensor(p["x"]).to("cuda", BF)
    cut = torch.as_tensor(cu).cuda()
    b = blk_gpu.forward(xt, cut)
    t = lambda a: None if a is None else torch.as_tensor(a).cuda()
    g = blk_gpu.backward(xt, cut, _bf(dy), dh_shared=t(dh_sh), dh_mem=t(dh_m))
    torch.cuda.synchronize()
    assert blk_gpu.device_errors() == {}
    got = {k: v.cpu().numpy().astype(np.float64) for k, v in g.items()}
    idx = b["idx"].cpu().numpy()
    # the oracle over the chosen sequences, packed
    rows = np.concatenate([np.arange(cu[s], cu[s + 1]) for s in seqs])
    sub_cu = np.concatenate([[0], np.cumsum([cu[s + 1] - cu[s] for s in seqs])]).astype(np.int64)
    oracle = lambda x_: bbwd.block_backward(x_, p, sub_cu, K, H, d, dy[rows], forced_idx=idx[rows],
                                            dh_shared=None if dh_sh is None else dh_sh[seqs],
                                            dh_mem=None if dh_m is None else dh_m[:, seqs], rule=rule)
    ref = oracle(p["x"][rows])
    got["dx"] = got["dx"][rows]
    got["dh0_shared"] = got["dh0_shared"][seqs]
    got["dh0_mem"] = got["dh0_mem"][:, seqs]
    errs = {k: max_abs_rel(a, r) for k, (a, r) in _pairs(got, ref, H, d).items()}
    return errs, _tolerances(oracle, p["x"][rows], ref, H, d, w.seed)


def _tolerances(oracle, x, ref, H, d, seed):
    """Per gradient: max(2e-2, 2 x the exact oracle's own change when x is
    scaled by 1 + u 2^-8, u uniform in [-1, 1])."""
    u = np.random.default_rng(seed + 200).uniform(-1.0, 1.0, x.shape)
    ref1 = oracle(np.asarray(x, np.float64) * (1.0 + u * 2.0 ** -8))
    pairs = _pairs(_as_gpu_layout(ref1), ref, H, d)
    return {k: max(2e-2, 2.0 * max_abs_rel(a, r)) for k, (a, r) in pairs.items()}


def _as_gpu_layout(r):
    """The oracle's gradients laid out as MoMBlock.backward returns them."""
    out = {k: r[k] for k in ("dx", "dw_o", "dw_norm", "dA", "db_a", "dw_r", "db_r", "dh0_shared", "dh0_mem")}
    if "dw_beta_mem" in r:
        out.update(dw_gate_mem=np.concatenate([r["dw_beta_mem"], r["dw_a_mem"]], axis=1), dA_mem=r["dA_mem"],
                   db_a_mem=r["db_a_mem"])
    out.update(dw_shared4=np.concatenate([r["dw_q"], r["dw_k_sh"], r["dw_v_sh"], r["dw_g"]]),
               dw_gate=np.concatenate([r["dw_beta"], r["dw_a"]]),
               dw_kv=np.concatenate([r["dw_k"], r["dw_v"]], axis=1),
               dconv_q=r["dconv_q"].T[None], dconv_k_sh=r["dconv_k_sh"].T[None], dconv_v_sh=r["dconv_v_sh"].T[None],
               dconv_k=np.swapaxes(r["dconv_k"], 1, 2), dconv_v=np.swapaxes(r["dconv_v"], 1, 2))
    return out


def _assert_within(res):
    errs, tol = res
    bad = {k: (e, tol[k]) for k, e in errs.items() if not e < tol[k]}
    assert not bad, (bad, errs)


@pytest.mark.parametrize("d,H,lens", [(64, 4, (190, 0, 77, 1)), (128, 2, (150, 61, 2)), (256, 1, (130, 65))])
def test_block_backward_small_ragged(d, H, lens):
    _assert_within(_run_block_bwd(*_problem(d, lens, H, seed=d + 1)))


@pytest.mark.parametrize("rule,with_states", [("gated_linear", True), ("gated_delta", False)])
def test_block_backward_other_rule_and_no_state_adjoints(rule, with_states):
    w, p = _problem(128, (120, 1, 70), 2, M=3, k=1, seed=12)
    _assert_within(_run_block_bwd(w, p, rule=rule, with_states=with_states))


def test_block_backward_per_memory_gates():
    """The block around memories with their own gates."""
    import dataclasses
    w, p = _problem(128, (150, 1, 60), 2, M=4, k=2, seed=14)
    w = dataclasses.replace(w, mem_gates=True)
    rng = np.random.default_rng(14)
    p.update({k: v for k, v in synth.make_weights(w, rng).items() if k.endswith("_mem")})
    _assert_within(_run_block_bwd(w, p))


def test_block_backward_380m_shape_one_sequence():
    """The mom380m_block workload (8 x 2048 tokens, d_model 1024, 4 heads of
    256, 4 memories top-2 + shared) through the GPU's backward, in the launch
    configuration the bench times; the output and state adjoints are
    nonzero on its third sequence alone, so that the oracle's backward of
    that sequence gives every gradient."""
    w = synth.WORKLOADS["mom380m_block"]
    p = synth.make_problem(w)
    _assert_within(_run_block_bwd(w, p, seqs=[2]))
