"""GPU parity of the block's decode step (mom_block_decode_step) and of the
windows a forward leaves (mom_block_conv_state) against the block oracle's
decode (constant-cost inference: the authors' MoM blog post, introduction
and "推理效率"; the block's form is a reading, the pages print none of it).

A prefill through MoMBlock.forward (ragged sequences, one of a single
token), its final states and windows, then several decode steps: every
step's y, and at the end every state and window, against the oracle run
from its own prefill under the GPU's routing.  Error measure as for the
block: 2e-2 max-abs-rel per tensor for the states and windows; y against
the bound carried from the 2e-2 bar through the gated RMS norm and W_o.
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


def _y_bound(p, parts, y_ref):
    """|y - y_ref| bound from a 2e-2 error of the combined output o carried
    through the per-head RMS norm and W_o (as in the block's forward test)."""
    o, g = parts["out"], parts["g"]
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + blk.RMS_EPS)
    gain = np.abs(np.asarray(p["w_norm"], np.float64) * blk.silu(g)) / rms
    b_ot = 2 * TOL["bf16"] * np.abs(o).max() * gain
    o_t = blk.rms_norm_gated(o, p["w_norm"], g)
    b_ot = b_ot + 4e-3 * np.abs(o_t).max()
    return b_ot.reshape(o.shape[0], -1) @ np.abs(np.asarray(p["w_o"], np.float64)).T + 4e-3 * np.abs(y_ref).max()


def _run(w, p, lens, steps, check_seqs, seed):
    from mixture_memories_layer_b200 import block as BL
    H, d, K, M = w.heads, w.d_head, w.top_k, w.n_mem
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    rng = np.random.default_rng(seed)
    x = synth.make_tokens(w, rng, int(cu[-1]))
    xs = [synth.make_tokens(w, rng, len(lens)) for _ in range(steps)]
    gpu = BL.MoMBlock(BL.pack_block_weights(p, BF), H, d, K)
    cu_d = torch.as_tensor(cu).cuda()
    b = gpu.forward(torch.as_tensor(x).to("cuda", BF), cu_d)
    conv_sh, conv_mem = gpu.conv_state(b, cu_d)
    S = len(lens)
    state = torch.empty((S, M + 1, H, d, d), device="cuda")
    state[:, :M] = b["h_mem"].permute(1, 0, 2, 3, 4)
    state[:, M] = b["h_shared"]
    idx_pre = b["idx"].cpu().numpy()
    ys, idxs = [], []
    for xt in xs:
        y, idx = gpu.decode_step(torch.as_tensor(xt).to("cuda", BF), state, conv_sh, conv_mem)
        ys.append(to_np(y))
        idxs.append(idx.cpu().numpy().copy())
    torch.cuda.synchronize()
    assert gpu.device_errors() == {}
    # the oracle, from its own prefill of the chosen sequences, under the GPU's routing
    sel = list(check_seqs)
    st, csh, cmem = [], [], []
    for s in sel:
        t0, t1 = int(cu[s]), int(cu[s + 1])
        r = blk.block_forward(x[t0:t1], p, np.array([0, t1 - t0]), K, H, d, forced_idx=idx_pre[t0:t1])
        st.append(orc.decode_state_from_prefill(r["h_shared"], r["h_mem"])[0])
        c = blk.block_conv_state(x[t0:t1], p, np.array([0, t1 - t0]), idx_pre[t0:t1], w.conv_width)
        csh.append(c[0][0])
        cmem.append(c[1][0])
    st, csh, cmem = np.stack(st), np.stack(csh), np.stack(cmem)
    # the windows the forward left (raw projections: bf16 on the GPU)
    Wm = w.conv_width - 1
    got_sh = to_np(gpu.conv_state(b, cu_d)[0]).reshape(S, 3, Wm, -1)[sel]
    assert max_abs_rel(got_sh, csh) < 1e-2
    for step, xt in enumerate(xs):
        y, st, csh, cmem, _, parts = blk.block_decode_step(xt[sel], p, st, csh, cmem, K, H, d,
                                                           forced_idx=idxs[step][sel])
        err = np.abs(ys[step][sel] - y)
        bound = _y_bound(p, parts, y)
        assert np.all(err <= bound), ("y", step, float((err / bound).max()))
    assert max_abs_rel(to_np(state)[sel], st) < TOL["bf16"]
    assert max_abs_rel(to_np(conv_sh).reshape(S, 3, Wm, -1)[sel], csh) < 1e-2
    # windows of memories a sequence never reached stay zero on both sides
    got_mem = to_np(conv_mem).reshape(S, M, 2, Wm, -1)[sel]
    assert max_abs_rel(got_mem, cmem) < 1e-2


def test_block_decode_small_ragged():
    w = synth.Workload("small_block", 0, 0, 256, 2, 128, 4, 2, "bf16", seed=21, block=True)
    p = synth.make_weights(w, np.random.default_rng(21))
    _run(w, p, (9, 1, 6, 40), steps=5, check_seqs=range(4), seed=22)


def test_block_decode_many_sequences_sampled():
    """256 sequences of the 380M block shape with 8 memories top-2 (the decode
    workload's), a 48-token prefill each, 4 steps; three sequences checked."""
    base = synth.WORKLOADS["decode_b256"]
    w = synth.small_workload(base, block=True, seed=23)
    p = synth.make_weights(w, np.random.default_rng(23))
    _run(w, p, (48,) * 256, steps=4, check_seqs=(0, 131, 255), seed=24)
