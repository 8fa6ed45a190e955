"""GPU tests of the memory-parallel layer's kernels and data flow, against
the single-GPU layer (explainer, "Memory count scaling"; paper card,
Summary):

* mom_copy_rows against torch indexing (gather, offsets, repeats) and its
  bad-index record;
* mom_proj_shared and mom_kv_proj_groups reproduce the layer's projections
  bit for bit -- one group per memory, each memory split into several
  groups, rows given pre-gathered;
* MemoryParallelMoM on a one-rank NCCL group equals MoMLayer bit for bit;
* two ranks' phases run one after the other in this process on the one GPU,
  the exchange done by slicing (no kernel waits on another rank): outputs
  and every final state equal MoMLayer on both ranks' sequences, bit for
  bit (the 380M shape at reduced length, and a skewed ragged batch).
"""
import os
import socket

import numpy as np
import pytest
import torch

from mixture_memories_layer_b200 import synth
from mixture_memories_layer_b200.mem_parallel import MemoryParallelMoM, Partition, receive_tables

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _problem(D=256, H=2, d=128, M=4, K=2, lens=(300, 77, 1, 130), seed=71, bias0=0.0, dtype="bf16",
             mem_gates=False):
    w = synth.Workload("mp", 0, 0, D, H, d, M, K, dtype, seed=seed, router_bias0=bias0, mem_gates=mem_gates)
    rng = np.random.default_rng(seed)
    p = synth.make_weights(w, rng)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    x = synth.make_tokens(w, rng, int(cu[-1]))
    return w, p, x, cu


def _layer(w, p, dt):
    from mixture_memories_layer_b200 import layer as L
    return L.MoMLayer(L.pack_weights(p, dt), w.heads, w.d_head, w.top_k)


def _local_weights(weights, part, g):
    """The replicated weights plus rank g's memories' own (w_kv and, with
    per-memory gates, w_gate_mem, A_mem, b_a_mem)."""
    own = ("w_kv", "w_gate_mem", "A_mem", "b_a_mem")
    lw = {k: v for k, v in weights.items() if k not in own}
    for k in own:
        if k in weights:
            lw[k] = weights[k][part.lo(g):part.hi(g)].contiguous()
    return lw


class _Rank:
    def __init__(self, rank, world):
        self.rank, self.world = rank, world


def test_copy_rows_gather_offsets_and_bad_index():
    from mixture_memories_layer_b200 import binding as B
    g = torch.Generator(device="cuda").manual_seed(3)
    src = torch.randint(0, 255, (37, 96), dtype=torch.uint8, device="cuda", generator=g)
    idx = torch.tensor([5, 5, 0, 36, 12, 7, 7, 7, 20], dtype=torch.int32, device="cuda")
    dst = torch.zeros((9, 160), dtype=torch.uint8, device="cuda")
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    B.mom_copy_rows(src, idx, dst, 48, src_off=32, dst_off=112, ws=ws)
    B.mom_copy_rows(src, None, dst, 64, src_off=0, dst_off=0, ws=ws, n_rows=9)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws)[0] == 0
    ref = torch.zeros_like(dst)
    ref[:, 112:160] = src[idx.long(), 32:80]
    ref[:, 0:64] = src[:9, 0:64]
    assert torch.equal(dst, ref)
    bad = idx.clone()
    bad[4] = 37
    dst.fill_(9)
    B.mom_copy_rows(src, bad, dst, 48, src_off=32, dst_off=112, ws=ws)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws) == (B.MOM_DEVERR_ROW_INDEX, 4)
    assert torch.all(dst[4, 112:160] == 0) and torch.equal(dst[3, 112:160], src[36, 32:80])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_shared_and_grouped_projections_equal_the_layers(dtype):
    from mixture_memories_layer_b200 import binding as B
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    w, p, x, cu = _problem(d=128 if dtype == "bf16" else 64, dtype=dtype)
    lay = _layer(w, p, dt)
    xt = torch.as_tensor(x).to("cuda", dt)
    b = lay.forward(xt, torch.as_tensor(cu).cuda())
    torch.cuda.synchronize()
    n, H, d, M = xt.shape[0], w.heads, w.d_head, w.n_mem
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    q, k_sh, v_sh = (torch.empty((n, H, d), dtype=dt, device="cuda") for _ in range(3))
    B.mom_proj_shared(xt, lay.w["w_shared"], H, d, q, k_sh, v_sh, ws)
    offs = b["mem_offset"]
    rows = int(offs[-1])
    kp, vp = torch.empty((rows, H, d), dtype=dt, device="cuda"), torch.empty((rows, H, d), dtype=dt, device="cuda")
    B.mom_kv_proj_groups(xt, b["perm"], offs, torch.arange(M, dtype=torch.int32, device="cuda"), lay.w["w_kv"], H, d,
                         kp, vp, ws)
    # every memory split in three groups, rows given pre-gathered
    o = offs.cpu().numpy()
    cuts = sorted(set(np.concatenate([o, o[:-1] + (o[1:] - o[:-1]) // 3, o[:-1] + 2 * (o[1:] - o[:-1]) // 3])))
    cuts = np.asarray(cuts, np.int32)
    gmem = np.searchsorted(o, cuts[:-1], side="right").astype(np.int32) - 1
    xg = xt[b["perm"][:rows].long()].contiguous()
    kp2, vp2 = torch.empty_like(kp), torch.empty_like(vp)
    B.mom_kv_proj_groups(xg, None, torch.as_tensor(cuts).cuda(), torch.as_tensor(gmem).cuda(), lay.w["w_kv"], H, d,
                         kp2, vp2, ws)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws)[0] == 0
    assert torch.equal(q, b["q"]) and torch.equal(k_sh, b["k_sh"]) and torch.equal(v_sh, b["v_sh"])
    assert torch.equal(kp, b["k_p"][:rows]) and torch.equal(vp, b["v_p"][:rows])
    assert torch.equal(kp2, b["k_p"][:rows]) and torch.equal(vp2, b["v_p"][:rows])


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_rank_nccl_group_equals_the_layer():
    import torch.distributed as dist
    from mixture_memories_layer_b200.mem_parallel import TorchComm
    w, p, x, cu = _problem()
    dt = torch.bfloat16
    lay = _layer(w, p, dt)
    xt = torch.as_tensor(x).to("cuda", dt)
    cut = torch.as_tensor(cu).cuda()
    ref = {k: v.clone() for k, v in lay.forward(xt, cut).items() if k in ("out", "h_shared", "h_mem")}
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        mp = MemoryParallelMoM(lay.w, w.heads, w.d_head, w.top_k, w.n_mem,
                               TorchComm(meta_group=dist.new_group(backend="gloo")))
        out, h_sh, h_mem, tables = mp.forward(xt, cut)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    assert torch.equal(out, ref["out"]) and torch.equal(h_sh, ref["h_shared"])
    S = len(cu) - 1
    for i in range(len(tables.seg_cu) - 1):
        m, s = int(tables.seg_mem[i]), int(tables.seg_seq[i])
        assert torch.equal(h_mem[i], ref["h_mem"][m, s])
    assert len(tables.seg_cu) - 1 == w.n_mem * S


def _emulated_ranks(w, p, x, cu, world, split):
    """Runs `world` ranks' phases in sequence; rank r gets sequences
    split[r] .. split[r+1].  Returns per-rank (out, h_shared, h_mem, tables)."""
    dt = torch.bfloat16
    lay = _layer(w, p, dt)
    part = Partition(w.n_mem, world)
    ranks = []
    for r in range(world):
        s0, s1 = split[r], split[r + 1]
        t0, t1 = int(cu[s0]), int(cu[s1])
        xr = torch.as_tensor(x[t0:t1]).to("cuda", dt)
        cur = torch.as_tensor((cu[s0:s1 + 1] - cu[s0]).astype(np.int32)).cuda()
        layer = MemoryParallelMoM(_local_weights(lay.w, part, r), w.heads, w.d_head, w.top_k, w.n_mem,
                                  _Rank(r, world))
        ranks.append((layer, layer.local_phase(xr, cur)))
    # exchange: rank r's rows for owner g start after its rows for owners < g
    starts = [np.concatenate([[0], np.cumsum(st.send_rows)]) for _, st in ranks]
    owner_out = []
    for g in range(world):
        tables = receive_tables([st.seg_out[g] for _, st in ranks], [st.n_seq for _, st in ranks], part, g)
        recv = torch.cat([st.send[starts[r][g]:starts[r][g] + st.send_rows[g]] for r, (_, st) in enumerate(ranks)])
        o, h = ranks[g][0].owner_phase(recv, tables, dt)
        owner_out.append((o, h, tables))
    res = []
    for r, (layer, st) in enumerate(ranks):
        pieces = []
        for g in range(world):
            o, _, tables = owner_out[g]
            off = int(np.sum(tables.rows[:r]))
            pieces.append(o[off:off + tables.rows[r]])
        out = layer.finish_phase(st, torch.cat(pieces))
        res.append((out, st.h_shared))
    torch.cuda.synchronize()
    return lay, res, owner_out


@pytest.mark.parametrize("case", ["mom380m_short", "skewed_ragged", "per_memory_gates"])
def test_two_emulated_ranks_equal_the_layer(case):
    if case == "per_memory_gates":
        # each owner computes its memories' gates for the rows it receives
        w, p, x, cu = _problem(M=5, lens=(300, 0, 77, 1, 130, 64), seed=74, mem_gates=True)
        split = (0, 3, 6)
    elif case == "mom380m_short":
        w0 = synth.WORKLOADS["mom380m"]
        w, p, x, cu = _problem(D=w0.d_model, H=w0.heads, d=w0.d_head, M=w0.n_mem, K=w0.top_k,
                               lens=(512,) * 8, seed=72)
        split = (0, 4, 8)
    else:
        w, p, x, cu = _problem(M=5, lens=(300, 0, 77, 1, 130, 64), seed=73, bias0=3.0)
        split = (0, 2, 6)
    lay, res, owner_out = _emulated_ranks(w, p, x, cu, 2, split)
    ref = lay.forward(torch.as_tensor(x).to("cuda", torch.bfloat16), torch.as_tensor(cu).cuda())
    torch.cuda.synchronize()
    for r in range(2):
        s0, s1 = split[r], split[r + 1]
        out, h_sh = res[r]
        assert torch.equal(out, ref["out"][int(cu[s0]):int(cu[s1])]), ("out", r)
        assert torch.equal(h_sh, ref["h_shared"][s0:s1]), ("h_shared", r)
    for g, (_, h, tables) in enumerate(owner_out):
        for i in range(len(tables.seg_cu) - 1):
            r, m, s = int(tables.seg_source[i]), int(tables.seg_mem[i]), int(tables.seg_seq[i])
            assert torch.equal(h[i], ref["h_mem"][m, split[r] + s]), ("h_mem", g, i)
