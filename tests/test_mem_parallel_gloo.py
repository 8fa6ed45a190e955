"""Memory-parallel layer, host side, on CPU: the partition, the send plan and
the receive tables on hand-made routings, and the whole orchestration of
MemoryParallelMoM run as gloo ranks (world sizes 2 and 3, an uneven memory
split, a rank owning no memory, empty sequences and memories) with the
kernel calls replaced by the oracle's steps -- the exchange, the tables and
the ordering are the layer's own.  Checked against the oracle layer run on
every rank's sequences at once ("MoM: Linear Sequence Modeling with
Mixture-of-Memories", Summary; explainer, "Memory count scaling").
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_memories_layer_b200 import synth
from mixture_memories_layer_b200.mem_parallel import MemoryParallelMoM, Partition, TorchComm, receive_tables, send_plan
from oracle import mom_oracle as orc


# ------------------------------------------------------------- the planning
def test_partition_blocks():
    for M in range(1, 9):
        for G in range(1, 6):
            part = Partition(M, G)
            sizes = [part.hi(g) - part.lo(g) for g in range(G)]
            assert sum(sizes) == M and max(sizes) - min(sizes) <= 1
            assert part.lo(0) == 0 and part.hi(G - 1) == M
            for m in range(M):
                g = part.owner(m)
                assert part.lo(g) <= m < part.hi(g)


def test_send_plan_and_receive_tables_by_hand():
    # M = 3 memories on 2 ranks (rank 0: 0, 1; rank 1: 2); two senders
    part = Partition(3, 2)
    # sender 0: 2 sequences; segment lengths [m][s]
    lens0 = np.array([[2, 1], [0, 3], [4, 0]])
    # sender 1: 1 sequence
    lens1 = np.array([[1], [2], [5]])
    plans = []
    for lens in (lens0, lens1):
        S = lens.shape[1]
        seg_cu = np.concatenate([[0], np.cumsum(lens.reshape(-1))])
        mem_offset = np.concatenate([[0], np.cumsum(lens.sum(1))])
        plans.append(send_plan(mem_offset, seg_cu, S, part))
    rows0, start0, seg0 = plans[0]
    assert rows0 == [6, 4] and start0 == [0, 6]
    assert list(seg0[0]) == [2, 1, 0, 3] and list(seg0[1]) == [4, 0]
    # rank 0 receives from senders 0 and 1
    t = receive_tables([plans[0][2][0], plans[1][2][0]], [2, 1], part, 0)
    assert t.rows == [6, 3]
    assert list(t.group_offset) == [0, 3, 6, 7, 9] and list(t.group_mem) == [0, 1, 0, 1]
    assert list(t.seg_cu) == [0, 2, 3, 3, 6, 7, 9]
    assert list(t.seg_source) == [0, 0, 0, 0, 1, 1] and list(t.seg_mem) == [0, 0, 1, 1, 0, 1]
    assert list(t.seg_seq) == [0, 1, 0, 1, 0, 0]
    # rank 1 owns memory 2 only
    t1 = receive_tables([plans[0][2][1], plans[1][2][1]], [2, 1], part, 1)
    assert t1.rows == [4, 5] and list(t1.group_offset) == [0, 4, 9] and list(t1.seg_cu) == [0, 4, 4, 9]


# ---------------------------------------------- the orchestration, on gloo
class OracleKernels:
    """The layer's kernel calls done by the oracle's steps on CPU tensors
    (float32 storage between steps, float64 arithmetic inside)."""

    def __init__(self, H, d):
        self.H, self.d = H, d

    def workspace(self, nbytes, device):
        return torch.zeros(256, dtype=torch.uint8)

    def router(self, x, w_r, b_r, top_k, idx, gate, stream):
        i, g, _, _ = orc.router_topk(x.numpy(), w_r.numpy(), b_r.numpy(), top_k)
        idx.copy_(torch.as_tensor(np.asarray(i, np.int32)))
        gate.copy_(torch.as_tensor(np.asarray(g, np.float32)))

    def permute_workspace_size(self, n_tok, top_k, n_mem, n_seq):
        return 256

    def permute(self, idx, n_mem, cu, perm, row_of, mem_offset, seg_cu, ws, stream):
        out = orc.permute(idx.numpy(), n_mem, cu.numpy())
        for t, v in zip((perm, row_of, mem_offset, seg_cu), out):
            t.copy_(torch.as_tensor(np.asarray(v, np.int32)))

    def proj_shared(self, x, w_shared, H, d, q, k_sh, v_sh, ws, stream):
        Hd = H * d
        w = w_shared.numpy()
        p = {"w_q": w[:Hd], "w_k_sh": w[Hd:2 * Hd], "w_v_sh": w[2 * Hd:], "w_beta": np.zeros((H, w.shape[1])),
             "w_a": np.zeros((H, w.shape[1])), "A": np.zeros(H), "b_a": np.zeros(H)}
        res = orc.shared_projections(x.numpy(), p, H, d)
        for t, v in zip((q, k_sh, v_sh), res[:3]):
            t.copy_(torch.as_tensor(np.asarray(v, np.float32)))

    def gates(self, x, w_gate, A, b_a, beta, log_alpha, ws, stream):
        H = beta.shape[1]
        xx = np.asarray(x.numpy(), np.float64)
        w = np.asarray(w_gate.numpy(), np.float64)
        b = orc.sigmoid(xx @ w[:H].T)
        la = -np.exp(np.asarray(A.numpy(), np.float64)) * orc.softplus(xx @ w[H:].T + np.asarray(b_a.numpy(), np.float64))
        beta.copy_(torch.as_tensor(b.astype(np.float32)))
        log_alpha.copy_(torch.as_tensor(la.astype(np.float32)))

    def mem_gates_groups(self, x, group_offset, group_mem, w_gate_mem, A_mem, b_a_mem, beta, log_alpha, ws, stream):
        H = beta.shape[1]
        xx = np.asarray(x.numpy(), np.float64)
        go, gm = group_offset.numpy(), group_mem.numpy()
        for g in range(len(gm)):
            a, b = int(go[g]), int(go[g + 1])
            m = int(gm[g])
            p = {"w_beta_mem": w_gate_mem.numpy()[:, :H], "w_a_mem": w_gate_mem.numpy()[:, H:],
                 "A_mem": A_mem.numpy(), "b_a_mem": b_a_mem.numpy()}
            bb, la = orc.memory_gates(xx[a:b], p, m)
            beta[a:b] = torch.as_tensor(bb.astype(np.float32))
            log_alpha[a:b] = torch.as_tensor(la.astype(np.float32))

    def copy_rows(self, src, idx, dst, row_bytes, src_off, dst_off, ws, stream):
        s = src.contiguous().view(torch.uint8).reshape(src.shape[0], -1).numpy()
        d = dst.view(torch.uint8).reshape(dst.shape[0], -1).numpy()
        rows = np.arange(d.shape[0]) if idx is None else idx.numpy()
        d[:, dst_off:dst_off + row_bytes] = s[rows, src_off:src_off + row_bytes]

    def kv_groups(self, x, group_offset, group_mem, w_kv, H, d, k_p, v_p, ws, stream):
        Hd = H * d
        w = w_kv.numpy()
        p = {"w_k": w[:, :Hd], "w_v": w[:, Hd:]}
        go, gm = group_offset.numpy(), group_mem.numpy()
        for g in range(len(gm)):
            a, b = int(go[g]), int(go[g + 1])
            if a == b:
                continue
            kk, vv = orc.memory_kv(x.numpy()[a:b], p, int(gm[g]), H, d)
            k_p[a:b] = torch.as_tensor(kk.astype(np.float32))
            v_p[a:b] = torch.as_tensor(vv.astype(np.float32))

    def recurrence(self, q, qidx, k, v, beta, log_alpha, seg_cu, scale, rule, h0, h_final, o, ws, stream):
        assert qidx is None and h0 is None
        cu = seg_cu.numpy()
        for s in range(len(cu) - 1):
            a, b = int(cu[s]), int(cu[s + 1])
            if a == b:
                h_final[s] = 0.0
                continue
            oo, S = orc.gdn_recurrence(q.numpy()[a:b], k.numpy()[a:b], v.numpy()[a:b], beta.numpy()[a:b],
                                       log_alpha.numpy()[a:b], None, scale, rule)
            o[a:b] = torch.as_tensor(oo.astype(np.float32))
            h_final[s] = torch.as_tensor(S.astype(np.float32))

    def gdn_workspace_size(self, n_rows, n_seg, H, d, dt):
        return 256

    def combine(self, o_sh, o_p, row_of, gate, out, ws, stream):
        N, K = gate.shape
        op = o_p.numpy()[row_of.numpy()].reshape(N, K, *o_p.shape[1:])
        res = o_sh.numpy().astype(np.float64) + np.einsum("nk,nkhd->nhd", gate.numpy().astype(np.float64), op)
        out.copy_(torch.as_tensor(res.astype(np.float32)))

    def rule_code(self, rule):
        return rule


def _problem(seed=61, M=5, K=2, H=2, d=8, D=32, lens=((9, 0, 13), (7, 11), (5,)), mem_gates=False):
    w = synth.Workload("mp", 0, 0, D, H, d, M, K, "f32", seed=seed, mem_gates=mem_gates)
    rng = np.random.default_rng(seed)
    p = synth.make_weights(w, rng)
    xs = [synth.make_tokens(w, rng, int(sum(l))) for l in lens]
    return w, p, xs, lens


def _pack(p, part, g):
    Hd = p["w_q"].shape[0]
    t = lambda a: torch.as_tensor(np.ascontiguousarray(np.asarray(a, np.float32)))
    lo, hi = part.lo(g), part.hi(g)
    return dict(w_r=t(p["w_r"]), b_r=t(p["b_r"]),
                w_shared=t(np.concatenate([p["w_q"], p["w_k_sh"], p["w_v_sh"]])),
                w_gate=t(np.concatenate([p["w_beta"], p["w_a"]])), A=t(p["A"]), b_a=t(p["b_a"]),
                w_kv=t(np.stack([np.concatenate([p["w_k"][m], p["w_v"][m]]) for m in range(lo, hi)])
                       if hi > lo else np.zeros((0, 2 * Hd, p["w_q"].shape[1]))),
                **({} if "w_beta_mem" not in p else dict(
                    w_gate_mem=t(np.concatenate([p["w_beta_mem"][lo:hi], p["w_a_mem"][lo:hi]], axis=1)),
                    A_mem=t(p["A_mem"][lo:hi]), b_a_mem=t(p["b_a_mem"][lo:hi]))))


def _rank_main(rank, world, port, seed, M, rule, q, mem_gates=False):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, p, xs, lens = _problem(seed=seed, M=M, lens=((9, 0, 13), (7, 11), (5,))[:world], mem_gates=mem_gates)
        part = Partition(M, world)
        layer = MemoryParallelMoM(_pack(p, part, rank), w.heads, w.d_head, w.top_k, M, TorchComm(), rule=rule,
                                  kernels=OracleKernels(w.heads, w.d_head))
        cu = torch.as_tensor(np.concatenate([[0], np.cumsum(lens[rank])]).astype(np.int32))
        out, h_sh, h_mem, tables = layer.forward(torch.as_tensor(xs[rank]), cu)
        ref = orc.mom_forward(xs[rank], p, cu.numpy(), w.top_k, w.heads, w.d_head, rule=rule)
        err_out = float(np.max(np.abs(out.numpy() - ref["out"])) / max(np.max(np.abs(ref["out"])), 1e-30))
        err_sh = float(np.max(np.abs(h_sh.numpy() - ref["h_shared"]))) if h_sh.numel() else 0.0
        # the memory states this rank owns: segments (source, memory, sequence)
        mem_refs = {}
        for r in range(world):
            cu_r = np.concatenate([[0], np.cumsum(lens[r])])
            mem_refs[r] = orc.mom_forward(xs[r], p, cu_r, w.top_k, w.heads, w.d_head, rule=rule)["h_mem"]
        err_mem = 0.0
        for i in range(len(tables.seg_cu) - 1):
            r, m, s = int(tables.seg_source[i]), int(tables.seg_mem[i]), int(tables.seg_seq[i])
            err_mem = max(err_mem, float(np.max(np.abs(h_mem[i].numpy() - mem_refs[r][m, s]))))
        q.put((rank, err_out, err_sh, err_mem, len(tables.seg_cu) - 1))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world,M,rule,mem_gates", [(2, 5, "gated_delta", False), (2, 4, "gated_linear", False),
                                                   (3, 2, "gated_delta", False), (2, 5, "gated_delta", True),
                                                   (3, 2, "gated_linear", True)])
def test_memory_parallel_forward_on_gloo_ranks(world, M, rule, mem_gates):
    """The data flow over 2 and 3 gloo ranks against the oracle, with the
    shared gates and with per-memory gates (computed by each owner for the
    rows it receives)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    mp.start_processes(_rank_main, args=(world, _free_port(), 61, M, rule, q, mem_gates), nprocs=world, join=True,
                       start_method="spawn")
    res = sorted(q.get() for _ in range(world))
    part = Partition(M, world)
    for rank, e_out, e_sh, e_mem, n_seg in res:
        assert e_out < 1e-5, (rank, e_out)
        assert e_sh < 1e-5 and e_mem < 1e-5, (rank, e_sh, e_mem)
        # one segment per (source, owned memory, source sequence)
        lens = ((9, 0, 13), (7, 11), (5,))[:world]
        assert n_seg == (part.hi(rank) - part.lo(rank)) * sum(len(l) for l in lens)
