"""Memory-parallel MoM layer: the routed memories sharded over the ranks of a
process group, each rank owning a contiguous block of memories and its
weights and states (explainer, "Memory count scaling": more memories, spread
over GPUs; paper card, Summary: each memory has its own key/value projections
and recurrent update, so a memory's work moves with it).

Per forward, on every rank r (its own sequences, as in the data-parallel
layer):

1. router, reordering, shared projections and gates, and the shared memory's
   recurrence, all local;
2. the routed rows (in the reordering's memory order, so the rows for one
   owner are contiguous) are packed as [x | q] rows by the row-copy kernel
   and sent to the owners of their memories (one all-to-all; the segment
   lengths go ahead of them in a small one);
3. the owner unpacks, computes the gates of the received rows, their key and
   value projections with the grouped GEMM over (source rank, memory)
   groups, and the recurrence over (source rank, memory, sequence) segments;
4. the output rows go back in the order they came (one all-to-all), and the
   combine runs on the source rank exactly as in the single-GPU layer.

Every step runs in the CUDA library; this module plans the exchange (split
sizes, group and segment tables -- a few integers per memory and sequence,
read on the host because the collective needs its split sizes there) and
moves the buffers with the process group's all-to-all.  With one rank the
result equals the single-GPU layer bit for bit.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch


MAX_GATE_GROUPS = 32        # mom_mem_gate_proj_groups' group limit (MOM_MAX_MEM)


# ----------------------------------------------------------------- planning
class Partition:
    """Memories [lo(g), hi(g)) of rank g: contiguous blocks whose sizes
    differ by at most one (the first M % G ranks own one more)."""

    def __init__(self, n_mem: int, world: int):
        if world < 1 or n_mem < 1:
            raise ValueError("need at least one rank and one memory")
        self.n_mem, self.world = n_mem, world
        base, extra = divmod(n_mem, world)
        sizes = [base + (1 if g < extra else 0) for g in range(world)]
        self.bounds = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int64)

    def lo(self, g: int) -> int:
        return int(self.bounds[g])

    def hi(self, g: int) -> int:
        return int(self.bounds[g + 1])

    def owned(self, g: int) -> range:
        return range(self.lo(g), self.hi(g))

    def owner(self, m: int) -> int:
        return int(np.searchsorted(self.bounds, m, side="right") - 1)


def send_plan(mem_offset: np.ndarray, seg_cu: np.ndarray, n_seq: int, part: Partition):
    """One rank's outgoing traffic from its reordering: rows[g] routed rows
    for rank g (contiguous in the reordered order, starting at start[g]) and
    seg[g] the lengths of its (memory, sequence) segments, memory-major, for
    the memories g owns."""
    mem_offset = np.asarray(mem_offset, np.int64)
    seg_cu = np.asarray(seg_cu, np.int64)
    seg_len = np.diff(seg_cu).reshape(part.n_mem, n_seq) if n_seq else np.zeros((part.n_mem, 0), np.int64)
    rows, start, seg = [], [], []
    for g in range(part.world):
        lo, hi = part.lo(g), part.hi(g)
        start.append(int(mem_offset[lo]))
        rows.append(int(mem_offset[hi] - mem_offset[lo]))
        seg.append(seg_len[lo:hi].reshape(-1).astype(np.int32))
    return rows, start, seg


@dataclass
class ReceiveTables:
    """The owner's view of what it received, rows in (source rank, memory,
    sequence, token) order: group_offset / group_mem over (source, memory)
    groups for the grouped projection, seg_cu over (source, memory,
    sequence) segments for the recurrence, rows[r] per source."""
    rows: List[int]
    group_offset: np.ndarray
    group_mem: np.ndarray
    seg_cu: np.ndarray
    seg_source: np.ndarray
    seg_mem: np.ndarray
    seg_seq: np.ndarray

    @property
    def n_rows(self) -> int:
        return int(self.group_offset[-1])


def receive_tables(seg_from: List[np.ndarray], n_seq_of: List[int], part: Partition, g: int) -> ReceiveTables:
    """Tables of rank g from the segment lengths each source sent it
    (seg_from[r]: memory-major over g's memories and r's sequences)."""
    owned = list(part.owned(g))
    offs, mems, seg_lens, s_src, s_mem, s_seq, rows = [0], [], [], [], [], [], []
    for r, lens in enumerate(seg_from):
        S = n_seq_of[r]
        lens = np.asarray(lens, np.int64).reshape(len(owned), S) if S else np.zeros((len(owned), 0), np.int64)
        rows.append(int(lens.sum()))
        for i, m in enumerate(owned):
            offs.append(offs[-1] + int(lens[i].sum()))
            mems.append(m)
            for s in range(S):
                seg_lens.append(int(lens[i, s]))
                s_src.append(r)
                s_mem.append(m)
                s_seq.append(s)
    return ReceiveTables(rows=rows,
                         group_offset=np.asarray(offs, np.int32),
                         group_mem=np.asarray(mems, np.int32),
                         seg_cu=np.concatenate([[0], np.cumsum(seg_lens, dtype=np.int64)]).astype(np.int32),
                         seg_source=np.asarray(s_src, np.int32), seg_mem=np.asarray(s_mem, np.int32),
                         seg_seq=np.asarray(s_seq, np.int32))


# ------------------------------------------------------------ communication
class TorchComm:
    """The exchanges of a memory-parallel layer over torch.distributed: the
    row buffers over `group` (NCCL for CUDA buffers), the few integers of
    metadata over `meta_group`, a CPU (gloo) group of the same ranks, so that
    reading them never waits for the GPU's queued work (None: `group`, with
    host tensors, for a CPU process group)."""

    def __init__(self, group=None, meta_group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        if meta_group is None and dist.get_backend(group) != "gloo":
            # every rank constructs its TorchComm, so this collective call is matched
            ranks = dist.get_process_group_ranks(group) if group is not None else None
            meta_group = dist.new_group(ranks=ranks, backend="gloo")
        self.meta = meta_group if meta_group is not None else group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def gather_ints(self, v: int) -> List[int]:
        t = torch.tensor([v], dtype=torch.int64)
        out = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(out, t, group=self.meta)
        return [int(o.item()) for o in out]

    def exchange_ints(self, per_dest: List[np.ndarray], in_sizes: List[int]) -> List[np.ndarray]:
        """per_dest[g] to rank g; returns what each rank sent here."""
        inp = torch.as_tensor(np.concatenate(per_dest).astype(np.int32) if per_dest else np.zeros(0, np.int32))
        out = torch.empty(sum(in_sizes), dtype=torch.int32)
        self.dist.all_to_all_single(out, inp, list(in_sizes), [len(a) for a in per_dest], group=self.meta)
        b = np.concatenate([[0], np.cumsum(in_sizes)]).astype(np.int64)
        o = out.numpy()
        return [o[b[r]:b[r + 1]] for r in range(len(in_sizes))]

    def all_to_all(self, out: torch.Tensor, inp: torch.Tensor, out_splits: List[int], in_splits: List[int]):
        self.dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)


# ------------------------------------------------------------------ kernels
class CudaKernels:
    """The CUDA library's calls the layer makes (device tensors)."""

    def __init__(self):
        from . import binding
        self.B = binding

    def workspace(self, nbytes, device):
        return self.B.new_workspace(nbytes, device)

    def router(self, x, w_r, b_r, top_k, idx, gate, stream):
        self.B.mom_router_topk(x, w_r, b_r, top_k, idx, gate, stream=stream)

    def permute(self, idx, n_mem, cu, perm, row_of, mem_offset, seg_cu, ws, stream):
        self.B.mom_permute(idx, n_mem, cu, perm, row_of, mem_offset, seg_cu, ws, stream=stream)

    def permute_workspace_size(self, n_tok, top_k, n_mem, n_seq):
        return self.B.mom_permute_workspace_size(n_tok, top_k, n_mem, n_seq)

    def proj_shared(self, x, w_shared, H, d, q, k_sh, v_sh, ws, stream):
        self.B.mom_proj_shared(x, w_shared, H, d, q, k_sh, v_sh, ws, stream=stream)

    def gates(self, x, w_gate, A, b_a, beta, log_alpha, ws, stream):
        self.B.mom_gate_proj(x, w_gate, A, b_a, beta, log_alpha, ws, stream=stream)

    def mem_gates_groups(self, x, group_offset, group_mem, w_gate_mem, A_mem, b_a_mem, beta, log_alpha, ws, stream):
        self.B.mom_mem_gate_proj_groups(x, group_offset, group_mem, w_gate_mem, A_mem, b_a_mem, beta, log_alpha, ws,
                                        stream=stream)

    def copy_rows(self, src, idx, dst, row_bytes, src_off, dst_off, ws, stream):
        self.B.mom_copy_rows(src, idx, dst, row_bytes, src_off=src_off, dst_off=dst_off, ws=ws, stream=stream)

    def kv_groups(self, x, group_offset, group_mem, w_kv, H, d, k_p, v_p, ws, stream):
        self.B.mom_kv_proj_groups(x, None, group_offset, group_mem, w_kv, H, d, k_p, v_p, ws, stream=stream)

    def recurrence(self, q, qidx, k, v, beta, log_alpha, seg_cu, scale, rule, h0, h_final, o, ws, stream):
        self.B.mom_memory_chunk_fwd(q, qidx, k, v, beta, log_alpha, seg_cu, scale, rule, h0, h_final, o, ws,
                                    stream=stream)

    def gdn_workspace_size(self, n_rows, n_seg, H, d, dt):
        return self.B.mom_gdn_workspace_size(n_rows, n_seg, H, d, self.B.dtype_code(dt))

    def combine(self, o_sh, o_p, row_of, gate, out, ws, stream):
        self.B.mom_combine_unpermute(o_sh, o_p, row_of, gate, out, ws, stream=stream)

    def rule_code(self, rule: str) -> int:
        return self.B.RULES[rule]


# -------------------------------------------------------------------- layer
@dataclass
class LocalState:
    """What one rank keeps between its sending and its combine."""
    idx: torch.Tensor
    gate: torch.Tensor
    row_of: torch.Tensor
    o_sh: torch.Tensor
    h_shared: torch.Tensor
    send: torch.Tensor
    send_rows: List[int]
    seg_out: List[np.ndarray]
    n_seq: int
    extras: dict = field(default_factory=dict)


class MemoryParallelMoM:
    """One MoM layer whose routed memories are sharded over `comm`'s ranks.

    weights: the replicated parameters (w_r, b_r, w_shared, w_gate, A, b_a
    as pack_weights lays them out) and, under "w_kv", this rank's memories
    only: [hi - lo, 2*H*d, d_model] for its block of the Partition; with
    per-memory gates also this rank's w_gate_mem [hi - lo, 2*H, d_model],
    A_mem and b_a_mem [hi - lo, H]: the owner computes the gates of the rows
    it receives with them."""

    def __init__(self, weights, heads: int, d_head: int, top_k: int, n_mem: int, comm, scale: float = 1.0,
                 rule: str = "gated_delta", kernels=None):
        self.w, self.H, self.d, self.top_k, self.n_mem = weights, heads, d_head, top_k, n_mem
        self.comm, self.scale, self.rule = comm, scale, rule
        self.k = kernels if kernels is not None else CudaKernels()
        self.part = Partition(n_mem, comm.world)
        self.rank = comm.rank
        self._ws = {}
        self._side = None
        own = self.part.hi(self.rank) - self.part.lo(self.rank)
        if weights["w_kv"].shape[0] != own:
            raise ValueError("w_kv holds %d memories; rank %d owns %d" % (weights["w_kv"].shape[0], self.rank, own))
        self.mem_gates = "w_gate_mem" in weights
        if self.mem_gates:
            for name in ("w_gate_mem", "A_mem", "b_a_mem"):
                if weights[name].shape[0] != own:
                    raise ValueError("%s holds %d memories; rank %d owns %d" % (name, weights[name].shape[0],
                                                                                self.rank, own))

    def _workspace(self, name, nbytes, device):
        """A workspace kept across calls (zeroed once, grown when needed)."""
        t = self._ws.get(name)
        if t is None or t.numel() < nbytes:
            t = self._ws[name] = self.k.workspace(nbytes, device)
        return t

    @staticmethod
    def _to_device(arr: np.ndarray, device) -> torch.Tensor:
        """A small host table on the device without waiting for the stream's
        queued work (pinned source, asynchronous copy)."""
        t = torch.as_tensor(np.ascontiguousarray(arr))
        if device.type != "cuda":
            return t
        return t.pin_memory().to(device, non_blocking=True)

    def _side_stream(self, device):
        if device.type != "cuda":
            return None
        if self._side is None:
            self._side = torch.cuda.Stream(device=device)
        return self._side

    # -- step 1 and the packing of step 2
    def local_phase(self, x: torch.Tensor, cu: torch.Tensor, stream=None) -> LocalState:
        k, w, H, d, K, M = self.k, self.w, self.H, self.d, self.top_k, self.n_mem
        dev, dt = x.device, x.dtype
        n_tok, D = x.shape
        S = cu.numel() - 1
        ws = self._workspace("local", 256, dev)
        idx = torch.empty((n_tok, K), dtype=torch.int32, device=dev)
        gate = torch.empty((n_tok, K), dtype=torch.float32, device=dev)
        k.router(x, w["w_r"], w["b_r"], K, idx, gate, stream)
        perm = torch.empty(n_tok * K, dtype=torch.int32, device=dev)
        row_of = torch.empty_like(perm)
        mem_offset = torch.empty(M + 1, dtype=torch.int32, device=dev)
        seg_cu = torch.empty(M * S + 1, dtype=torch.int32, device=dev)
        ws_perm = self._workspace("perm", k.permute_workspace_size(n_tok, K, M, S), dev)
        k.permute(idx, M, cu, perm, row_of, mem_offset, seg_cu, ws_perm, stream)
        # the split sizes go to the host as soon as they exist; the GPU goes on
        # with the projections, the gates and the packing meanwhile
        if dev.type == "cuda":
            counts = torch.empty(M + 1 + M * S + 1, dtype=torch.int32, pin_memory=True)
            cur = stream if stream is not None else torch.cuda.current_stream(dev)
            with torch.cuda.stream(cur):
                counts[:M + 1].copy_(mem_offset, non_blocking=True)
                counts[M + 1:].copy_(seg_cu, non_blocking=True)
            counted = torch.cuda.Event()
            counted.record(cur)
        else:
            counts, counted = torch.cat([mem_offset, seg_cu]), None
        q, k_sh, v_sh = (torch.empty((n_tok, H, d), dtype=dt, device=dev) for _ in range(3))
        k.proj_shared(x, w["w_shared"], H, d, q, k_sh, v_sh, ws, stream)
        beta = torch.empty((n_tok, H), dtype=torch.float32, device=dev)
        log_alpha = torch.empty_like(beta)
        k.gates(x, w["w_gate"], w["A"], w["b_a"], beta, log_alpha, ws, stream)
        o_sh = torch.empty_like(q)
        h_shared = torch.empty((S, H, d, d), dtype=torch.float32, device=dev)
        ws_gdn = self._workspace("gdn_sh", k.gdn_workspace_size(n_tok, S, H, d, dt), dev)
        # the shared memory's recurrence beside the exchange and the owners' work
        side, shared_done = self._side_stream(dev), None
        if side is not None:
            ready = torch.cuda.Event()
            ready.record(stream if stream is not None else torch.cuda.current_stream(dev))
            side.wait_event(ready)
            # the allocator must not hand these to the current stream while the side stream reads them
            for t in (q, k_sh, v_sh, beta, log_alpha, cu, o_sh, h_shared):
                t.record_stream(side)
        k.recurrence(q, None, k_sh, v_sh, beta, log_alpha, cu, self.scale, k.rule_code(self.rule), None, h_shared,
                     o_sh, ws_gdn, side if side is not None else stream)
        if side is not None:
            shared_done = torch.cuda.Event()
            shared_done.record(side)
        # pack [x | q] of every routed row in the reordered order
        xb, qb = D * x.element_size(), H * d * q.element_size()
        send = torch.empty((n_tok * K, xb + qb), dtype=torch.uint8, device=dev)
        k.copy_rows(x.view(n_tok, D), perm, send, xb, 0, 0, ws, stream)
        k.copy_rows(q.view(n_tok, H * d), perm, send, qb, 0, xb, ws, stream)
        if counted is not None:
            counted.synchronize()
        c = counts.numpy()
        send_rows, _, seg_out = send_plan(c[:M + 1], c[M + 1:], S, self.part)
        return LocalState(idx=idx, gate=gate, row_of=row_of, o_sh=o_sh, h_shared=h_shared, send=send,
                          send_rows=send_rows, seg_out=seg_out, n_seq=S,
                          extras={"ws": ws, "shared_done": shared_done})

    # -- step 3
    def owner_phase(self, recv: torch.Tensor, tables: ReceiveTables, dt: torch.dtype, stream=None):
        """Gates, key / value projections and the recurrence of the received
        rows.  Returns (o rows in received order, final states per received
        segment [n_seg, H, d, d])."""
        k, w, H, d = self.k, self.w, self.H, self.d
        dev = recv.device
        n = tables.n_rows
        esz = torch.tensor([], dtype=dt).element_size()
        D = w["w_r"].shape[1]
        xb, qb = D * esz, H * d * esz
        n_seg = len(tables.seg_cu) - 1
        o = torch.empty((n, H, d), dtype=dt, device=dev)
        h = torch.empty((n_seg, H, d, d), dtype=torch.float32, device=dev)
        if n == 0:
            if n_seg:
                h.zero_()
            return o, h
        ws = self._workspace("owner", 256, dev)
        x_r = torch.empty((n, D), dtype=dt, device=dev)
        q_r = torch.empty((n, H, d), dtype=dt, device=dev)
        k.copy_rows(recv, None, x_r.view(torch.uint8).view(n, xb), xb, 0, 0, ws, stream)
        k.copy_rows(recv, None, q_r.view(torch.uint8).view(n, qb), qb, xb, 0, ws, stream)
        beta = torch.empty((n, H), dtype=torch.float32, device=dev)
        log_alpha = torch.empty_like(beta)
        lo = self.part.lo(self.rank)
        go = self._to_device(tables.group_offset, dev)
        gm = self._to_device(tables.group_mem - lo, dev)             # index into this rank's weight blocks
        if self.mem_gates:
            # each (source, memory) group on its memory's own gates
            if len(tables.group_mem) > MAX_GATE_GROUPS:
                raise ValueError("per-memory gates take at most %d (source, memory) groups per owner, not %d"
                                 % (MAX_GATE_GROUPS, len(tables.group_mem)))
            k.mem_gates_groups(x_r, go, gm, w["w_gate_mem"], w["A_mem"], w["b_a_mem"], beta, log_alpha, ws, stream)
        else:
            k.gates(x_r, w["w_gate"], w["A"], w["b_a"], beta, log_alpha, ws, stream)
        seg = self._to_device(tables.seg_cu, dev)
        k_p = torch.empty((n, H, d), dtype=dt, device=dev)
        v_p = torch.empty_like(k_p)
        k.kv_groups(x_r, go, gm, w["w_kv"], H, d, k_p, v_p, ws, stream)
        ws_gdn = self._workspace("gdn_owner", k.gdn_workspace_size(n, n_seg, H, d, dt), dev)
        k.recurrence(q_r, None, k_p, v_p, beta, log_alpha, seg, self.scale, k.rule_code(self.rule), None, h, o,
                     ws_gdn, stream)
        return o, h

    # -- step 4
    def finish_phase(self, st: LocalState, o_back: torch.Tensor, stream=None) -> torch.Tensor:
        n_tok = st.idx.shape[0]
        out = torch.empty((n_tok, self.H, self.d), dtype=st.o_sh.dtype, device=st.o_sh.device)
        if st.extras.get("shared_done") is not None:
            (stream if stream is not None else torch.cuda.current_stream(out.device)).wait_event(st.extras["shared_done"])
        self.k.combine(st.o_sh, o_back, st.row_of, st.gate, out, st.extras["ws"], stream)
        return out

    # -- the whole layer over the process group
    def forward(self, x: torch.Tensor, cu: torch.Tensor, stream=None):
        """Returns (out [N, H, d], h_shared [S, H, d, d], h_mem of the
        segments this rank received [n_seg, H, d, d], their ReceiveTables)."""
        st = self.local_phase(x, cu, stream)
        dev, G = x.device, self.comm.world
        n_seq_of = self.comm.gather_ints(st.n_seq)
        # segment lengths from each source: len(owned(this rank)) * S_r ints
        own = self.part.hi(self.rank) - self.part.lo(self.rank)
        seg_from = self.comm.exchange_ints(st.seg_out, [own * n_seq_of[r] for r in range(G)])
        tables = receive_tables(seg_from, n_seq_of, self.part, self.rank)
        if G == 1:
            # one rank owns every memory: both exchanges are the identity
            recv = st.send
        else:
            recv = torch.empty((tables.n_rows, st.send.shape[1]), dtype=torch.uint8, device=dev)
            self.comm.all_to_all(recv, st.send, tables.rows, st.send_rows)
        o_r, h_r = self.owner_phase(recv, tables, x.dtype, stream)
        if G == 1:
            o_back = o_r
        else:
            o_back = torch.empty((st.send.shape[0], self.H, self.d), dtype=x.dtype, device=dev)
            self.comm.all_to_all(o_back, o_r, st.send_rows, tables.rows)
        return self.finish_phase(st, o_back, stream), st.h_shared, h_r, tables
