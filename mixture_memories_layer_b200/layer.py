"""One MoM layer on the GPU: the six C-ABI calls in order, with torch used
only to hold device memory.

    router -> permute -> projections -> GDN prep (shared, routed)
           -> GDN state walks (shared | routed, two streams) -> combine

("MoM: Linear Sequence Modeling with Mixture-of-Memories", Summary; "MoM:
Mixture-of-Memories Fixes Linear Attention Recall", Router mechanics and
Solving scatter-gather without new kernels.)  Every step runs in the CUDA
library; this module packs weights, allocates outputs and workspaces once
per shape, and passes pointers.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import binding as B


def pack_weights(p: Dict[str, np.ndarray], dtype: torch.dtype, device="cuda") -> Dict[str, torch.Tensor]:
    """Stack the per-projection weights into the layouts the library reads:
    w_shared = [W_q; W_k_sh; W_v_sh], w_gate = [W_beta; W_a],
    w_kv[m] = [W_k^m; W_v^m] (all [out, in]); with per-memory gates also
    w_gate_mem[m] = [W_beta^m; W_a^m], A_mem, b_a_mem [M, H]."""
    t = lambda a, dt=dtype: torch.as_tensor(np.ascontiguousarray(a)).to(device=device, dtype=dt)
    M = p["w_k"].shape[0]
    mem_gates = {}
    if "w_beta_mem" in p:
        mem_gates = dict(
            w_gate_mem=t(np.stack([np.concatenate([p["w_beta_mem"][m], p["w_a_mem"][m]], axis=0) for m in range(M)])),
            A_mem=t(p["A_mem"], torch.float32),
            b_a_mem=t(p["b_a_mem"], torch.float32),
        )
    return dict(**mem_gates,
        w_r=t(p["w_r"]),
        b_r=t(p["b_r"], torch.float32),
        w_shared=t(np.concatenate([p["w_q"], p["w_k_sh"], p["w_v_sh"]], axis=0)),
        w_gate=t(np.concatenate([p["w_beta"], p["w_a"]], axis=0)),
        A=t(p["A"], torch.float32),
        b_a=t(p["b_a"], torch.float32),
        w_kv=t(np.stack([np.concatenate([p["w_k"][m], p["w_v"][m]], axis=0) for m in range(M)])),
    )


class MoMLayer:
    """Holds packed weights and reusable buffers for one layer shape."""

    def __init__(self, weights: Dict[str, torch.Tensor], heads: int, d_head: int, top_k: int,
                 scale: float = 1.0, gdn_schedule: str = "streams", rule: str = "gated_delta"):
        """gdn_schedule: "streams" (each problem's GDN prep and walk on its own
        stream, the shared memory's on a high-priority one) or "phased" (both
        problems' prep on the whole GPU, then both walks).  Measured on B200:
        380M-shape layer 0.295 vs 0.308 ms, 1.3B-shape layer 0.904 vs
        0.963 ms.  rule: the memories' update rule, "gated_delta" (Gated
        DeltaNet, the default) or "gated_linear" (S_t = alpha_t S_{t-1} +
        beta_t v_t k_t^T: linear attention, RetNet, Mamba2-style memories).
        Weights that carry w_gate_mem / A_mem / b_a_mem (pack_weights of
        per-memory gates) give every routed memory its own beta and alpha."""
        if rule not in B.RULES:
            raise ValueError("rule must be one of %s" % sorted(B.RULES))
        self.rule = B.RULES[rule]
        self.w = weights
        self.H, self.d, self.top_k, self.scale = heads, d_head, top_k, scale
        if gdn_schedule not in ("phased", "streams"):
            raise ValueError("gdn_schedule must be 'phased' or 'streams'")
        self.gdn_schedule = gdn_schedule
        self.n_mem, self.d_model = weights["w_r"].shape
        self.dtype = weights["w_r"].dtype
        self.device = weights["w_r"].device
        self._bufs = {}
        self._c_weights = B.MomWeights(*[ctypes_ptr(weights[k]) for k in
                                         ("w_r", "b_r", "w_shared", "w_gate", "A", "b_a", "w_kv")])
        self.mem_gates = "w_gate_mem" in weights
        self._c_mem_gates = (B.MomMemoryGates(*[ctypes_ptr(weights[k]) for k in ("w_gate_mem", "A_mem", "b_a_mem")])
                             if self.mem_gates else None)

    # -------------------------------------------------------------- buffers
    def _buf(self, name, shape, dtype):
        key = (name, tuple(shape), dtype)
        t = self._bufs.get(key)
        if t is None:
            t = torch.empty(shape, dtype=dtype, device=self.device)
            self._bufs[key] = t
        return t

    def _ws(self, name, nbytes):
        key = ("ws", name)
        t = self._bufs.get(key)
        if t is None or t.numel() < nbytes:
            t = B.new_workspace(nbytes, self.device)
            self._bufs[key] = t
        return t

    def buffers(self, n_tok: int, n_seq: int):
        H, d, K, M, dt = self.H, self.d, self.top_k, self.n_mem, self.dtype
        f32, i32 = torch.float32, torch.int32
        b = dict(
            idx=self._buf("idx", (n_tok, K), i32), gate=self._buf("gate", (n_tok, K), f32),
            perm=self._buf("perm", (n_tok * K,), i32), row_of=self._buf("row_of", (n_tok * K,), i32),
            mem_offset=self._buf("mem_offset", (M + 1,), i32), seg_cu=self._buf("seg_cu", (M * n_seq + 1,), i32),
            q=self._buf("q", (n_tok, H, d), dt), k_sh=self._buf("k_sh", (n_tok, H, d), dt),
            v_sh=self._buf("v_sh", (n_tok, H, d), dt), beta=self._buf("beta", (n_tok, H), f32),
            log_alpha=self._buf("log_alpha", (n_tok, H), f32),
            k_p=self._buf("k_p", (n_tok * K, H, d), dt), v_p=self._buf("v_p", (n_tok * K, H, d), dt),
            o_sh=self._buf("o_sh", (n_tok, H, d), dt), o_p=self._buf("o_p", (n_tok * K, H, d), dt),
            out=self._buf("out", (n_tok, H, d), dt),
            h_shared=self._buf("h_shared", (n_seq, H, d, d), f32),
            h_mem=self._buf("h_mem", (M, n_seq, H, d, d), f32),
        )
        if self.mem_gates:
            b["beta_p"] = self._buf("beta_p", (n_tok * K, H), f32)
            b["log_alpha_p"] = self._buf("log_alpha_p", (n_tok * K, H), f32)
            b["ws_mem_gate"] = self._ws("mem_gate", B.MOM_WS_HEADER_BYTES)
        dtc = B.dtype_code(dt)
        b["ws_perm"] = self._ws("perm", B.mom_permute_workspace_size(n_tok, K, M, n_seq))
        b["ws_proj"] = self._ws("proj", B.mom_kv_proj_workspace_size(n_tok, self.d_model, H, d, M, K))
        b["ws_gate"] = self._ws("gate", B.mom_gate_proj_workspace_size(n_tok, self.d_model, H))
        b["ws_gdn_sh"] = self._ws("gdn_sh", B.mom_gdn_workspace_size(n_tok, n_seq, H, d, dtc))
        b["ws_gdn_p"] = self._ws("gdn_p", B.mom_gdn_workspace_size(n_tok * K, M * n_seq, H, d, dtc))
        b["ws_comb"] = self._ws("comb", B.MOM_WS_HEADER_BYTES)
        return b

    # -------------------------------------------------------------- forward
    STEPS = ("router", "permute", "proj", "gdn", "combine")

    def forward(self, x: torch.Tensor, cu_seqlens: torch.Tensor, h0_shared=None, h0_mem=None,
                want_states: bool = True, stream=None, marks=None) -> Dict[str, torch.Tensor]:
        """x [N, d_model] (device), cu_seqlens [S+1] int32 (device).  Returns
        the buffers dict; ``out`` is the layer output, ``h_shared`` [S,H,d,d]
        and ``h_mem`` [M,S,H,d,d] the final states.  ``marks``: optional list
        of 6 CUDA events, recorded before the first call and after each step
        of STEPS (per-step timing on the launching stream).  The gates and
        the routed recurrences run on a side stream joined back before the
        steps that read them."""
        n_tok = x.shape[0]
        n_seq = cu_seqlens.numel() - 1
        w, b = self.w, self.buffers(n_tok, n_seq)
        st = stream if stream is not None else torch.cuda.current_stream()
        mark = (lambda i: marks[i].record(st)) if marks is not None else (lambda i: None)
        side = self._side_stream()
        mark(0)
        # the gates need no routing: they run beside the router and the reordering
        start = torch.cuda.Event()
        start.record(st)
        side.wait_event(start)
        B.mom_gate_proj(x, w["w_gate"], w["A"], w["b_a"], b["beta"], b["log_alpha"], b["ws_gate"], stream=side)
        gates_done = torch.cuda.Event()
        gates_done.record(side)
        B.mom_router_topk(x, w["w_r"], w["b_r"], self.top_k, b["idx"], b["gate"], stream=st)
        mark(1)
        B.mom_permute(b["idx"], self.n_mem, cu_seqlens, b["perm"], b["row_of"], b["mem_offset"], b["seg_cu"],
                      b["ws_perm"], stream=st)
        if self.mem_gates:
            # the routed rows' own gates, beside the projections
            permuted = torch.cuda.Event()
            permuted.record(st)
            side.wait_event(permuted)
            B.mom_mem_gate_proj(x, b["perm"], b["mem_offset"], w["w_gate_mem"], w["A_mem"], w["b_a_mem"],
                                self.top_k, b["beta_p"], b["log_alpha_p"], b["ws_mem_gate"], stream=side)
            gates_done.record(side)
        mark(2)
        B.mom_kv_proj_grouped(x, b["perm"], b["mem_offset"], w["w_shared"], None, None, None,
                              w["w_kv"], self.H, self.d, self.top_k, b["q"], b["k_sh"], b["v_sh"], None,
                              None, b["k_p"], b["v_p"], b["ws_proj"], stream=st)
        st.wait_event(gates_done)
        mark(3)
        self._gdn_calls(b, cu_seqlens, h0_shared, h0_mem, want_states, st, side)
        mark(4)
        B.mom_combine_unpermute(b["o_sh"], b["o_p"], b["row_of"], b["gate"], b["out"], b["ws_comb"], stream=st)
        mark(5)
        return b

    def _gdn_calls(self, b, cu_seqlens, h0_shared, h0_mem, want_states, st, side):
        """The shared and routed recurrences (b: the buffers, q, k and v
        filled); on return st waits for both."""
        hs = b["h_shared"] if want_states else None
        hm = b["h_mem"] if want_states else None
        gdn_sh = (b["q"], None, b["k_sh"], b["v_sh"], b["beta"], b["log_alpha"], cu_seqlens,
                  self.scale, self.rule, h0_shared, hs, b["o_sh"], b["ws_gdn_sh"])
        if self.mem_gates:
            gdn_p = (b["q"], b["perm"], b["k_p"], b["v_p"], b["beta_p"], b["log_alpha_p"], b["seg_cu"],
                     self.scale, self.rule, h0_mem, hm, b["o_p"], b["ws_gdn_p"])
            gates_p = B.MOM_GATES_BY_ROW
        else:
            gdn_p = (b["q"], b["perm"], b["k_p"], b["v_p"], b["beta"], b["log_alpha"], b["seg_cu"],
                     self.scale, self.rule, h0_mem, hm, b["o_p"], b["ws_gdn_p"])
            gates_p = B.MOM_GATES_BY_TOKEN
        fork = torch.cuda.Event()
        if self.gdn_schedule == "phased":
            # both problems' state-independent chunk work first, on the whole
            # GPU; then the two serial walks side by side, the shared memory's
            # (whole sequences: the longest chain) launched first so that its
            # CTAs hold SMs before the routed walks fill the rest
            B.mom_memory_chunk_prep(*gdn_sh, stream=st)
            B.mom_memory_chunk_prep(*gdn_p, stream=st, gates=gates_p)
            fork.record(st)
            B.mom_memory_chunk_state(*gdn_sh, stream=st)
            side.wait_event(fork)
            B.mom_memory_chunk_state(*gdn_p, stream=side, gates=gates_p)
        else:
            # each problem's prep then walk on its own stream: the shared
            # problem on a high-priority stream (its CTAs are dispatched first,
            # so its walk starts as soon as its smaller prep is done), the
            # routed prep and walks filling the rest of the GPU around it
            hi = self._hi_stream()
            fork.record(st)
            hi.wait_event(fork)
            side.wait_event(fork)
            B.mom_memory_chunk_prep(*gdn_sh, stream=hi)
            B.mom_memory_chunk_state(*gdn_sh, stream=hi)
            B.mom_memory_chunk_prep(*gdn_p, stream=side, gates=gates_p)
            B.mom_memory_chunk_state(*gdn_p, stream=side, gates=gates_p)
            hi_done = torch.cuda.Event()
            hi_done.record(hi)
            st.wait_event(hi_done)
        join = torch.cuda.Event()
        join.record(side)
        st.wait_event(join)

    def _side_stream(self):
        """Side stream: the gate projections beside the router and the
        reordering, and the routed memories' GDN beside the shared memory's."""
        s = getattr(self, "_side", None)
        if s is None:
            s = self._side = torch.cuda.Stream(device=self.device)
        return s

    def _hi_stream(self):
        """High-priority stream for the shared memory's GDN (the longest serial
        chain of the layer) in the "streams" schedule."""
        s = getattr(self, "_hi", None)
        if s is None:
            _, hi = torch.cuda.Stream.priority_range()
            s = self._hi = torch.cuda.Stream(device=self.device, priority=hi)
        return s

    def device_errors(self):
        """(code, info) of every workspace with a recorded violation."""
        errs = {}
        for key, t in self._bufs.items():
            if isinstance(key, tuple) and key[0] == "ws":
                code, info = B.mom_get_error(t)
                if code:
                    errs[key[1]] = (code, info)
        return errs

    # ------------------------------------------------------------- backward
    def backward(self, x: torch.Tensor, cu_seqlens: torch.Tensor, dout: torch.Tensor, dh_shared=None, dh_mem=None,
                 h0_shared=None, h0_mem=None, stream=None) -> Dict[str, torch.Tensor]:
        """Gradients of <dout, out> + <dh_shared, h_shared> + <dh_mem, h_mem>
        for the forward just run on the same x and cu_seqlens (its buffers
        are read): dx, dw_r, db_r, dw_shared [3Hd, D] (W_q | W_k_sh | W_v_sh),
        dw_gate [2H, D] (W_beta | W_a), dA, db_a, dw_kv [M, 2Hd, D], dh0_shared
        [S, H, d, d], dh0_mem [M, S, H, d, d]; all float32.  The routing is
        held fixed; gradients flow through the renormalised gates.  With
        per-memory gates also dw_gate_mem [M, 2H, D] (W_beta^m | W_a^m),
        dA_mem, db_a_mem [M, H], and dw_gate, dA, db_a carry the shared
        memory's adjoints alone.  Every step runs in the CUDA library (the
        recurrences' reverse passes, then the combine, router, norm and gate
        adjoints and the projections' GEMMs)."""
        n_tok, D = x.shape
        n_seq = cu_seqlens.numel() - 1
        H, d, K, dt = self.H, self.d, self.top_k, self.dtype
        Hd, R = H * d, n_tok * K
        w, b = self.w, self.buffers(n_tok, n_seq)
        st = stream if stream is not None else torch.cuda.current_stream()
        g = self._bwd_buf
        ws = self._ws("bwd", B.MOM_WS_HEADER_BYTES)
        # the lengths the norms' backward needs (the projections again, with their norm outputs)
        qn, kshn, kpn = g("qn", (n_tok, H)), g("kshn", (n_tok, H)), g("kpn", (R, H))
        B.mom_proj_shared(x, w["w_shared"], H, d, g("q2", (n_tok, H, d), dt), g("k2", (n_tok, H, d), dt),
                          g("v2", (n_tok, H, d), dt), ws, stream=st, q_norm=qn, k_sh_norm=kshn)
        B.mom_kv_proj_groups(x, b["perm"], b["mem_offset"], self._mem_groups(st), w["w_kv"], H, d,
                             g("kp2", (R, H, d), dt), g("vp2", (R, H, d), dt), ws, stream=st, k_norm=kpn)
        c = self._core_bwd(b, cu_seqlens, dout, dh_shared, dh_mem, h0_shared, h0_mem, st, ws)
        # pre-activation gradients: shared [N, 3Hd + 2H] (q | k_sh | v_sh | beta | a), routed [N*K, 2Hd] (k | v)
        ldz = (3 * Hd + 2 * H + 3) // 4 * 4        # rows 16-byte aligned for the row copies
        dz = g("dz", (n_tok, ldz))
        B.mom_l2norm_bwd(b["q"], c["dq"], qn, dz, 0, stream=st)
        B.mom_l2norm_bwd(b["k_sh"], c["dk_sh"], kshn, dz, Hd, stream=st)
        B.mom_copy_rows(c["dv_sh"].view(n_tok, Hd), None, dz, Hd * 4, src_off=0, dst_off=2 * Hd * 4, ws=ws,
                        stream=st)
        dala = g("dala", (n_tok, H))
        B.mom_gates_bwd(b["beta"], b["log_alpha"], c["dbeta"], c["dla"], w["A"], dz, 3 * Hd, 3 * Hd + H, dala,
                        stream=st)
        dzr = g("dzr", (R, 2 * Hd))
        B.mom_l2norm_bwd(b["k_p"], c["dk_p"], kpn, dzr, 0, stream=st)
        B.mom_copy_rows(c["dv_p"].view(R, Hd), None, dzr, Hd * 4, src_off=0, dst_off=Hd * 4, ws=ws, stream=st)
        mg = self._mem_gates_bwd(b, c, st)
        r = self._proj_bwd(x, b, dz, 3 * Hd, w["w_shared"], dzr, c["dlogits"], dala, st, ws, mg)
        out = dict(dx=r["dx"], dw_r=r["dw_r"], db_r=r["db_r"], dw_shared=r["dw_sh"], dw_gate=r["dw_gate"],
                   dA=r["dA"], db_a=r["db_a"], dw_kv=r["dw_kv"], dh0_shared=c["dh0_shared"], dh0_mem=c["dh0_mem"])
        out.update({k_: r[k_] for k_ in ("dw_gate_mem", "dA_mem", "db_a_mem") if k_ in r})
        return out

    def _mem_gates_bwd(self, b, c, st):
        """With per-memory gates: the routed rows' gate adjoints under their
        memory's A (pre-activation gradients [N*K, 2H]: beta | a) and
        dla * log alpha per row; None without them."""
        if not self.mem_gates:
            return None
        R, H = c["db_p"].shape
        dzg, dala_p = self._bwd_buf("dzg", (R, 2 * H)), self._bwd_buf("dala_p", (R, H))
        B.mom_gates_bwd_by_group(b["beta_p"], b["log_alpha_p"], c["db_p"], c["dla_p"], self.w["A_mem"],
                                 b["mem_offset"], dzg, 0, H, dala_p, stream=st)
        return dict(dzg=dzg, dala_p=dala_p)

    def _bwd_buf(self, name, shape, dtype=torch.float32):
        return self._buf("bwd_" + name, shape, dtype)

    def _mem_groups(self, st):
        """[0, 1, .., M-1] int32 on the device (made on the launching stream
        st): group g of the routed rows is memory g."""
        mem_index = getattr(self, "_mem_index", None)
        if mem_index is None:
            with torch.cuda.stream(st):
                mem_index = self._mem_index = torch.arange(self.n_mem, dtype=torch.int32, device=self.device)
        return mem_index

    def _core_bwd(self, b, cu_seqlens, dout, dh_shared, dh_mem, h0_shared, h0_mem, st, ws):
        """The reverse pass from the adjoint of the combined output (dout [N, H,
        d], the model dtype) to the recurrences' inputs: the combine's and the
        router's adjoints, both recurrences' reverse passes, and each token's
        routed rows summed into its own (with per-memory gates the routed rows'
        beta and alpha adjoints stay per row: dbeta, dla are then the shared
        memory's).  Returns float32 dq, dk_sh, dv_sh [N, H, d], dk_p, dv_p
        [N*K, H, d], dbeta, dla [N, H], dlogits [N, M], dh0_shared, dh0_mem,
        and the routed rows' db_p, dla_p [N*K, H]."""
        n_tok, n_seq = b["idx"].shape[0], cu_seqlens.numel() - 1
        H, d, K, M = self.H, self.d, self.top_k, self.n_mem
        Hd, R = H * d, n_tok * K
        g = self._bwd_buf
        do_p, dgate = g("do_p", (R, H, d), self.dtype), g("dgate", (n_tok, K))
        B.mom_combine_bwd(dout, b["o_p"], b["row_of"], b["gate"], do_p, dgate, ws, stream=st)
        dlogits = g("dlogits", (n_tok, M))
        B.mom_router_bwd(b["idx"], b["gate"], dgate, dlogits, ws, stream=st)
        dq_sh, dk_sh, dv_sh = (g(n, (n_tok, H, d)) for n in ("dq_sh", "dk_sh", "dv_sh"))
        db_sh, dla_sh = g("db_sh", (n_tok, H)), g("dla_sh", (n_tok, H))
        dq_p, dk_p, dv_p = (g(n, (R, H, d)) for n in ("dq_p", "dk_p", "dv_p"))
        db_p, dla_p = g("db_p", (R, H)), g("dla_p", (R, H))
        dh0_sh, dh0_m = g("dh0_sh", (n_seq, H, d, d)), g("dh0_m", (M, n_seq, H, d, d))
        ws_sh = self._ws("bwd_sh", B.mom_memory_chunk_bwd_workspace_size(n_tok, n_seq, H, d))
        ws_p = self._ws("bwd_p", B.mom_memory_chunk_bwd_workspace_size(R, M * n_seq, H, d))
        # the two reverse passes side by side: the shared memory's (whole
        # sequences, the longest chains) on the high-priority stream, so that
        # its CTAs are dispatched first, the routed memories' filling the rest
        hi, side = self._hi_stream(), self._side_stream()
        fork = torch.cuda.Event()
        fork.record(st)
        hi.wait_event(fork)
        side.wait_event(fork)
        B.mom_memory_chunk_bwd(b["q"], None, b["k_sh"], b["v_sh"], b["beta"], b["log_alpha"], cu_seqlens, self.scale,
                               self.rule, h0_shared, dout, dh_shared, dq_sh, dk_sh, dv_sh, db_sh, dla_sh, dh0_sh, ws_sh,
                               stream=hi)
        dhm = None if dh_mem is None else dh_mem.reshape(M * n_seq, H, d, d)
        h0m = None if h0_mem is None else h0_mem.reshape(M * n_seq, H, d, d)
        if self.mem_gates:
            gates_p = (b["beta_p"], b["log_alpha_p"], B.MOM_GATES_BY_ROW)
        else:
            gates_p = (b["beta"], b["log_alpha"], B.MOM_GATES_BY_TOKEN)
        B.mom_memory_chunk_bwd(b["q"], b["perm"], b["k_p"], b["v_p"], gates_p[0], gates_p[1], b["seg_cu"],
                               self.scale, self.rule, h0m, do_p, dhm, dq_p, dk_p, dv_p, db_p, dla_p,
                               dh0_m.view(M * n_seq, H, d, d), ws_p, stream=side, gates=gates_p[2])
        for s_ in (hi, side):
            done = torch.cuda.Event()
            done.record(s_)
            st.wait_event(done)
        # per token: the shared memory's gradients plus those of its routed rows
        # (with per-memory gates the routed rows' gate adjoints stay per row)
        dq = g("dq", (n_tok, H, d))
        B.mom_rows_sum(dq_p.view(R, Hd), b["row_of"], K, dq_sh.view(n_tok, Hd), dq.view(n_tok, Hd), ws, stream=st)
        if self.mem_gates:
            dbeta, dla = db_sh, dla_sh
        else:
            dbeta, dla = g("dbeta", (n_tok, H)), g("dla", (n_tok, H))
            B.mom_rows_sum(db_p, b["row_of"], K, db_sh, dbeta, ws, stream=st)
            B.mom_rows_sum(dla_p, b["row_of"], K, dla_sh, dla, ws, stream=st)
        return dict(dq=dq, dk_sh=dk_sh, dv_sh=dv_sh, dk_p=dk_p, dv_p=dv_p, dbeta=dbeta, dla=dla, dlogits=dlogits,
                    dh0_shared=dh0_sh, dh0_mem=dh0_m, db_p=db_p, dla_p=dla_p)

    def _proj_bwd(self, x, b, dz, n_sh, w_sh, dzr, dlogits, dala, st, ws, mg=None):
        """The projections' input and weight gradients from the pre-activation
        gradients: dz [N, ldz] float32 holds n_sh columns against w_sh [n_sh,
        D] then beta | a (2H) against w_gate; dzr [N*K, 2Hd] the routed rows'
        against w_kv; dlogits [N, M] against w_r; with per-memory gates (mg:
        _mem_gates_bwd's) the routed rows' gate gradients against w_gate_mem.
        Returns dx, dw_sh, dw_gate, dw_r, dw_kv, db_r, dA, db_a (float32), and
        dw_gate_mem, dA_mem, db_a_mem with mg."""
        n_tok, D = x.shape
        H, Hd, K, M = self.H, self.H * self.d, self.top_k, self.n_mem
        R = n_tok * K
        w, g = self.w, self._bwd_buf
        one = self._buf("one_group", (2,), torch.int32)     # one group of all n_tok rows
        if getattr(self, "_one_n", None) != n_tok:
            with torch.cuda.stream(st):                      # ordered before the GEMMs that read it
                one.copy_(torch.tensor([0, n_tok], dtype=torch.int32))
            self._one_n = n_tok
        # the weight gradients on the side stream beside the input gradient
        # (both only read dz, dzr, dlogits, dala): their last waves fill each
        # other's idle SMs
        side = self._side_stream()
        fork = torch.cuda.Event()
        fork.record(st)
        side.wait_event(fork)
        dx = g("dx", (n_tok, D))
        B.mom_gemm_grouped(0, dz, w_sh, dx, 0, D, n_sh, one, None, 1, ws, total_rows=n_tok, stream=st)
        B.mom_gemm_grouped(0, dz, w["w_gate"], dx, 0, D, 2 * H, one, None, 1, ws, a_col=n_sh, total_rows=n_tok,
                           accumulate=True, stream=st)
        B.mom_gemm_grouped(0, dlogits, w["w_r"], dx, 0, D, M, one, None, 1, ws, total_rows=n_tok, accumulate=True,
                           stream=st)
        dx_rows = g("dx_rows", (R, D))
        B.mom_gemm_grouped(0, dzr, w["w_kv"], dx_rows, 0, D, 2 * Hd, b["mem_offset"], None, M, ws, total_rows=R,
                           b_group_stride=2 * Hd * D, stream=st)
        if mg is not None:
            B.mom_gemm_grouped(0, mg["dzg"], w["w_gate_mem"], dx_rows, 0, D, 2 * H, b["mem_offset"], None, M, ws,
                               total_rows=R, b_group_stride=2 * H * D, accumulate=True, stream=st)
        B.mom_rows_sum(dx_rows, b["row_of"], K, dx, dx, ws, stream=st)
        dw_sh, dw_gate, dw_r = g("dw_sh", (n_sh, D)), g("dw_gate", (2 * H, D)), g("dw_r", (M, D))
        dw_kv = g("dw_kv", (M, 2 * Hd, D))
        ws_w = self._ws("bwd_w", B.MOM_WS_HEADER_BYTES)
        B.mom_gemm_grouped(1, dz, x, dw_sh, n_sh, D, 0, one, None, 1, ws_w, stream=side)
        B.mom_gemm_grouped(1, dz, x, dw_gate, 2 * H, D, 0, one, None, 1, ws_w, a_col=n_sh, stream=side)
        B.mom_gemm_grouped(1, dlogits, x, dw_r, M, D, 0, one, None, 1, ws_w, stream=side)
        B.mom_gemm_grouped(1, dzr, x, dw_kv.view(M * 2 * Hd, D), 2 * Hd, D, 0, b["mem_offset"], None, M, ws_w,
                           b_rows=b["perm"], c_group_stride=2 * Hd * D, stream=side)
        db_r, dA, db_a = g("db_r", (M,)), g("dA", (H,)), g("db_a", (H,))
        B.mom_col_sums(dlogits, db_r, stream=side)
        B.mom_col_sums(dala, dA, stream=side)
        B.mom_col_sums(dz, db_a, col0=n_sh + H, stream=side)
        out = dict(dx=dx, dw_sh=dw_sh, dw_gate=dw_gate, dw_r=dw_r, dw_kv=dw_kv, db_r=db_r, dA=dA, db_a=db_a)
        if mg is not None:
            dw_gm, dA_m, db_am = g("dw_gate_mem", (M, 2 * H, D)), g("dA_mem", (M, H)), g("db_a_mem", (M, H))
            B.mom_gemm_grouped(1, mg["dzg"], x, dw_gm.view(M * 2 * H, D), 2 * H, D, 0, b["mem_offset"], None, M, ws_w,
                               b_rows=b["perm"], c_group_stride=2 * H * D, stream=side)
            B.mom_col_sums_grouped(mg["dala_p"], b["mem_offset"], dA_m, stream=side)
            B.mom_col_sums_grouped(mg["dzg"], b["mem_offset"], db_am, col0=H, cols=H, stream=side)
            out.update(dw_gate_mem=dw_gm, dA_mem=dA_m, db_a_mem=db_am)
        done = torch.cuda.Event()
        done.record(side)
        st.wait_event(done)
        return out

    # --------------------------------------------------------------- decode
    def decode_step(self, x: torch.Tensor, state: torch.Tensor, stream=None):
        """x [B, d_model]; state [B, M+1, H, d, d] float32, updated in place.
        Returns (out [B,H,d], topk_idx [B,k])."""
        Bn = x.shape[0]
        out = self._buf("dec_out", (Bn, self.H, self.d), self.dtype)
        idx = self._buf("dec_idx", (Bn, self.top_k), torch.int32)
        ws = self._ws("decode", B.mom_decode_workspace_size(Bn, self.d_model, self.H, self.d, self.n_mem, self.top_k))
        B.mom_decode_step_rule(x, self._c_weights, self.H, self.d, self.n_mem, self.top_k, self.scale, self.rule,
                               state, out, idx, ws, stream=stream, mem_gates=self._c_mem_gates)
        return out, idx


def ctypes_ptr(t: Optional[torch.Tensor]):
    """Device address of a weight tensor (checked like every pointer the
    binding passes: a dense CUDA tensor)."""
    p = B._p(t)
    return None if p is None else p.value
