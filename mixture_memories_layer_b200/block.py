"""The MoM layer inside its Gated DeltaNet block, on the GPU.

The pages name Gated DeltaNet as every memory's token mixer (the authors'
MoM blog post, experiments section) and print nothing of the block around
it; the plain Gated DeltaNet block is taken:

    router -> permute -> projections (unnormalised, plus the output gate g)
           -> short causal convolutions + SiLU (+ L2 norm of q, k)
           -> GDN prep / walks (shared | routed) -> combine + gated RMS norm
           -> output projection W_o

Every step runs in the CUDA library (mom_block_proj, mom_short_conv, the
recurrences, mom_combine_norm_gate, mom_linear; the reverse pass adds
mom_norm_gate_bwd, mom_short_conv_bwd, mom_convert and the layer's backward
calls); this module packs weights, holds buffers and passes pointers.
bf16 only.
"""
from __future__ import annotations

from typing import Dict

import numpy as np
import torch

from . import binding as B
from .layer import MoMLayer, pack_weights

RMS_EPS = 1e-5


def pack_block_weights(p: Dict[str, np.ndarray], dtype: torch.dtype, device="cuda") -> Dict[str, torch.Tensor]:
    """pack_weights plus the block's: w_shared4 = [W_q; W_k_sh; W_v_sh; W_g],
    w_o [d_model, H d] and its transpose w_o_t, the convolution filters
    tap-major as float32 [groups, width, H d] (conv_q, conv_k_sh, conv_v_sh:
    one group; conv_k, conv_v: one group per memory) and w_norm [d]."""
    w = pack_weights(p, dtype, device)
    t = lambda a, dt=dtype: torch.as_tensor(np.ascontiguousarray(a)).to(device=device, dtype=dt)
    f32 = torch.float32
    w["w_shared4"] = t(np.concatenate([p["w_q"], p["w_k_sh"], p["w_v_sh"], p["w_g"]], axis=0))
    w["w_o"] = t(p["w_o"])
    w["w_o_t"] = t(np.transpose(p["w_o"]))                # [H d, d_model]: the reverse pass's dy W_o
    for name in ("conv_q", "conv_k_sh", "conv_v_sh"):
        w[name] = t(np.swapaxes(p[name][None], 1, 2), f32)
    w["conv_k"] = t(np.swapaxes(p["conv_k"], 1, 2), f32)
    w["conv_v"] = t(np.swapaxes(p["conv_v"], 1, 2), f32)
    w["w_norm"] = t(p["w_norm"], f32)
    return w


class MoMBlock(MoMLayer):
    """The layer with its block: forward(x, cu_seqlens)["y"] [N, d_model]."""

    STEPS = ("router", "permute", "proj_conv", "gdn", "combine_norm", "o_proj")

    def __init__(self, weights: Dict[str, torch.Tensor], heads: int, d_head: int, top_k: int, scale: float = 1.0,
                 gdn_schedule: str = "streams", rule: str = "gated_delta", eps: float = RMS_EPS):
        super().__init__(weights, heads, d_head, top_k, scale, gdn_schedule, rule)
        if self.dtype != torch.bfloat16:
            raise ValueError("the block runs in bf16")
        self.eps = eps

    def block_buffers(self, n_tok: int, n_seq: int):
        b = self.buffers(n_tok, n_seq)
        H, d, K, dt = self.H, self.d, self.top_k, self.dtype
        for name, rows in (("q_raw", n_tok), ("k_sh_raw", n_tok), ("v_sh_raw", n_tok), ("g", n_tok),
                           ("k_p_raw", n_tok * K), ("v_p_raw", n_tok * K), ("o_tilde", n_tok)):
            b[name] = self._buf(name, (rows, H, d), dt)
        b["y"] = self._buf("y", (n_tok, self.d_model), dt)
        b["ws_conv"] = self._ws("conv", B.MOM_WS_HEADER_BYTES)
        b["ws_lin"] = self._ws("lin", B.MOM_WS_HEADER_BYTES)
        return b

    def forward(self, x: torch.Tensor, cu_seqlens: torch.Tensor, h0_shared=None, h0_mem=None,
                want_states: bool = True, stream=None, marks=None) -> Dict[str, torch.Tensor]:
        """x [N, d_model] bf16, cu_seqlens [S+1] int32 (device).  Returns the
        buffers dict: ``y`` the block output, ``o_tilde`` the normalised and
        gated memories' output, ``h_shared`` / ``h_mem`` the final states.
        ``marks``: optional 7 CUDA events, recorded before the first call and
        after each of router, permute, projections + convolutions, GDN,
        combine + norm, output projection."""
        n_tok = x.shape[0]
        n_seq = cu_seqlens.numel() - 1
        w, b = self.w, self.block_buffers(n_tok, n_seq)
        st = stream if stream is not None else torch.cuda.current_stream()
        mark = (lambda i: marks[i].record(st)) if marks is not None else (lambda i: None)
        side = self._side_stream()
        mark(0)
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
            permuted = torch.cuda.Event()
            permuted.record(st)
            side.wait_event(permuted)
            B.mom_mem_gate_proj(x, b["perm"], b["mem_offset"], w["w_gate_mem"], w["A_mem"], w["b_a_mem"],
                                self.top_k, b["beta_p"], b["log_alpha_p"], b["ws_mem_gate"], stream=side)
            gates_done.record(side)
        mark(2)
        B.mom_block_proj(x, b["perm"], b["mem_offset"], w["w_shared4"], w["w_kv"], self.H, self.d, self.top_k,
                         b["q_raw"], b["k_sh_raw"], b["v_sh_raw"], b["g"], b["k_p_raw"], b["v_p_raw"], b["ws_proj"],
                         stream=st)
        # one launch for the five convolutions; memory m's rows of sequence s
        # are segment m * S + s of seg_cu
        B.mom_short_conv_batch([
            dict(z=b["q_raw"], out=b["q"], seg_cu=cu_seqlens, w=w["conv_q"], l2norm=True),
            dict(z=b["k_sh_raw"], out=b["k_sh"], seg_cu=cu_seqlens, w=w["conv_k_sh"], l2norm=True),
            dict(z=b["v_sh_raw"], out=b["v_sh"], seg_cu=cu_seqlens, w=w["conv_v_sh"]),
            dict(z=b["k_p_raw"], out=b["k_p"], seg_cu=b["seg_cu"], w=w["conv_k"], seg_per_group=n_seq, l2norm=True),
            dict(z=b["v_p_raw"], out=b["v_p"], seg_cu=b["seg_cu"], w=w["conv_v"], seg_per_group=n_seq),
        ], self.d, b["ws_conv"], stream=st)
        st.wait_event(gates_done)
        mark(3)
        self._gdn_calls(b, cu_seqlens, h0_shared, h0_mem, want_states, st, side)
        mark(4)
        B.mom_combine_norm_gate(b["o_sh"], b["o_p"], b["row_of"], b["gate"], b["g"], w["w_norm"], self.eps,
                                b["o_tilde"], b["ws_comb"], stream=st)
        mark(5)
        B.mom_linear(b["o_tilde"].view(n_tok, -1), w["w_o"], b["y"], b["ws_lin"], stream=st)
        mark(6)
        return b

    # ------------------------------------------------------------ decode
    @property
    def width(self) -> int:
        return self.w["conv_q"].shape[1]

    def _c_block(self):
        cb = getattr(self, "_cb", None)
        if cb is None:
            from .layer import ctypes_ptr
            cb = self._cb = B.MomBlockWeights(*[ctypes_ptr(self.w[k]) for k in
                                                ("w_shared4", "w_o", "conv_q", "conv_k_sh", "conv_v_sh", "conv_k",
                                                 "conv_v", "w_norm")])
        return cb

    def new_conv_state(self, n_seq: int):
        """Zero windows: conv_sh [S, 3, W-1, H, d], conv_mem [S, M, 2, W-1, H, d]."""
        Wm = self.width - 1
        z = lambda *shape: torch.zeros(shape, dtype=self.dtype, device=self.device)
        return z(n_seq, 3, Wm, self.H, self.d), z(n_seq, self.n_mem, 2, Wm, self.H, self.d)

    def conv_state(self, b, cu_seqlens, stream=None):
        """The windows the forward that returned buffers ``b`` leaves (for
        decode_step): (conv_sh, conv_mem)."""
        n_seq = cu_seqlens.numel() - 1
        conv_sh, conv_mem = self.new_conv_state(n_seq)
        B.mom_block_conv_state(b["q_raw"], b["k_sh_raw"], b["v_sh_raw"], b["k_p_raw"], b["v_p_raw"], cu_seqlens,
                               b["seg_cu"], self.n_mem, self.top_k, self.width, conv_sh, conv_mem, b["ws_conv"],
                               stream=stream)
        return conv_sh, conv_mem

    def decode_step(self, x: torch.Tensor, state: torch.Tensor, conv_sh: torch.Tensor, conv_mem: torch.Tensor,
                    stream=None):
        """x [B, d_model]; state [B, M+1, H, d, d] float32 and the windows,
        all updated in place.  Returns (y [B, d_model], topk_idx [B, k])."""
        Bn = x.shape[0]
        y = self._buf("bdec_y", (Bn, self.d_model), self.dtype)
        idx = self._buf("bdec_idx", (Bn, self.top_k), torch.int32)
        ws = self._ws("bdecode", B.mom_block_decode_workspace_size(Bn, self.d_model, self.H, self.d, self.n_mem,
                                                                   self.top_k))
        B.mom_block_decode_step(x, self._c_weights, self._c_block(), self.width, self.eps, self.H, self.d, self.n_mem,
                                self.top_k, self.scale, self.rule, state, conv_sh, conv_mem, y, idx, ws,
                                stream=stream, mem_gates=self._c_mem_gates)
        return y, idx

    # ----------------------------------------------------------- backward
    def backward(self, x: torch.Tensor, cu_seqlens: torch.Tensor, dy: torch.Tensor, dh_shared=None, dh_mem=None,
                 h0_shared=None, h0_mem=None, stream=None) -> Dict[str, torch.Tensor]:
        """Gradients of <dy, y> + <dh_shared, h_shared> + <dh_mem, h_mem> for
        the forward just run on the same x and cu_seqlens (its buffers are
        read; dy [N, d_model] bf16).  Returns float32: dx; dw_o [d_model, Hd];
        dw_norm [d]; dw_shared4 [4Hd, D] (W_q | W_k_sh | W_v_sh | W_g);
        dw_gate [2H, D]; dA, db_a; dw_r, db_r; dw_kv [M, 2Hd, D]; the filters'
        dconv_q, dconv_k_sh, dconv_v_sh [1, W, Hd] and dconv_k, dconv_v [M, W,
        Hd] (tap-major, as packed); dh0_shared, dh0_mem.  The routing is held
        fixed.  Every step runs in the CUDA library: the output projection's
        two GEMMs, the gated norm's adjoint (which also gives the output
        gate's), the layer's reverse pass, the five convolutions' adjoints in
        one launch pair, the gates' adjoint and the projections' GEMMs.  With
        per-memory gates also dw_gate_mem [M, 2H, D], dA_mem, db_a_mem [M, H]
        (as MoMLayer.backward)."""
        n_tok, D = x.shape
        n_seq = cu_seqlens.numel() - 1
        H, d, K, M, dt = self.H, self.d, self.top_k, self.n_mem, self.dtype
        Hd, R = H * d, n_tok * K
        w, b = self.w, self.block_buffers(n_tok, n_seq)
        st = stream if stream is not None else torch.cuda.current_stream()
        g = self._bwd_buf
        ws = self._ws("bwd", B.MOM_WS_HEADER_BYTES)
        # y = o~ W_o^T: do~ = dy W_o (tensor cores, bf16 out), dW_o = dy^T o~
        dot = g("do_tilde", (n_tok, H, d), dt)
        B.mom_linear(dy, w["w_o_t"], dot.view(n_tok, Hd), b["ws_lin"], stream=st)
        dy32 = g("dy32", (n_tok, D))
        B.mom_convert(dy, dy32, stream=st)
        dw_o = g("dw_o", (D, Hd))
        one = self._buf("one_group", (2,), torch.int32)
        if getattr(self, "_one_n", None) != n_tok:
            with torch.cuda.stream(st):                      # ordered before the GEMMs that read it
                one.copy_(torch.tensor([0, n_tok], dtype=torch.int32))
            self._one_n = n_tok
        B.mom_gemm_grouped(1, dy32, b["o_tilde"].view(n_tok, Hd), dw_o, D, Hd, 0, one, None, 1, ws, stream=st)
        # o~ = rmsnorm(o) w_norm SiLU(g): do (bf16), dg into the pre-activation
        # gradients' g columns, dw_norm.  dz [N, 4Hd + 2H]: q | k_sh | v_sh | g | beta | a
        ldz = (4 * Hd + 2 * H + 3) // 4 * 4
        dz = g("dz4", (n_tok, ldz))
        do = g("do", (n_tok, H, d), dt)
        dw_norm = g("dw_norm", (d,))
        B.mom_norm_gate_bwd(b["o_sh"], b["o_p"], b["row_of"], b["gate"], b["g"], w["w_norm"], self.eps, dot, do,
                            dz[:, 3 * Hd:], dw_norm, ws, stream=st)
        c = self._core_bwd(b, cu_seqlens, do, dh_shared, dh_mem, h0_shared, h0_mem, st, ws)
        # the convolutions (+ SiLU, + L2 norm of q and k) backwards, from the
        # recurrences' input gradients into the raw projections' columns
        dzr = g("dzr", (R, 2 * Hd))
        f = lambda t: t.view(t.shape[0], Hd)
        dconv = {n: g("d" + n, tuple(w[n].shape)) for n in ("conv_q", "conv_k_sh", "conv_v_sh", "conv_k", "conv_v")}
        B.mom_short_conv_bwd([
            dict(z=b["q_raw"], dout=f(c["dq"]), dz=dz[:, 0:Hd], seg_cu=cu_seqlens, w=w["conv_q"],
                 dw=dconv["conv_q"], l2norm=True),
            dict(z=b["k_sh_raw"], dout=f(c["dk_sh"]), dz=dz[:, Hd:2 * Hd], seg_cu=cu_seqlens,
                 w=w["conv_k_sh"], dw=dconv["conv_k_sh"], l2norm=True),
            dict(z=b["v_sh_raw"], dout=f(c["dv_sh"]), dz=dz[:, 2 * Hd:3 * Hd], seg_cu=cu_seqlens,
                 w=w["conv_v_sh"], dw=dconv["conv_v_sh"]),
            dict(z=b["k_p_raw"], dout=f(c["dk_p"]), dz=dzr[:, 0:Hd], seg_cu=b["seg_cu"],
                 seg_per_group=n_seq, w=w["conv_k"], dw=dconv["conv_k"], l2norm=True),
            dict(z=b["v_p_raw"], dout=f(c["dv_p"]), dz=dzr[:, Hd:], seg_cu=b["seg_cu"],
                 seg_per_group=n_seq, w=w["conv_v"], dw=dconv["conv_v"]),
        ], d, ws, stream=st)
        dala = g("dala", (n_tok, H))
        B.mom_gates_bwd(b["beta"], b["log_alpha"], c["dbeta"], c["dla"], w["A"], dz, 4 * Hd, 4 * Hd + H, dala,
                        stream=st)
        mg = self._mem_gates_bwd(b, c, st)
        r = self._proj_bwd(x, b, dz, 4 * Hd, w["w_shared4"], dzr, c["dlogits"], dala, st, ws, mg)
        out = dict(dx=r["dx"], dw_o=dw_o, dw_norm=dw_norm, dw_shared4=r["dw_sh"], dw_gate=r["dw_gate"], dA=r["dA"],
                   db_a=r["db_a"], dw_r=r["dw_r"], db_r=r["db_r"], dw_kv=r["dw_kv"], dh0_shared=c["dh0_shared"],
                   dh0_mem=c["dh0_mem"])
        out.update({"d" + n: t for n, t in dconv.items()})
        out.update({k_: r[k_] for k_ in ("dw_gate_mem", "dA_mem", "db_a_mem") if k_ in r})
        return out
