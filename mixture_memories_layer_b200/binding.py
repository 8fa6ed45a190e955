"""Thin ctypes binding of the C ABI in ``include/mom.h``.

Argument marshalling only: every function here passes device pointers and
sizes through to the CUDA library, which does all the work.  Tensors are
torch tensors on the current CUDA device; ``stream`` defaults to torch's
current stream.  If the library is missing this module raises at import --
there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional
from ctypes import POINTER, c_char_p, c_float, c_int, c_int32, c_int64, c_size_t, c_void_p

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmom_b200.so")

MOM_OK, MOM_ERR_ARG, MOM_ERR_UNSUPPORTED, MOM_ERR_CUDA, MOM_ERR_DEVICE = 0, 1, 2, 3, 4
MOM_F32, MOM_BF16 = 0, 1
MOM_DEVERR_NONE, MOM_DEVERR_MEM_INDEX, MOM_DEVERR_ROW_INDEX, MOM_DEVERR_SEGMENT, MOM_DEVERR_TIMEOUT = 0, 1, 2, 3, 4
MOM_WS_HEADER_BYTES = 256
MOM_SELFTEST_WAIT_SITE = 990

# every function the header declares, with (restype, argtypes)
_VP, _I, _I64, _F, _SZ = c_void_p, c_int, c_int64, c_float, c_size_t
SIGNATURES = {
    "mom_status_string": (c_char_p, [_I]),
    "mom_get_error": (_I, [_VP, POINTER(c_int32), POINTER(c_int32), _VP]),
    "mom_clear_error": (_I, [_VP, _VP]),
    "mom_launch_count": (ctypes.c_uint64, []),
    "mom_selftest_wait_timeout": (_I, [_VP, _SZ, _I64, _VP]),
    "mom_router_topk": (_I, [_VP, _VP, _VP, _I, _I64, _I, _I, _I, _VP, _VP, _VP, _VP]),
    "mom_permute_workspace_size": (_SZ, [_I64, _I, _I, _I]),
    "mom_permute": (_I, [_VP, _I64, _I, _I, _VP, _I, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "mom_permute_noalloc": (_I, [_VP, _I64, _I, _I, _VP, _I, _VP, _VP, _VP, _VP, _VP, _VP]),
    "mom_kv_proj_workspace_size": (_SZ, [_I64, _I, _I, _I, _I, _I]),
    "mom_gate_proj_workspace_size": (_SZ, [_I64, _I, _I]),
    "mom_gate_proj": (_I, [_VP, _VP, _VP, _VP, _I, _I64, _I, _I, _VP, _VP, _VP, _SZ, _VP]),
    "mom_kv_proj_grouped": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I, _I, _I, _I, _I,
                                 _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "mom_gdn_workspace_size": (_SZ, [_I64, _I, _I, _I, _I]),
    "mom_gdn_chunk_fwd": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I64, _I, _I, _F, _I,
                               _VP, _VP, _VP, _VP, _SZ, _VP]),
    "mom_gdn_chunk_prep": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I64, _I, _I, _F, _I,
                               _VP, _VP, _VP, _VP, _SZ, _VP]),
    "mom_gdn_chunk_state": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I64, _I, _I, _F, _I,
                               _VP, _VP, _VP, _VP, _SZ, _VP]),
    "mom_memory_chunk_fwd": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I64, _I, _I, _F, _I, _I, _I,
                                  _VP, _VP, _VP, _VP, _SZ, _VP]),
    "mom_memory_chunk_prep": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I64, _I, _I, _F, _I, _I, _I,
                                   _VP, _VP, _VP, _VP, _SZ, _VP]),
    "mom_memory_chunk_state": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I64, _I, _I, _F, _I, _I, _I,
                                    _VP, _VP, _VP, _VP, _SZ, _VP]),
    "mom_combine_unpermute": (_I, [_VP, _VP, _VP, _VP, _I64, _I, _I, _I, _I, _VP, _VP, _SZ, _VP]),
    "mom_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "mom_decode_step": (_I, [_VP, _VP, _I, _I, _I, _I, _I, _I, _F, _I, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "mom_decode_step_rule": (_I, [_VP, _VP, _VP, _I, _I, _I, _I, _I, _I, _F, _I, _I, _VP, _VP, _VP, _VP, _SZ,
                                  _VP]),
    "mom_mem_gate_proj": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I, _I, _I, _I, _VP, _VP, _VP, _SZ, _VP]),
    "mom_proj_shared": (_I, [_VP, _VP, _I, _I64, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "mom_kv_proj_groups": (_I, [_VP, _I64, _VP, _I64, _VP, _VP, _I, _VP, _I, _I, _I, _I, _I, _VP, _VP, _VP, _VP, _SZ,
                                _VP]),
    "mom_copy_rows": (_I, [_VP, _I64, _I64, _I64, _VP, _I64, _I64, _VP, _I64, _I64, _VP, _SZ, _VP]),
    "mom_memory_chunk_bwd_workspace_size": (_SZ, [_I64, _I, _I, _I]),
    "mom_combine_bwd": (_I, [_VP, _VP, _VP, _VP, _I64, _I, _I64, _I, _I, _I, _VP, _VP, _VP, _SZ, _VP]),
    "mom_router_bwd": (_I, [_VP, _VP, _VP, _I64, _I, _I, _VP, _VP, _SZ, _VP]),
    "mom_rows_sum": (_I, [_VP, _I64, _VP, _I, _VP, _I64, _I, _VP, _VP, _SZ, _VP]),
    "mom_l2norm_bwd": (_I, [_VP, _VP, _VP, _I64, _I, _I, _I, _VP, _I64, _I64, _VP]),
    "mom_gates_bwd": (_I, [_VP, _VP, _VP, _VP, _VP, _I64, _I, _VP, _I64, _I64, _I64, _VP, _VP]),
    "mom_col_sums": (_I, [_VP, _I64, _I64, _I64, _VP, _VP]),
    "mom_mem_gate_proj_groups": (_I, [_VP, _I64, _VP, _I64, _VP, _VP, _I, _VP, _VP, _VP, _I, _I, _I, _I, _VP, _VP,
                                      _VP, _SZ, _VP]),
    "mom_gates_bwd_by_group": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I, _VP, _I64, _I64, _I64, _VP, _VP]),
    "mom_col_sums_grouped": (_I, [_VP, _I64, _I64, _I64, _VP, _I, _VP, _VP]),
    "mom_gemm_grouped": (_I, [_I, _VP, _I64, _VP, _I64, _I, _VP, _I64, _VP, _I64, _I64, _I64, _I64, _I64, _VP, _VP,
                              _I, _I64, _I64, _I, _VP, _SZ, _VP]),
    "mom_memory_chunk_bwd": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _VP, _I, _I64, _I64, _I, _I, _F, _I, _I, _I,
                                  _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _SZ, _VP]),
    "mom_block_proj": (_I, [_VP, _VP, _VP, _VP, _VP, _I, _I64, _I, _I, _I, _I, _I, _VP, _VP, _VP, _VP, _VP, _VP,
                            _VP, _SZ, _VP]),
    "mom_short_conv": (_I, [_VP, _I64, _I, _VP, _I, _I, _I, _VP, _I, _I, _I, _I, _VP, _VP, _SZ, _VP]),
    "mom_short_conv_batch": (_I, [_VP, _I, _I, _I, _I, _I, _VP, _SZ, _VP]),
    "mom_combine_norm_gate": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _F, _I64, _I, _I, _I, _I, _VP, _VP, _SZ, _VP]),
    "mom_linear": (_I, [_VP, _VP, _I, _I64, _I, _I, _VP, _VP, _SZ, _VP]),
    "mom_norm_gate_bwd": (_I, [_VP, _VP, _VP, _VP, _VP, _VP, _F, _VP, _I64, _I, _I, _I, _I, _VP, _VP, _I64, _VP, _VP,
                               _SZ, _VP]),
    "mom_short_conv_bwd": (_I, [_VP, _I, _I, _I, _I, _I, _VP, _SZ, _VP]),
    "mom_convert": (_I, [_VP, _I, _VP, _I, _I64, _VP]),
    "mom_block_decode_workspace_size": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "mom_block_decode_step": (_I, [_VP, _VP, _VP, _VP, _I, _F, _I, _I, _I, _I, _I, _I, _F, _I, _I, _VP, _VP, _VP, _VP,
                                   _VP, _VP, _SZ, _VP]),
    "mom_block_conv_state": (_I, [_VP, _VP, _VP, _VP, _VP, _I64, _I, _VP, _VP, _I, _I, _I, _I, _I, _VP, _VP, _VP, _SZ,
                                  _VP]),
}


class MomWeights(ctypes.Structure):
    """Mirror of ``struct mom_weights`` (device pointers)."""
    _fields_ = [("w_r", c_void_p), ("b_r", c_void_p), ("w_shared", c_void_p), ("w_gate", c_void_p),
                ("A", c_void_p), ("b_a", c_void_p), ("w_kv", c_void_p)]


class MomConvProblem(ctypes.Structure):
    """Mirror of ``struct mom_conv_problem``."""
    _fields_ = [("z", c_void_p), ("out", c_void_p), ("n_rows", c_int64), ("seg_cu", c_void_p), ("n_seg", c_int),
                ("seg_per_group", c_int), ("n_groups", c_int), ("w", c_void_p), ("l2norm", c_int)]


class MomBlockWeights(ctypes.Structure):
    """Mirror of ``struct mom_block_weights`` (device pointers)."""
    _fields_ = [("w_shared4", c_void_p), ("w_o", c_void_p), ("conv_q", c_void_p), ("conv_k_sh", c_void_p),
                ("conv_v_sh", c_void_p), ("conv_k", c_void_p), ("conv_v", c_void_p), ("w_norm", c_void_p)]


class MomConvBwdProblem(ctypes.Structure):
    """Mirror of ``struct mom_conv_bwd_problem``."""
    _fields_ = [("z", c_void_p), ("dout", c_void_p), ("da", c_void_p), ("dz", c_void_p), ("ldz", c_int64),
                ("col0", c_int64), ("n_rows", c_int64), ("seg_cu", c_void_p), ("n_seg", c_int),
                ("seg_per_group", c_int), ("n_groups", c_int), ("w", c_void_p), ("dw", c_void_p), ("l2norm", c_int)]


class MomMemoryGates(ctypes.Structure):
    """Mirror of ``struct mom_memory_gates`` (device pointers)."""
    _fields_ = [("w_gate_mem", c_void_p), ("A_mem", c_void_p), ("b_a_mem", c_void_p)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("MoM CUDA library not built (%s missing); run "
                           "`python -m mixture_memories_layer_b200.build`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


class MomError(RuntimeError):
    pass


def _check(status: int, what: str):
    if status != MOM_OK:
        raise MomError("%s failed: %s (%d)" % (what, lib.mom_status_string(status).decode(), status))


def _p(t):
    """Device pointer of a tensor (None -> NULL).  The C ABI reads dense
    row-major buffers in device memory: a host tensor or a strided view is
    refused here instead of being read as if it were one."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("MoM: a tensor on %s was passed; the library takes CUDA tensors" % t.device)
    if not t.is_contiguous():
        raise ValueError("MoM: a non-contiguous tensor (shape %s, strides %s) was passed; use .contiguous()"
                         % (tuple(t.shape), t.stride()))
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return MOM_BF16
    if t == torch.float32:
        return MOM_F32
    raise ValueError("unsupported dtype %s" % t)


# ------------------------------------------------------------------ helpers

def new_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zeroed workspace (the error record starts clear)."""
    return torch.zeros(max(int(nbytes), MOM_WS_HEADER_BYTES), dtype=torch.uint8, device=device or "cuda")


def mom_get_error(ws: torch.Tensor, stream=None):
    code, info = c_int32(0), c_int32(0)
    st = lib.mom_get_error(_p(ws), ctypes.byref(code), ctypes.byref(info), _s(stream))
    if st not in (MOM_OK, MOM_ERR_DEVICE):
        _check(st, "mom_get_error")
    return code.value, info.value


def mom_launch_count() -> int:
    return int(lib.mom_launch_count())


def mom_clear_error(ws: torch.Tensor, stream=None):
    _check(lib.mom_clear_error(_p(ws), _s(stream)), "mom_clear_error")


def mom_selftest_wait_timeout(ws: torch.Tensor, limit_cycles: int, stream=None):
    _check(lib.mom_selftest_wait_timeout(_p(ws), ws.numel(), int(limit_cycles), _s(stream)),
           "mom_selftest_wait_timeout")


# ------------------------------------------------------- the six entry points

def mom_router_topk(x, w_r, b_r, top_k, topk_idx, topk_gate, logits=None, stream=None):
    n_tok, d_model = x.shape
    _check(lib.mom_router_topk(_p(x), _p(w_r), _p(b_r), dtype_code(x.dtype), n_tok, d_model, w_r.shape[0],
                               top_k, _p(topk_idx), _p(topk_gate), _p(logits), _s(stream)), "mom_router_topk")


def mom_permute_workspace_size(n_tok, top_k, n_mem, n_seq):
    return lib.mom_permute_workspace_size(n_tok, top_k, n_mem, n_seq)


def mom_permute(topk_idx, n_mem, cu_seqlens, perm_token, row_of, mem_offset, seg_cu, ws, stream=None):
    n_tok, top_k = topk_idx.shape
    n_seq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _check(lib.mom_permute(_p(topk_idx), n_tok, top_k, n_mem, _p(cu_seqlens), n_seq, _p(perm_token), _p(row_of),
                           _p(mem_offset), _p(seg_cu), _p(ws), ws.numel(), _s(stream)), "mom_permute")


MOM_PERMUTE_NOALLOC_MAX_TOKENS = 1 << 20


def mom_permute_noalloc(topk_idx, n_mem, cu_seqlens, perm_token, row_of, mem_offset, seg_cu, status=None,
                        stream=None):
    """mom_permute for callers that cannot allocate device memory: no
    workspace; scratch is a fixed array inside the library (shared by all
    calls on the device, so calls must not overlap on the GPU)."""
    n_tok, top_k = topk_idx.shape
    n_seq = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    _check(lib.mom_permute_noalloc(_p(topk_idx), n_tok, top_k, n_mem, _p(cu_seqlens), n_seq, _p(perm_token),
                                   _p(row_of), _p(mem_offset), _p(seg_cu), _p(status), _s(stream)),
           "mom_permute_noalloc")


def mom_kv_proj_workspace_size(n_tok, d_model, H, d, n_mem, top_k):
    return lib.mom_kv_proj_workspace_size(n_tok, d_model, H, d, n_mem, top_k)


def mom_kv_proj_grouped(x, perm_token, mem_offset, w_shared, w_gate, A, b_a, w_kv, H, d, top_k,
                        q, k_sh, v_sh, beta, log_alpha, k_p, v_p, ws, stream=None):
    n_tok, d_model = x.shape
    _check(lib.mom_kv_proj_grouped(_p(x), _p(perm_token), _p(mem_offset), _p(w_shared), _p(w_gate), _p(A), _p(b_a),
                                   _p(w_kv), dtype_code(x.dtype), n_tok, d_model, H, d, w_kv.shape[0], top_k,
                                   _p(q), _p(k_sh), _p(v_sh), _p(beta), _p(log_alpha), _p(k_p), _p(v_p),
                                   _p(ws), ws.numel(), _s(stream)), "mom_kv_proj_grouped")


def mom_gate_proj_workspace_size(n_tok, d_model, H):
    return lib.mom_gate_proj_workspace_size(n_tok, d_model, H)


def mom_gate_proj(x, w_gate, A, b_a, beta, log_alpha, ws, stream=None):
    n_tok, d_model = x.shape
    H = A.shape[0]
    _check(lib.mom_gate_proj(_p(x), _p(w_gate), _p(A), _p(b_a), dtype_code(x.dtype), n_tok, d_model, H,
                             _p(beta), _p(log_alpha), _p(ws), ws.numel(), _s(stream)), "mom_gate_proj")


def mom_mem_gate_proj(x, perm, mem_offset, w_gate_mem, A_mem, b_a_mem, top_k, beta_p, log_alpha_p, ws,
                      stream=None):
    """Per-memory gates of the routed rows: beta_p, log_alpha_p [n_tok*top_k, H]."""
    n_tok, d_model = x.shape
    n_mem, H = A_mem.shape
    _check(lib.mom_mem_gate_proj(_p(x), _p(perm), _p(mem_offset), _p(w_gate_mem), _p(A_mem), _p(b_a_mem),
                                 dtype_code(x.dtype), n_tok, d_model, H, n_mem, top_k, _p(beta_p),
                                 _p(log_alpha_p), _p(ws), ws.numel(), _s(stream)), "mom_mem_gate_proj")


def mom_proj_shared(x, w_shared, H, d, q, k_sh, v_sh, ws, stream=None, q_norm=None, k_sh_norm=None):
    n_tok, d_model = x.shape
    _check(lib.mom_proj_shared(_p(x), _p(w_shared), dtype_code(x.dtype), n_tok, d_model, H, d, _p(q), _p(k_sh),
                               _p(v_sh), _p(q_norm), _p(k_sh_norm), _p(ws), ws.numel(), _s(stream)), "mom_proj_shared")


def mom_kv_proj_groups(x, perm, group_offset, group_mem, w_kv, H, d, k_p, v_p, ws, stream=None, k_norm=None):
    """Routed k/v projections over groups: group g = rows group_offset[g] ..
    group_offset[g+1] with memory group_mem[g]'s weights (perm None: row r
    reads x row r)."""
    n_x, d_model = x.shape
    _check(lib.mom_kv_proj_groups(_p(x), n_x, _p(perm), k_p.shape[0], _p(group_offset), _p(group_mem),
                                  group_mem.numel(), _p(w_kv), dtype_code(x.dtype), d_model, H, d, w_kv.shape[0],
                                  _p(k_p), _p(v_p), _p(k_norm), _p(ws), ws.numel(), _s(stream)), "mom_kv_proj_groups")


def mom_copy_rows(src, idx, dst, row_bytes, src_off=0, dst_off=0, ws=None, stream=None, n_rows=None):
    """dst row i (bytes dst_off ..) = src row idx[i] (or i) (bytes src_off ..);
    src and dst are 2-D tensors whose rows are byte rows of their stride."""
    n_src = src.shape[0]
    n = dst.shape[0] if n_rows is None else n_rows
    src_stride = src.stride(0) * src.element_size()
    dst_stride = dst.stride(0) * dst.element_size()
    _check(lib.mom_copy_rows(_p(src), n_src, src_stride, src_off, _p(idx), n, row_bytes, _p(dst), dst_stride,
                             dst_off, _p(ws), ws.numel(), _s(stream)), "mom_copy_rows")


def mom_gdn_workspace_size(n_rows, n_seg, H, d, dt):
    return lib.mom_gdn_workspace_size(n_rows, n_seg, H, d, dt)


def _gdn(name, q, qidx, k, v, beta, log_alpha, seg_cu, scale, h0, h_final, o, ws, stream):
    n_rows, H, d = k.shape
    _check(getattr(lib, name)(_p(q), _p(qidx), _p(k), _p(v), _p(beta), _p(log_alpha), _p(seg_cu),
                              seg_cu.numel() - 1, n_rows, q.shape[0], H, d, float(scale),
                              dtype_code(k.dtype), _p(h0), _p(h_final), _p(o), _p(ws), ws.numel(),
                              _s(stream)), name)


def mom_gdn_chunk_fwd(q, qidx, k, v, beta, log_alpha, seg_cu, scale, h0, h_final, o, ws, stream=None):
    _gdn("mom_gdn_chunk_fwd", q, qidx, k, v, beta, log_alpha, seg_cu, scale, h0, h_final, o, ws, stream)


def mom_gdn_chunk_prep(q, qidx, k, v, beta, log_alpha, seg_cu, scale, h0, h_final, o, ws, stream=None):
    _gdn("mom_gdn_chunk_prep", q, qidx, k, v, beta, log_alpha, seg_cu, scale, h0, h_final, o, ws, stream)


def mom_gdn_chunk_state(q, qidx, k, v, beta, log_alpha, seg_cu, scale, h0, h_final, o, ws, stream=None):
    _gdn("mom_gdn_chunk_state", q, qidx, k, v, beta, log_alpha, seg_cu, scale, h0, h_final, o, ws, stream)


MOM_RULE_GATED_DELTA, MOM_RULE_GATED_LINEAR = 0, 1
RULES = {"gated_delta": MOM_RULE_GATED_DELTA, "gated_linear": MOM_RULE_GATED_LINEAR}
MOM_GATES_BY_TOKEN, MOM_GATES_BY_ROW = 0, 1


def _memory(name, q, qidx, k, v, beta, log_alpha, seg_cu, scale, rule, h0, h_final, o, ws, stream, gates):
    n_rows, H, d = k.shape
    _check(getattr(lib, name)(_p(q), _p(qidx), _p(k), _p(v), _p(beta), _p(log_alpha), _p(seg_cu),
                              seg_cu.numel() - 1, n_rows, q.shape[0], H, d, float(scale),
                              dtype_code(k.dtype), int(rule), int(gates), _p(h0), _p(h_final), _p(o), _p(ws),
                              ws.numel(), _s(stream)), name)


def mom_memory_chunk_fwd(q, qidx, k, v, beta, log_alpha, seg_cu, scale, rule, h0, h_final, o, ws, stream=None,
                         gates=MOM_GATES_BY_TOKEN):
    _memory("mom_memory_chunk_fwd", q, qidx, k, v, beta, log_alpha, seg_cu, scale, rule, h0, h_final, o, ws, stream,
            gates)


def mom_memory_chunk_prep(q, qidx, k, v, beta, log_alpha, seg_cu, scale, rule, h0, h_final, o, ws, stream=None,
                          gates=MOM_GATES_BY_TOKEN):
    _memory("mom_memory_chunk_prep", q, qidx, k, v, beta, log_alpha, seg_cu, scale, rule, h0, h_final, o, ws, stream,
            gates)


def mom_memory_chunk_state(q, qidx, k, v, beta, log_alpha, seg_cu, scale, rule, h0, h_final, o, ws, stream=None,
                           gates=MOM_GATES_BY_TOKEN):
    _memory("mom_memory_chunk_state", q, qidx, k, v, beta, log_alpha, seg_cu, scale, rule, h0, h_final, o, ws, stream,
            gates)


def mom_memory_chunk_bwd_workspace_size(n_rows, n_seg, H, d):
    return lib.mom_memory_chunk_bwd_workspace_size(n_rows, n_seg, H, d)


def mom_memory_chunk_bwd(q, qidx, k, v, beta, log_alpha, seg_cu, scale, rule, h0, d_o, dh_final,
                         dq, dk, dv, dbeta, dlog_alpha, dh0, ws, stream=None, gates=MOM_GATES_BY_TOKEN):
    """Reverse pass of mom_memory_chunk_fwd: float32 gradients per row."""
    n_rows, H, d = k.shape
    _check(lib.mom_memory_chunk_bwd(_p(q), _p(qidx), _p(k), _p(v), _p(beta), _p(log_alpha), _p(seg_cu),
                                    seg_cu.numel() - 1, n_rows, q.shape[0], H, d, float(scale), dtype_code(k.dtype),
                                    int(rule), int(gates), _p(h0), _p(d_o), _p(dh_final), _p(dq), _p(dk), _p(dv),
                                    _p(dbeta), _p(dlog_alpha), _p(dh0), _p(ws), ws.numel(), _s(stream)),
           "mom_memory_chunk_bwd")


def _pa(t, off_elems=0):
    """Device pointer of a dense CUDA tensor advanced by off_elems elements
    (a column offset into its rows)."""
    p = _p(t)
    return p if p is None or off_elems == 0 else ctypes.c_void_p(p.value + off_elems * t.element_size())


def mom_combine_bwd(dout, o_p, row_of, gate, do_p, dgate, ws, stream=None):
    n_tok, H, d = dout.shape
    _check(lib.mom_combine_bwd(_p(dout), _p(o_p), _p(row_of), _p(gate), n_tok, gate.shape[1], o_p.shape[0], H, d,
                               dtype_code(dout.dtype), _p(do_p), _p(dgate), _p(ws), ws.numel(), _s(stream)),
           "mom_combine_bwd")


def mom_router_bwd(topk_idx, gate, dgate, dlogits, ws, stream=None):
    n_tok, K = topk_idx.shape
    _check(lib.mom_router_bwd(_p(topk_idx), _p(gate), _p(dgate), n_tok, K, dlogits.shape[1], _p(dlogits), _p(ws),
                              ws.numel(), _s(stream)), "mom_router_bwd")


def mom_rows_sum(src, row_of, top_k, base, dst, ws, stream=None):
    """dst[t] = base[t] + sum_j src[row_of[t*top_k+j]] (float32 rows)."""
    n_tok = dst.shape[0]
    W = dst.numel() // max(n_tok, 1)
    _check(lib.mom_rows_sum(_p(src), src.shape[0], _p(row_of), top_k, _p(base), n_tok, W, _p(dst), _p(ws), ws.numel(),
                            _s(stream)), "mom_rows_sum")


def mom_l2norm_bwd(y, dy, norm, dz, col0, stream=None):
    rows, H, d = y.shape
    _check(lib.mom_l2norm_bwd(_p(y), _p(dy), _p(norm), rows, H, d, dtype_code(y.dtype), _p(dz), dz.shape[1], col0,
                              _s(stream)), "mom_l2norm_bwd")


def mom_gates_bwd(beta, log_alpha, dbeta, dlog_alpha, A, dz, col_b, col_a, dala, stream=None):
    n, H = beta.shape
    _check(lib.mom_gates_bwd(_p(beta), _p(log_alpha), _p(dbeta), _p(dlog_alpha), _p(A), n, H, _p(dz), dz.shape[1],
                             col_b, col_a, _p(dala), _s(stream)), "mom_gates_bwd")


def mom_gates_bwd_by_group(beta, log_alpha, dbeta, dlog_alpha, A, group_offset, dz, col_b, col_a, dala,
                           stream=None):
    """mom_gates_bwd with A [n_groups, H] taken per row group."""
    n, H = beta.shape
    _check(lib.mom_gates_bwd_by_group(_p(beta), _p(log_alpha), _p(dbeta), _p(dlog_alpha), _p(A), _p(group_offset),
                                      group_offset.numel() - 1, n, H, _p(dz), dz.shape[1], col_b, col_a, _p(dala),
                                      _s(stream)), "mom_gates_bwd_by_group")


def mom_col_sums_grouped(a, group_offset, out, col0=0, cols=None, stream=None):
    """out [n_groups, cols]: per row group, the sums of a's columns col0 ..."""
    rows, lda = a.shape
    cols = out.shape[-1] if cols is None else cols
    _check(lib.mom_col_sums_grouped(_pa(a, col0), rows, lda, cols, _p(group_offset), group_offset.numel() - 1,
                                    _p(out), _s(stream)), "mom_col_sums_grouped")


def mom_mem_gate_proj_groups(x, group_offset, group_mem, w_gate_mem, A_mem, b_a_mem, beta_p, log_alpha_p, ws,
                             perm_token=None, stream=None):
    """Per-memory gates of rows grouped by (group_offset, group_mem); row r
    reads x row perm_token[r] (None: row r)."""
    n_rows, H = beta_p.shape
    _check(lib.mom_mem_gate_proj_groups(_p(x), x.shape[0], _p(perm_token), n_rows, _p(group_offset), _p(group_mem),
                                        group_mem.numel(), _p(w_gate_mem), _p(A_mem), _p(b_a_mem), w_gate_mem.shape[0],
                                        dtype_code(x.dtype), x.shape[1], H, _p(beta_p), _p(log_alpha_p), _p(ws),
                                        ws.numel(), _s(stream)), "mom_mem_gate_proj_groups")


def mom_col_sums(a, out, col0=0, stream=None):
    """out[c] = sum over rows of a[:, col0 + c]."""
    rows, lda = a.shape
    _check(lib.mom_col_sums(_pa(a, col0), rows, lda, out.numel(), _p(out), _s(stream)), "mom_col_sums")


def mom_gemm_grouped(trans_a, A, B, C, M, N, K, group_offset, group_index, n_groups, ws, a_col=0, b_rows=None,
                     total_rows=0, b_group_stride=0, c_group_stride=0, accumulate=False, stream=None):
    """float32 C (+)= op(A) B over groups (see include/mom.h); A, C float32
    2-D (A read from column a_col), B the weights or tokens (2-D or 3-D,
    rows of B.shape[-1])."""
    ldb = B.shape[-1]
    _check(lib.mom_gemm_grouped(int(trans_a), _pa(A, a_col), A.shape[1], _p(B), ldb, dtype_code(B.dtype), _p(b_rows),
                                B.numel() // ldb, _p(C), C.shape[-1], M, N, K, total_rows, _p(group_offset),
                                _p(group_index), n_groups, b_group_stride, c_group_stride, int(accumulate), _p(ws),
                                ws.numel(), _s(stream)), "mom_gemm_grouped")


def mom_combine_unpermute(o_sh, o_p, row_of, topk_gate, out, ws, stream=None):
    n_tok, H, d = o_sh.shape
    top_k = topk_gate.shape[1]
    _check(lib.mom_combine_unpermute(_p(o_sh), _p(o_p), _p(row_of), _p(topk_gate), n_tok, top_k, H, d,
                                     dtype_code(o_sh.dtype), _p(out), _p(ws), ws.numel(), _s(stream)),
           "mom_combine_unpermute")


# -------------------------------------------------- the Gated DeltaNet block

def mom_block_proj(x, perm, mem_offset, w_shared4, w_kv, H, d, top_k, q, k_sh, v_sh, g, k_p, v_p, ws, stream=None):
    """Unnormalised q, k_sh, v_sh, the output gate g (x W_shared4^T) and the
    routed rows' unnormalised k_p, v_p."""
    n_tok, d_model = x.shape
    _check(lib.mom_block_proj(_p(x), _p(perm), _p(mem_offset), _p(w_shared4), _p(w_kv), dtype_code(x.dtype), n_tok,
                              d_model, H, d, w_kv.shape[0], top_k, _p(q), _p(k_sh), _p(v_sh), _p(g), _p(k_p), _p(v_p),
                              _p(ws), ws.numel(), _s(stream)), "mom_block_proj")


def mom_short_conv(z, seg_cu, w, out, ws, seg_per_group=None, head_dim=0, l2norm=False, stream=None, n_rows=None):
    """out = SiLU(causal depthwise conv of z along the segments of seg_cu)
    (then the per-head L2 norm when l2norm); w [n_groups, width, C] float32
    (tap-major), segment s using group s // seg_per_group (default: one
    group)."""
    n = z.shape[0] if n_rows is None else n_rows
    C = z.numel() // max(z.shape[0], 1)
    n_seg = seg_cu.numel() - 1
    n_groups, width, _ = w.shape
    spg = n_seg if seg_per_group is None else seg_per_group
    _check(lib.mom_short_conv(_p(z), n, C, _p(seg_cu), n_seg, spg, n_groups, _p(w), width, head_dim, int(l2norm),
                              dtype_code(z.dtype), _p(out), _p(ws), ws.numel(), _s(stream)), "mom_short_conv")


def mom_short_conv_batch(problems, head_dim, ws, stream=None):
    """problems: a list of dicts with z, out, seg_cu, w and optionally
    seg_per_group (default: one group), l2norm; the same channel count and
    width for all."""
    arr = (MomConvProblem * len(problems))()
    C = width = None
    for i, q in enumerate(problems):
        z, seg_cu, w = q["z"], q["seg_cu"], q["w"]
        n_seg = seg_cu.numel() - 1
        C = z.numel() // max(z.shape[0], 1)
        width = w.shape[1]
        arr[i] = MomConvProblem(_p(z).value, _p(q["out"]).value, z.shape[0], _p(seg_cu).value, n_seg,
                                q.get("seg_per_group") or n_seg, w.shape[0], _p(w).value, int(q.get("l2norm", False)))
    _check(lib.mom_short_conv_batch(arr, len(problems), C, width, head_dim, dtype_code(problems[0]["z"].dtype),
                                    _p(ws), ws.numel(), _s(stream)), "mom_short_conv_batch")


def mom_combine_norm_gate(o_sh, o_p, row_of, topk_gate, g, w_norm, eps, out, ws, stream=None):
    n_tok, H, d = o_sh.shape
    top_k = topk_gate.shape[1]
    _check(lib.mom_combine_norm_gate(_p(o_sh), _p(o_p), _p(row_of), _p(topk_gate), _p(g), _p(w_norm), eps, n_tok,
                                     top_k, H, d, dtype_code(o_sh.dtype), _p(out), _p(ws), ws.numel(), _s(stream)),
           "mom_combine_norm_gate")


def mom_linear(x, w, y, ws, stream=None):
    """y = x w^T (x [n, k_in], w [n_out, k_in])."""
    n, k_in = x.shape
    _check(lib.mom_linear(_p(x), _p(w), dtype_code(x.dtype), n, k_in, w.shape[0], _p(y), _p(ws), ws.numel(),
                          _s(stream)), "mom_linear")


def mom_norm_gate_bwd(o_sh, o_p, row_of, topk_gate, g, w_norm, eps, d_y, d_o, dg, dw_norm, ws, stream=None,
                      ldg=None):
    """d_o [N, H, d] (dt), dg [N, ldg] float32 (columns 0 .. H*d of each row),
    dw_norm [d] float32."""
    n_tok, H, d = o_sh.shape
    top_k = 0 if topk_gate is None else topk_gate.shape[1]
    ldg = dg.stride(0) if ldg is None else ldg
    _check(lib.mom_norm_gate_bwd(_p(o_sh), _p(o_p), _p(row_of), _p(topk_gate), _p(g), _p(w_norm), eps, _p(d_y), n_tok,
                                 top_k, H, d, dtype_code(o_sh.dtype), _p(d_o), ctypes.c_void_p(dg.data_ptr()), ldg,
                                 _p(dw_norm), _p(ws), ws.numel(), _s(stream)), "mom_norm_gate_bwd")


def mom_short_conv_bwd(problems, head_dim, ws, stream=None):
    """problems: dicts with z, dout, dz (a 2-D float32 tensor, possibly a
    column slice: its row stride and offset are passed), seg_cu, w, dw and
    optionally seg_per_group, l2norm (da: reserved, ignored)."""
    arr = (MomConvBwdProblem * len(problems))()
    C = width = None
    for i, q in enumerate(problems):
        z, w, dz = q["z"], q["w"], q["dz"]
        n_seg = q["seg_cu"].numel() - 1
        C = 1
        for n in z.shape[1:]:
            C *= n
        width = w.shape[1]
        if not dz.is_cuda or dz.dtype != torch.float32 or dz.dim() != 2 or dz.stride(1) != 1:
            raise ValueError("MoM: dz must be a 2-D float32 CUDA tensor of unit column stride")
        ldz = dz.stride(0)
        col0 = dz.storage_offset() % ldz if ldz else 0
        da = q.get("da")
        arr[i] = MomConvBwdProblem(_p(z).value, _p(q["dout"]).value, None if da is None else _p(da).value,
                                   dz.data_ptr() - col0 * dz.element_size(), ldz, col0, z.shape[0],
                                   _p(q["seg_cu"]).value, n_seg, q.get("seg_per_group") or n_seg, w.shape[0],
                                   _p(w).value, _p(q["dw"]).value, int(q.get("l2norm", False)))
    _check(lib.mom_short_conv_bwd(arr, len(problems), C, width, head_dim, dtype_code(problems[0]["z"].dtype), _p(ws),
                                  ws.numel(), _s(stream)), "mom_short_conv_bwd")


def mom_convert(src, dst, stream=None):
    _check(lib.mom_convert(_p(src), dtype_code(src.dtype), _p(dst), dtype_code(dst.dtype), src.numel(), _s(stream)),
           "mom_convert")


def mom_block_decode_workspace_size(B, d_model, H, d, n_mem, top_k):
    return lib.mom_block_decode_workspace_size(B, d_model, H, d, n_mem, top_k)


def mom_block_decode_step(x, weights, block_weights, width, eps, H, d, n_mem, top_k, scale, rule, state, conv_sh,
                          conv_mem, y, topk_idx, ws, stream=None, mem_gates=None):
    """One token per sequence through the block; state, conv_sh, conv_mem
    updated in place.  weights / block_weights / mem_gates: MomWeights,
    MomBlockWeights, MomMemoryGates (or None)."""
    B, d_model = x.shape
    _check(lib.mom_block_decode_step(_p(x), ctypes.byref(weights), ctypes.byref(block_weights),
                                     None if mem_gates is None else ctypes.byref(mem_gates), width, eps, B, d_model, H,
                                     d, n_mem, top_k, scale, dtype_code(x.dtype), rule, _p(state), _p(conv_sh),
                                     _p(conv_mem), _p(y), _p(topk_idx), _p(ws), ws.numel(), _s(stream)),
           "mom_block_decode_step")


def mom_block_conv_state(q_raw, k_sh_raw, v_sh_raw, k_p_raw, v_p_raw, cu_seqlens, seg_cu, n_mem, top_k, width,
                         conv_sh, conv_mem, ws, stream=None):
    n_tok = q_raw.shape[0]
    C = q_raw.numel() // max(n_tok, 1)
    _check(lib.mom_block_conv_state(_p(q_raw), _p(k_sh_raw), _p(v_sh_raw), _p(k_p_raw), _p(v_p_raw), n_tok, top_k,
                                    _p(cu_seqlens), _p(seg_cu), cu_seqlens.numel() - 1, n_mem, C, width,
                                    dtype_code(q_raw.dtype), _p(conv_sh), _p(conv_mem), _p(ws), ws.numel(),
                                    _s(stream)), "mom_block_conv_state")


def mom_decode_workspace_size(B, d_model, H, d, n_mem, top_k):
    return lib.mom_decode_workspace_size(B, d_model, H, d, n_mem, top_k)


def mom_decode_step(x, weights: MomWeights, H, d, n_mem, top_k, scale, state, out, topk_idx, ws, stream=None):
    B, d_model = x.shape
    _check(lib.mom_decode_step(_p(x), ctypes.byref(weights), B, d_model, H, d, n_mem, top_k, float(scale),
                               dtype_code(x.dtype), _p(state), _p(out), _p(topk_idx), _p(ws), ws.numel(),
                               _s(stream)), "mom_decode_step")


def mom_decode_step_rule(x, weights: MomWeights, H, d, n_mem, top_k, scale, rule, state, out, topk_idx, ws,
                         stream=None, mem_gates: Optional[MomMemoryGates] = None):
    B, d_model = x.shape
    mg = ctypes.byref(mem_gates) if mem_gates is not None else None
    _check(lib.mom_decode_step_rule(_p(x), ctypes.byref(weights), mg, B, d_model, H, d, n_mem, top_k, float(scale),
                                    dtype_code(x.dtype), int(rule), _p(state), _p(out), _p(topk_idx), _p(ws),
                                    ws.numel(), _s(stream)), "mom_decode_step_rule")
