"""The C-ABI library loads, exports every entry point that include/mom.h
declares, and rejects bad arguments on the host before any launch (these
calls never reach the GPU, so they run without one)."""
import ctypes
import os
import re

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "mom.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^(?:mom_status|size_t|uint64_t|const char\*)\s+(mom_\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def lib():
    from mixture_memories_layer_b200 import build
    build.build(verbose=False)
    from mixture_memories_layer_b200 import binding
    return binding


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib.lib, n), n
    assert set(names) == set(lib.SIGNATURES), "binding signatures out of sync with mom.h"


def test_host_validation_rejects_bad_arguments(lib):
    L, B = lib.lib, lib
    fake = ctypes.c_void_p(0x10000)       # never dereferenced: validation fails first
    s = L.mom_router_topk(fake, fake, None, B.MOM_BF16, 10, 64, 4, 5, fake, fake, None, None)
    assert s == B.MOM_ERR_ARG                                   # top_k > n_mem
    s = L.mom_router_topk(fake, fake, None, B.MOM_BF16, 10, 60, 4, 2, fake, fake, None, None)
    assert s == B.MOM_ERR_ARG                                   # d_model % 8
    s = L.mom_router_topk(fake, fake, None, 7, 10, 64, 4, 2, fake, fake, None, None)
    assert s == B.MOM_ERR_ARG                                   # dtype
    s = L.mom_kv_proj_grouped(*([fake] * 8), B.MOM_BF16, 10, 256, 2, 96, 4, 2, *([fake] * 8), 4096, None)
    assert s == B.MOM_ERR_UNSUPPORTED                           # d = 96
    s = L.mom_gdn_chunk_fwd(*([fake] * 7), 3, 10, 10, 2, 64, 1.0, B.MOM_BF16, None, None, fake, fake, 8, None)
    assert s == B.MOM_ERR_ARG                                   # workspace too small
    s = L.mom_permute(fake, 10, 2, 4, None, 2, fake, fake, fake, fake, fake, 1 << 20, None)
    assert s == B.MOM_ERR_ARG                                   # no cu_seqlens with 2 sequences
    s = L.mom_get_error(None, None, None, None)
    assert s == B.MOM_ERR_ARG
    assert L.mom_status_string(B.MOM_ERR_UNSUPPORTED) == b"unsupported shape or type"


def test_workspace_sizes_are_monotone(lib):
    L = lib.lib
    a = L.mom_permute_workspace_size(1000, 2, 4, 3)
    b = L.mom_permute_workspace_size(100000, 2, 4, 3)
    assert lib.MOM_WS_HEADER_BYTES <= a <= b
    assert L.mom_decode_workspace_size(256, 1024, 4, 256, 8, 2) > L.mom_decode_workspace_size(16, 1024, 4, 256, 8, 2)


def test_host_validation_at_the_size_limits(lib):
    """The largest problems the ABI takes: (token, slot) pairs are counted in
    int32, so n_tok * top_k must stay below 2^31; M and H have fixed caps; the
    allocation-free reordering holds at most MOM_PERMUTE_NOALLOC_MAX_TOKENS
    tokens.  Past a limit the call returns an error and launches nothing."""
    L, B = lib.lib, lib
    fake = ctypes.c_void_p(0x10000)       # never dereferenced: validation fails first
    big = 1 << 30
    s = L.mom_permute(fake, big, 2, 4, fake, 1, fake, fake, fake, fake, fake, 1 << 20, None)
    assert s == B.MOM_ERR_UNSUPPORTED                           # n_tok * top_k = 2^31
    s = L.mom_kv_proj_grouped(*([fake] * 8), B.MOM_BF16, big, 256, 2, 64, 4, 2, *([fake] * 8), 4096, None)
    assert s == B.MOM_ERR_UNSUPPORTED
    s = L.mom_permute(fake, 10, 2, 33, fake, 1, fake, fake, fake, fake, fake, 1 << 20, None)
    assert s == B.MOM_ERR_ARG                                   # M = 33 > MOM_MAX_MEM
    s = L.mom_router_topk(fake, fake, None, B.MOM_BF16, 10, 64, 33, 2, fake, fake, None, None)
    assert s == B.MOM_ERR_ARG
    s = L.mom_kv_proj_grouped(*([fake] * 8), B.MOM_BF16, 10, 256, 65, 64, 4, 2, *([fake] * 8), 4096, None)
    assert s == B.MOM_ERR_ARG                                   # H = 65 > MOM_MAX_HEADS
    s = L.mom_permute_noalloc(fake, (1 << 20) + 1, 2, 4, fake, 1, fake, fake, fake, fake, fake, None)
    assert s == B.MOM_ERR_UNSUPPORTED                           # past the static scratch
    s = L.mom_permute(fake, -1, 2, 4, fake, 1, fake, fake, fake, fake, fake, 1 << 20, None)
    assert s == B.MOM_ERR_ARG                                   # negative token count


def test_binding_refuses_host_tensors(lib):
    import torch
    with pytest.raises(ValueError, match="CUDA tensors"):
        lib._p(torch.zeros(4))
    assert lib._p(None) is None


def test_block_calls_validate_on_the_host(lib):
    """The Gated DeltaNet block's calls refuse bad shapes before any launch."""
    L, B = lib.lib, lib
    fake, other = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x20000)
    conv = lambda z, out, C, width, hd, l2, dt=B.MOM_BF16, spg=1, ng=1: L.mom_short_conv(
        z, 10, C, fake, 2, spg, ng, fake, width, hd, l2, dt, out, fake, 4096, None)
    assert conv(fake, other, 256, 5, 64, 1) == B.MOM_ERR_UNSUPPORTED          # width > 4
    assert conv(fake, other, 256, 4, 64, 1, dt=B.MOM_F32) == B.MOM_ERR_UNSUPPORTED
    assert conv(fake, other, 256, 4, 96, 1) == B.MOM_ERR_ARG                  # head_dim not a power of two
    assert conv(fake, other, 252, 4, 64, 0) == B.MOM_ERR_ARG                  # channels % 8
    assert conv(fake, fake, 256, 4, 64, 1) == B.MOM_ERR_ARG                   # in place
    assert conv(fake, other, 256, 4, 64, 1, spg=0) == B.MOM_ERR_ARG           # no segments per group
    s = L.mom_combine_norm_gate(*([fake] * 6), 1e-5, 10, 2, 2, 96, B.MOM_BF16, fake, fake, 4096, None)
    assert s == B.MOM_ERR_ARG                                                 # d = 96
    s = L.mom_combine_norm_gate(*([fake] * 6), -1.0, 10, 2, 2, 64, B.MOM_BF16, fake, fake, 4096, None)
    assert s == B.MOM_ERR_ARG                                                 # eps < 0
    s = L.mom_combine_norm_gate(*([fake] * 6), 1e-5, 10, 2, 2, 64, B.MOM_F32, fake, fake, 4096, None)
    assert s == B.MOM_ERR_UNSUPPORTED
    s = L.mom_linear(fake, fake, B.MOM_BF16, 10, 100, 256, fake, fake, 8, None)
    assert s == B.MOM_ERR_ARG                                                 # workspace too small
    s = L.mom_block_proj(*([fake] * 5), B.MOM_BF16, 10, 256, 2, 96, 4, 2, *([fake] * 6), fake, 4096, None)
    assert s == B.MOM_ERR_UNSUPPORTED                                         # d = 96


def test_block_backward_calls_validate_on_the_host(lib):
    """The block's reverse-pass calls refuse bad shapes and pointers before
    any launch."""
    L, B = lib.lib, lib
    fake, odd = ctypes.c_void_p(0x10000), ctypes.c_void_p(0x10004)
    ng = lambda o_p=fake, w_norm=fake, eps=1e-5, top_k=2, d=64, dt=B.MOM_BF16, dg=fake, ldg=128, ws_bytes=4096: \
        L.mom_norm_gate_bwd(fake, o_p, fake, fake, fake, w_norm, eps, fake, 10, top_k, 2, d, dt, fake, dg, ldg,
                            fake, fake, ws_bytes, None)
    assert ng(d=96) == B.MOM_ERR_ARG                                          # d not a power of two
    assert ng(eps=-1.0) == B.MOM_ERR_ARG
    assert ng(ldg=100) == B.MOM_ERR_ARG                                       # ldg < H d
    assert ng(ldg=130) == B.MOM_ERR_ARG                                       # rows not 16-byte aligned
    assert ng(dt=B.MOM_F32) == B.MOM_ERR_UNSUPPORTED
    assert ng(w_norm=None) == B.MOM_ERR_ARG
    assert ng(dg=odd) == B.MOM_ERR_ARG
    assert ng(o_p=None) == B.MOM_ERR_ARG                                      # routed rows missing, top_k 2
    assert ng(ws_bytes=8) == B.MOM_ERR_ARG

    def conv(**kw):
        q = dict(z=fake.value, dout=fake.value, da=fake.value, dz=fake.value, ldz=256, col0=0, n_rows=10,
                 seg_cu=fake.value, n_seg=2, seg_per_group=1, n_groups=2, w=fake.value, dw=fake.value, l2norm=1)
        channels = kw.pop("channels", 256)
        width = kw.pop("width", 4)
        head_dim = kw.pop("head_dim", 64)
        n = kw.pop("n", 1)
        q.update(kw)
        arr = (B.MomConvBwdProblem * 9)(*[B.MomConvBwdProblem(**q)] * 9)
        return L.mom_short_conv_bwd(arr, n, channels, width, head_dim, B.MOM_BF16, fake, 4096, None)
    assert conv(width=5) == B.MOM_ERR_UNSUPPORTED
    assert conv(n=9) == B.MOM_ERR_UNSUPPORTED                                 # more than 8 problems
    assert conv(n=0) == B.MOM_ERR_ARG
    assert conv(channels=252) == B.MOM_ERR_ARG                                # channels % 8
    assert conv(head_dim=96) == B.MOM_ERR_ARG                                 # with the L2 norm
    assert conv(ldz=200) == B.MOM_ERR_ARG                                     # ldz < col0 + channels
    assert conv(col0=2, ldz=260) == B.MOM_ERR_ARG                             # col0 not 16-byte aligned
    assert conv(seg_per_group=0) == B.MOM_ERR_ARG
    assert conv(l2norm=2) == B.MOM_ERR_ARG
    assert conv(dz=0) == B.MOM_ERR_ARG
    assert conv(w=odd.value) == B.MOM_ERR_ARG
    assert L.mom_convert(fake, B.MOM_F32, fake, B.MOM_BF16, -1, None) == B.MOM_ERR_ARG
    assert L.mom_convert(fake, B.MOM_F32, fake, B.MOM_BF16, 0, None) == B.MOM_OK  # nothing to do
    assert L.mom_convert(None, B.MOM_F32, fake, B.MOM_BF16, 5, None) == B.MOM_ERR_ARG


def test_grouped_gate_calls_validate_on_the_host(lib):
    """The per-memory gates' grouped calls (backward and memory-parallel
    owner) refuse bad shapes and pointers before any launch."""
    L, B = lib.lib, lib
    fake = ctypes.c_void_p(0x10000)
    gb = lambda n_groups=2, ldz=4, col_b=0, col_a=2, A=fake: L.mom_gates_bwd_by_group(
        fake, fake, fake, fake, A, fake, n_groups, 10, 2, fake, ldz, col_b, col_a, fake, None)
    assert gb(n_groups=0) == B.MOM_ERR_ARG
    assert gb(ldz=3) == B.MOM_ERR_ARG                                         # col_a + H > ldz
    assert gb(col_b=-1) == B.MOM_ERR_ARG
    assert gb(A=None) == B.MOM_ERR_ARG
    cs = lambda n_groups=2, lda=4, cols=2, goff=fake: L.mom_col_sums_grouped(fake, 10, lda, cols, goff, n_groups,
                                                                             fake, None)
    assert cs(n_groups=0) == B.MOM_ERR_ARG
    assert cs(lda=1) == B.MOM_ERR_ARG                                         # lda < cols
    assert cs(goff=None) == B.MOM_ERR_ARG
    assert cs(cols=0) == B.MOM_OK                                             # nothing to sum
    mg = lambda n_x=10, perm=None, n_groups=2, d_model=64, ws_bytes=4096: L.mom_mem_gate_proj_groups(
        fake, n_x, perm, 10, fake, fake, n_groups, fake, fake, fake, 4, B.MOM_BF16, d_model, 2, fake, fake, fake,
        ws_bytes, None)
    assert mg(n_groups=33) == B.MOM_ERR_ARG                                   # more groups than MOM_MAX_MEM
    assert mg(n_groups=0) == B.MOM_ERR_ARG
    assert mg(d_model=60) == B.MOM_ERR_ARG                                    # d_model % 8
    assert mg(n_x=5) == B.MOM_ERR_ARG                                         # row r reads x row r: n_x < n_rows
    assert mg(ws_bytes=8) == B.MOM_ERR_ARG
