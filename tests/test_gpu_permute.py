"""GPU reordering (mom_permute) against the oracle's stable counting sort,
bit-exact ("MoM: Mixture-of-Memories Fixes Linear Attention Recall", Solving
scatter-gather without new kernels), on both of its launch paths: the single
cooperative launch (memory x tile table up to 8192 entries) and the
four-launch path beyond it; many ragged and empty sequences; no tokens."""
import numpy as np
import pytest
import torch

from mixture_memories_layer_b200 import binding as B
from oracle import mom_oracle as orc

pytestmark = pytest.mark.gpu


def _run(idx, M, cu):
    n_tok, K = idx.shape
    S = len(cu) - 1
    i32 = dict(dtype=torch.int32, device="cuda")
    perm = torch.full((max(n_tok * K, 1),), -1, **i32)
    row_of = torch.full((max(n_tok * K, 1),), -1, **i32)
    offs = torch.empty(M + 1, **i32)
    seg = torch.empty(M * S + 1, **i32)
    ws = B.new_workspace(B.mom_permute_workspace_size(n_tok, K, M, S))
    B.mom_permute(torch.as_tensor(idx).cuda(), M, torch.as_tensor(cu).cuda(), perm, row_of, offs, seg, ws)
    torch.cuda.synchronize()
    assert B.mom_get_error(ws) == (0, 0)
    return perm.cpu().numpy()[:n_tok * K], row_of.cpu().numpy()[:n_tok * K], offs.cpu().numpy(), seg.cpu().numpy()


def _routing(rng, n_tok, M, K):
    # K distinct memories per token, skewed towards the low ids
    w = 1.0 / np.arange(1, M + 1)
    keys = rng.random((n_tok, M)) ** (1.0 / w)
    return np.argsort(-keys, axis=1)[:, :K].astype(np.int32)


def _check(idx, M, cu):
    got = _run(idx, M, cu)
    ref = orc.permute(idx, M, cu)
    for g, r, name in zip(got, ref, ("perm_token", "row_of", "mem_offset", "seg_cu")):
        assert np.array_equal(g, r), name


@pytest.mark.parametrize("n_tok,M,K", [(300_000, 32, 4), (70_000, 32, 2)])
def test_four_launch_path(n_tok, M, K):
    """More than 8192 (memory, tile) entries: the count / scan / scatter /
    bounds launches."""
    assert M * ((n_tok + 255) // 256) > 8192
    rng = np.random.default_rng(n_tok)
    idx = _routing(rng, n_tok, M, K)
    lens = rng.integers(0, 3000, 400)
    cu = np.concatenate([[0], np.cumsum(lens)])
    cu = cu[cu < n_tok]
    cu = np.concatenate([cu, [n_tok]]).astype(np.int32)
    _check(idx, M, cu)


def test_cooperative_path_many_ragged_sequences():
    rng = np.random.default_rng(7)
    n_tok, M, K = 20_000, 16, 4
    idx = _routing(rng, n_tok, M, K)
    lens = rng.integers(0, 60, 2000)            # many short sequences, some empty
    cu = np.concatenate([[0], np.cumsum(lens)])
    cu = cu[cu < n_tok]
    cu = np.concatenate([cu, [n_tok, n_tok]]).astype(np.int32)   # a trailing empty sequence
    _check(idx, M, cu)


def test_no_tokens():
    idx = np.zeros((0, 2), dtype=np.int32)
    cu = np.array([0, 0, 0], dtype=np.int32)
    perm, row_of, offs, seg = _run(idx, 4, cu)
    assert offs.tolist() == [0] * 5
    assert seg.tolist() == [0] * (4 * 2 + 1)
