"""mom_permute_noalloc: the reordering for callers that cannot allocate
device memory (for example a plug-in whose host engine owns all device
memory through its own pool, or a serving loop where cudaMalloc is not
allowed because it can block the host and synchronise the device).

It takes no workspace; its scratch is a fixed array inside the library that
every call on the device shares.  These tests call it through the C ABI
twice in a row, on two different problems, and check each result against
the workspace-taking mom_permute on the same inputs (integer outputs: bit
for bit).  The file is named to run last, after every other test, and also
passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from mixture_memories_layer_b200 import binding as B

pytestmark = pytest.mark.gpu


def _problem(rng, n_tok, M, K, lens):
    idx = np.stack([rng.choice(M, K, replace=False) for _ in range(n_tok)]).astype(np.int32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    assert cu[-1] == n_tok
    return torch.as_tensor(idx).cuda(), torch.as_tensor(cu).cuda()


def _outputs(n_tok, M, K, S):
    i32 = dict(dtype=torch.int32, device="cuda")
    return (torch.full((n_tok * K,), -1, **i32), torch.full((n_tok * K,), -1, **i32),
            torch.full((M + 1,), -1, **i32), torch.full((M * S + 1,), -1, **i32))


def _reference(idx, M, cu):
    n_tok, K = idx.shape
    S = cu.numel() - 1
    perm, row_of, offs, seg = _outputs(n_tok, M, K, S)
    ws = B.new_workspace(B.mom_permute_workspace_size(n_tok, K, M, S))
    B.mom_permute(idx, M, cu, perm, row_of, offs, seg, ws)
    return perm, row_of, offs, seg


def test_noalloc_matches_workspace_permute_two_calls_in_a_row():
    assert torch.cuda.is_available(), "needs a CUDA device"
    rng = np.random.default_rng(2024)
    # a larger problem first, then a smaller one with fewer memories: the
    # second call must not see anything the first left in the shared array
    cases = [(5000, 8, 2, [1200, 0, 3000, 800]), (700, 4, 2, [300, 400])]
    status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    for n_tok, M, K, lens in cases:
        idx, cu = _problem(rng, n_tok, M, K, lens)
        S = len(lens)
        perm, row_of, offs, seg = _outputs(n_tok, M, K, S)
        B.mom_permute_noalloc(idx, M, cu, perm, row_of, offs, seg, status)
        r_perm, r_row, r_offs, r_seg = _reference(idx, M, cu)
        torch.cuda.synchronize()
        assert torch.equal(perm, r_perm)
        assert torch.equal(row_of, r_row)
        assert torch.equal(offs, r_offs)
        assert torch.equal(seg, r_seg)
        assert status.tolist() == [0, 0]


def test_noalloc_four_launch_path_matches_workspace_permute():
    """A tile-count table above the single cooperative launch's limit
    (32 memories x 274 tiles of 256 tokens) takes the four-launch path, whose
    scan also keeps its per-tile bases in the fixed array: bit for bit
    against mom_permute, twice in a row."""
    rng = np.random.default_rng(77)
    n_tok, M, K = 70000, 32, 2
    lens = [30000, 1, 0, 39999]
    status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    for _ in range(2):
        idx, cu = _problem(rng, n_tok, M, K, lens)
        perm, row_of, offs, seg = _outputs(n_tok, M, K, len(lens))
        B.mom_permute_noalloc(idx, M, cu, perm, row_of, offs, seg, status)
        ref = _reference(idx, M, cu)
        torch.cuda.synchronize()
        for got, want in zip((perm, row_of, offs, seg), ref):
            assert torch.equal(got, want)
        assert status.tolist() == [0, 0]


def test_noalloc_reports_a_bad_memory_index_in_status_out():
    """A memory index >= M planted on the host is dropped and reported in
    status_out as {MOM_DEVERR_MEM_INDEX, token}; the next clean call starts
    from a cleared record and reports {0, 0}."""
    rng = np.random.default_rng(5)
    n_tok, M, K = 300, 4, 2
    idx, cu = _problem(rng, n_tok, M, K, [n_tok])
    idx[123, 1] = 9
    status = torch.full((2,), -1, dtype=torch.int32, device="cuda")
    perm, row_of, offs, seg = _outputs(n_tok, M, K, 1)
    B.mom_permute_noalloc(idx, M, cu, perm, row_of, offs, seg, status)
    torch.cuda.synchronize()
    assert status.tolist() == [B.MOM_DEVERR_MEM_INDEX, 123]
    assert int(offs[-1]) == n_tok * K - 1            # the bad pair was dropped
    assert int(row_of[123 * K + 1]) == -1
    idx[123, 1] = (int(idx[123, 0]) + 1) % M
    B.mom_permute_noalloc(idx, M, cu, perm, row_of, offs, seg, status)
    ref = _reference(idx, M, cu)
    torch.cuda.synchronize()
    assert status.tolist() == [0, 0]
    for got, want in zip((perm, row_of, offs, seg), ref):
        assert torch.equal(got, want)


def test_noalloc_refuses_problems_beyond_its_fixed_scratch():
    n_tok = B.MOM_PERMUTE_NOALLOC_MAX_TOKENS + 1
    idx = torch.zeros((n_tok, 1), dtype=torch.int32, device="cuda")
    perm = torch.empty(n_tok, dtype=torch.int32, device="cuda")
    offs = torch.empty(2, dtype=torch.int32, device="cuda")
    with pytest.raises(B.MomError, match="unsupported"):
        B.mom_permute_noalloc(idx, 1, None, perm, perm, offs, offs)
