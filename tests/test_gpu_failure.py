"""The failure path of the pipelined kernels, exercised without a fault: a
bounded barrier wait on a barrier that nothing signals runs out after a short
limit, the kernel records MOM_DEVERR_TIMEOUT in the workspace and returns,
the host reads the record, and the context keeps working (a layer forward
right after it still matches the oracle)."""
import pytest
import torch

from mixture_memories_layer_b200 import binding as B
from tests.test_gpu_layer import _check_layer, _small
from tests.gpu_helpers import run_layer

pytestmark = pytest.mark.gpu


def test_wait_that_nothing_ends_times_out_and_is_reported():
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    limit = 2_000_000                      # SM cycles: about a millisecond
    B.mom_selftest_wait_timeout(ws, limit)
    torch.cuda.synchronize()               # the kernel returned on its own
    assert B.mom_get_error(ws) == (B.MOM_DEVERR_TIMEOUT, B.MOM_SELFTEST_WAIT_SITE)
    B.mom_clear_error(ws)
    assert B.mom_get_error(ws) == (0, 0)
    # the context is intact: a full layer call right after still matches the oracle
    w, p = _small(128, lens=(70, 9))
    lay, res = run_layer(w, p)
    assert lay.device_errors() == {}
    _check_layer(w, p, res)


def test_selftest_rejects_bad_arguments():
    ws = B.new_workspace(B.MOM_WS_HEADER_BYTES)
    with pytest.raises(B.MomError):
        B.mom_selftest_wait_timeout(ws, 0)
    with pytest.raises(B.MomError):
        B.mom_selftest_wait_timeout(ws[:16], 1000)
