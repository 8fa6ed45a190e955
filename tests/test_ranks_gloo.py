"""The N > 1 path of bench.py on CPU: two ranks over gloo (127.0.0.1).

The layer shards by sequence (weak scaling): every rank gets the replicated
weights and its own batch, nothing on the data path crosses ranks, and the
only collectives are the barrier and the max over ranks of the timed
region.  These tests run that plumbing -- rank environment, process group,
barrier, max, per-rank batches, the whole-job throughput, the reference
arm's rank-0-only rule -- in two processes without a GPU.
"""
import json
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench
    from mixture_memories_layer_b200 import synth
    ranks = bench.Ranks("gloo", timeout_s=60)
    ranks.barrier()
    # the slowest rank's time is every rank's step time
    mx = ranks.max(10.0 * (rank + 1))
    w = synth.WORKLOADS["tiny_fp32"]
    p = bench.rank_problem(w, rank)
    value = bench.aggregate_throughput(w.n_tokens, ranks.world, 3, mx)
    # the reference arm: only rank 0 times the oracle; the others return at once
    ref = None
    if rank != 0:
        class A:
            steps, warmup, gpus = 1, 3, world
        ref = bench.reference_arm(A())
    ranks.barrier()
    ranks.close()
    rec = {"rank": rank, "world": ranks.world, "max": mx, "value": value,
           "x_sum": float(np.asarray(p["x"], dtype=np.float64).sum()), "x_shape": list(p["x"].shape),
           "w_sum": float(np.asarray(p["w_r"], dtype=np.float64).sum()), "ref_is_none": ref is None}
    with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as fh:
        json.dump(rec, fh)


def test_two_ranks_over_gloo():
    from tests.conftest import ROOT
    out_dir = os.path.join(ROOT, "mixture_memories_layer_b200", "_build", "gloo_ranks")   # git-ignored scratch
    os.makedirs(out_dir, exist_ok=True)
    for r in range(2):
        stale = os.path.join(out_dir, "rank%d.json" % r)
        if os.path.exists(stale):
            os.remove(stale)
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out_dir)) for r in range(2)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=180)
        if pr.is_alive():
            pr.kill()
            pytest.fail("a rank did not finish")
        assert pr.exitcode == 0
    recs = [json.load(open(os.path.join(out_dir, "rank%d.json" % r))) for r in range(2)]
    assert all(r["world"] == 2 for r in recs)
    assert all(r["max"] == 20.0 for r in recs)                  # max over ranks
    assert recs[0]["x_shape"] == recs[1]["x_shape"]            # same per-rank work
    assert recs[0]["x_sum"] != recs[1]["x_sum"]                # ... on each rank's own tokens
    assert recs[0]["w_sum"] == recs[1]["w_sum"]                # replicated weights
    # whole-job throughput: both ranks' tokens over the slowest rank's time
    from mixture_memories_layer_b200 import synth
    n = synth.WORKLOADS["tiny_fp32"].n_tokens
    assert recs[0]["value"] == pytest.approx(n * 2 * 3 / 0.020)
    assert recs[1]["ref_is_none"]


def test_single_rank_defaults(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench
    r = bench.Ranks("gloo")
    assert (r.world, r.rank, r.local) == (1, 0, 0)
    assert r.max(3.5) == 3.5
    r.barrier()
    r.close()


def test_reference_arm_line(monkeypatch, capsys):
    """`bench.py --impl reference` (rank 0): the oracle timed on bounded
    windows of the bench workload, printed as one JSON line with the GPU
    arm's metric and unit and impl = reference."""
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    import bench

    class A:
        steps, warmup, gpus = 1, 3, 1
    out = bench.reference_arm(A())
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line == json.loads(json.dumps(out))
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["cpu_baseline"]["kind"] == "oracle"
