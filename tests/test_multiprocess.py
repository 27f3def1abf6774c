"""The data-parallel host logic of bench.py with two ranks on the CPU (gloo
backend, no GPU): process-group set-up from the torchrun environment, the
barrier, the max over ranks of the timed step, the whole-job weak-scaling
value, the per-rank input shards, and the reference arm running on rank 0
only.  The GPU path shards the same way (replicas, no data-path
collective), so these are the pieces that differ between N = 1 and N > 1."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    from retentive_network_scale_b200.synth import WORKLOADS, make_inputs
    try:
        w, r, local = bench.dist_setup(None)
        assert (w, r, local) == (world, rank, rank)
        assert dist.get_backend() == "gloo"
        bench.barrier(w)
        # each rank's own step time; everybody gets the slowest
        ms = bench.max_over_ranks(1.0 + 2.0 * r, w)
        tiny = WORKLOADS["tiny_fp32"]
        x = make_inputs(tiny, shard=r)
        digest = float(x["Q"].double().sum())
        q.put((r, ms, digest))
        bench.barrier(w)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_gloo():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get() for _ in range(world))
    assert [g[1] for g in got] == [3.0, 3.0]            # max over ranks, on every rank
    assert got[0][2] != got[1][2]                        # the replicas draw different shards


def test_whole_job_value_is_weak_scaling():
    sys.path.insert(0, ROOT)
    import bench
    # 4 ranks x 32768 tokens in the slowest rank's 0.5 ms
    assert bench.whole_job_value(4, 32768, 0.5) == pytest.approx(4 * 32768 / 0.5e-3)
    assert bench.whole_job_value(1, 32768, 0.5) * 4 == pytest.approx(bench.whole_job_value(4, 32768, 0.5))
    with pytest.raises(ValueError):
        bench.whole_job_value(0, 1, 1.0)
    with pytest.raises(ValueError):
        bench.whole_job_value(2, 1, 0.0)


def test_shards_are_independent_and_reproducible():
    sys.path.insert(0, ROOT)
    from retentive_network_scale_b200.synth import WORKLOADS, make_inputs, shard_seed
    w = WORKLOADS["tiny_fp32"]
    a0, a0b, a1 = make_inputs(w, shard=0), make_inputs(w, shard=0), make_inputs(w, shard=1)
    assert torch.equal(a0["Q"], a0b["Q"])                     # reproducible
    assert torch.equal(a0["Q"], make_inputs(w)["Q"])         # shard 0 = the workload's own draw
    assert not torch.equal(a0["Q"], a1["Q"])                 # shards differ
    assert len({shard_seed(w.seed, s) for s in range(64)}) == 64
    with pytest.raises(ValueError):
        shard_seed(w.seed, -1)


def test_reference_arm_only_on_rank_zero():
    sys.path.insert(0, ROOT)
    import bench
    args = type("A", (), {"steps": 1, "warmup": 0, "gpus": 2})()
    out = io.StringIO()
    with redirect_stdout(out):
        bench.run_reference(args, 2, 1)   # rank 1 of 2: no work, no line
    assert out.getvalue() == ""
