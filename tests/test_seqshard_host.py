"""The host logic of the sequence-sharded chunkwise path
(``retentive_network_scale_b200.seqshard``) with two ranks on the CPU over
gloo: segment starts and absolute positions, the rank order of the
all-gather, and the scan of the gathered states.  The three per-rank
computations are the oracle's, passed in through ``SegmentOps``, so no GPU
is needed; the GPU tests run the same function on the library's kernels.

"Retentive Network" paper summary, section 2.1, chunkwise form (3): the
state recurrence between blocks of rows, here between segments."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def oracle_ops():
    """SegmentOps whose computations are the fp64 oracle's (test only)."""
    from oracle import oracle as orc
    from retentive_network_scale_b200.seqshard import SegmentOps

    def segment_state(K, V, gamma, pos_offset=0, stream=None, rotate=False, theta_base=10000.0):
        return torch.from_numpy(orc.segment_state(K.numpy(), V.numpy(), gamma, rotate=rotate,
                                                  theta_base=theta_base, pos_offset=pos_offset))

    def state_scan(U_all, seg_lens, rank, gamma, state_in=None, stream=None):
        s0 = None if state_in is None else state_in.numpy()
        return torch.from_numpy(orc.state_scan(U_all.numpy(), seg_lens, gamma, state_in=s0)[rank])

    def chunkwise(Q, K, V, gamma, chunk, O=None, G=None, Y=None, state_in=None, state_out=None,
                  gn_eps=1e-5, pos_offset=0, stream=None, rotate=False, theta_base=10000.0):
        o, s = orc.recurrent(Q.numpy(), K.numpy(), V.numpy(), gamma, rotate=rotate,
                             theta_base=theta_base, pos_offset=pos_offset,
                             state_in=None if state_in is None else state_in.numpy())
        y = None if G is None else torch.from_numpy(orc.gate_groupnorm(o, G.numpy(), gn_eps))
        return torch.from_numpy(o), y, torch.from_numpy(s)

    return SegmentOps(segment_state, state_scan, chunkwise)


def _problem():
    rng = np.random.default_rng(5)
    B, H, L, dk, dv = 1, 2, 23, 4, 6
    t = lambda *s: torch.from_numpy(rng.standard_normal(s))  # noqa: E731
    return dict(Q=t(B, H, L, dk) * 0.5, K=t(B, H, L, dk) * 0.5, V=t(B, H, L, dv),
                G=t(B, L, H * dv), S0=t(B, H, dk, dv), gamma=[0.7, 0.95], lens=[9, 14])


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from oracle import oracle as orc
    from retentive_network_scale_b200.seqshard import chunkwise_sequence_sharded
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = _problem()
        lens = x["lens"]
        a = sum(lens[:rank])
        n = lens[rank]
        own = lambda t: t[:, :, a:a + n].contiguous()  # noqa: E731
        O, Y, S = chunkwise_sequence_sharded(
            own(x["Q"]), own(x["K"]), own(x["V"]), x["gamma"], 128, lens, rank,
            G=x["G"][:, a:a + n].contiguous(), state_in=x["S0"], rotate=True, pos_offset=3,
            ops=oracle_ops())
        O_ref, S_ref = orc.recurrent(x["Q"].numpy(), x["K"].numpy(), x["V"].numpy(), x["gamma"],
                                     rotate=True, pos_offset=3, state_in=x["S0"].numpy())
        Y_ref = orc.gate_groupnorm(O_ref, x["G"].numpy())
        errs = (float(np.abs(O.numpy() - O_ref[:, :, a:a + n]).max()),
                float(np.abs(Y.numpy() - Y_ref[:, a:a + n]).max()),
                float(np.abs(S.numpy() - S_ref).max()) if rank == world - 1 else 0.0)
        q.put((rank, errs))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_ranks_join_through_their_states():
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
    for rank, errs in got:
        assert max(errs) <= 1e-10, (rank, errs)


def test_gather_stand_in_and_checks():
    """One process, the all-gather replaced by a function: three segments
    in sequence reproduce one uncut run; bad ranks and row counts raise."""
    sys.path.insert(0, ROOT)
    from oracle import oracle as orc
    from retentive_network_scale_b200.seqshard import chunkwise_sequence_sharded
    x = _problem()
    lens = [7, 10, 6]
    starts = np.cumsum([0] + lens[:-1])
    ops = oracle_ops()
    U_all = torch.stack([ops.segment_state(x["K"][:, :, a:a + n], x["V"][:, :, a:a + n], x["gamma"],
                                           pos_offset=a, rotate=False)
                         for a, n in zip(starts, lens)])
    O_ref, S_ref = orc.recurrent(x["Q"].numpy(), x["K"].numpy(), x["V"].numpy(), x["gamma"])
    for r, (a, n) in enumerate(zip(starts, lens)):
        sl = lambda t: t[:, :, a:a + n].contiguous()  # noqa: E731
        O, _, S = chunkwise_sequence_sharded(sl(x["Q"]), sl(x["K"]), sl(x["V"]), x["gamma"], 128,
                                             lens, r, gather=lambda U: U_all, ops=ops)
        assert np.abs(O.numpy() - O_ref[:, :, a:a + n]).max() <= 1e-10
    assert np.abs(S.numpy() - S_ref).max() <= 1e-10
    with pytest.raises(ValueError):
        chunkwise_sequence_sharded(x["Q"], x["K"], x["V"], x["gamma"], 128, lens, 3,
                                   gather=lambda U: U_all, ops=ops)
    with pytest.raises(ValueError):   # Q does not hold segment 0's rows
        chunkwise_sequence_sharded(x["Q"], x["K"], x["V"], x["gamma"], 128, lens, 0,
                                   gather=lambda U: U_all, ops=ops)


def test_segment_lengths():
    sys.path.insert(0, ROOT)
    from retentive_network_scale_b200.seqshard import segment_lengths
    assert segment_lengths(4096, 4) == [1024] * 4
    assert segment_lengths(1000, 3) == [256, 256, 488]
    assert segment_lengths(10, 3) == [3, 3, 4]
    assert sum(segment_lengths(65537, 8)) == 65537
    with pytest.raises(ValueError):
        segment_lengths(2, 3)
