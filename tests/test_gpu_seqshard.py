"""The sequence-sharded chunkwise path on the GPU: ret_segment_state and
ret_state_scan against the fp64 oracle (itself pinned to one uncut
recurrent run), and whole sequences cut into segments that run one after
another on this GPU -- each through the same function a rank runs, with the
all-gather replaced by the stacked segment states -- against the oracle's
uncut run: outputs, the fused GroupNorm + gate, and the final state; and
ret_chunkwise_segmented, which runs all segments of a sequence at once.

"Retentive Network" paper summary, section 2.1, chunkwise form (3)."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from parity import normwise, rel_l2, TOL_BF16, TOL_F32
from retentive_network_scale_b200 import retention as R
from retentive_network_scale_b200.seqshard import chunkwise_sequence_sharded, segment_lengths
from retentive_network_scale_b200.synth import random_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from retentive_network_scale_b200 import build
    build.build()
    R.load_library()
    yield
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0


def _qkv(B, H, L, dk, dv, seed):
    Q = random_tensor((B, H, L, dk), seed, dk ** -0.5).bfloat16()
    K = random_tensor((B, H, L, dk), seed + 1, dk ** -0.5).bfloat16()
    V = random_tensor((B, H, L, dv), seed + 2).bfloat16()
    return Q, K, V


@pytest.mark.parametrize("L,dk,dv,rotate", [(300, 128, 128, True), (1, 256, 256, False),
                                            (700, 64, 40, True)])
def test_segment_state_matches_oracle(L, dk, dv, rotate):
    B, H = 2, 3
    g = [0.9, 0.99, 1.0]
    Q, K, V = _qkv(B, H, L, dk, dv, 40)
    U = R.ret_segment_state(K.cuda(), V.cuda(), g, rotate=rotate, pos_offset=1000)
    ref = orc.segment_state(K, V, g, rotate=rotate, pos_offset=1000)
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(H):
            assert rel_l2(U[b, h], ref[b, h]) <= TOL_BF16, (b, h)


def test_empty_segment_is_the_zero_state():
    U = R.ret_segment_state(torch.zeros(1, 2, 0, 16, device="cuda", dtype=torch.bfloat16),
                            torch.zeros(1, 2, 0, 8, device="cuda", dtype=torch.bfloat16), [0.5, 0.9],
                            U=torch.full((1, 2, 16, 8), 7.0, device="cuda"))
    assert float(U.abs().max()) == 0.0


@pytest.mark.parametrize("rank", [0, 1, 3, 4])
@pytest.mark.parametrize("with_in", [False, True])
def test_state_scan_matches_oracle(rank, with_in):
    B, H, dk, dv = 2, 2, 16, 12
    lens = [128, 7, 300, 1]
    g = [0.97, 0.999]
    U = torch.stack([random_tensor((B, H, dk, dv), 60 + s) for s in range(4)])
    S0 = random_tensor((B, H, dk, dv), 70) if with_in else None
    Rg = R.ret_state_scan(U.cuda(), lens, rank, g, state_in=None if S0 is None else S0.cuda())
    ref = orc.state_scan(U, lens, g, state_in=S0)[rank]
    torch.cuda.synchronize()
    if rank == 0 and not with_in:
        assert float(Rg.abs().max()) == 0.0
    else:
        assert normwise(Rg, ref) <= TOL_F32


@pytest.mark.parametrize("L,parts,dk,dv,gate", [
    (1100, 3, 256, 512, True),     # RetNet-1.3B head shape, tensor-core path, fused gate
    (640, 2, 128, 256, False),     # O and the final state
    (257, 4, 64, 32, False),       # CUDA-core path, ragged segments
])
def test_segments_reproduce_the_uncut_sequence(L, parts, dk, dv, gate):
    B, H = 1, 2
    g = [0.96875, 0.999]
    Q, K, V = _qkv(B, H, L, dk, dv, 90)
    G = random_tensor((B, L, H * dv), 95).bfloat16()
    S0 = random_tensor((B, H, dk, dv), 96, 0.1)
    lens = segment_lengths(L, parts)
    starts = np.cumsum([0] + lens[:-1])
    Qd, Kd, Vd, Gd = Q.cuda(), K.cuda(), V.cuda(), G.cuda()
    sl = lambda t, a, n: t[:, :, a:a + n].contiguous()  # noqa: E731
    U_all = torch.stack([R.ret_segment_state(sl(Kd, a, n), sl(Vd, a, n), g, rotate=True,
                                             pos_offset=5 + a) for a, n in zip(starts, lens)])
    O_ref, S_ref = orc.recurrent(Q, K, V, g, rotate=True, pos_offset=5, state_in=S0)
    Y_ref = orc.gate_groupnorm(O_ref, G)
    for r, (a, n) in enumerate(zip(starts, lens)):
        O = torch.empty(B, H, n, dv, device="cuda", dtype=torch.bfloat16)
        Y = torch.empty(B, n, H * dv, device="cuda", dtype=torch.bfloat16) if gate else None
        S = torch.empty(B, H, dk, dv, device="cuda")
        chunkwise_sequence_sharded(sl(Qd, a, n), sl(Kd, a, n), sl(Vd, a, n), g, 128, lens, r,
                                   O=O, G=Gd[:, a:a + n].contiguous() if gate else None, Y=Y,
                                   state_in=S0.cuda(), state_out=S, rotate=True, pos_offset=5,
                                   gather=lambda U: U_all)
        torch.cuda.synchronize()
        for h in range(H):
            assert rel_l2(O[0, h], O_ref[0, h, a:a + n]) <= TOL_BF16, (r, h)
            if gate:
                assert rel_l2(Y[0, :, h * dv:(h + 1) * dv],
                              Y_ref[0, a:a + n, h * dv:(h + 1) * dv]) <= TOL_BF16, (r, h)
    for h in range(H):
        assert rel_l2(S[0, h], S_ref[0, h]) <= TOL_BF16, h


@pytest.mark.parametrize("L,S,dk,dv,with_in,rotate", [
    (2048, 4, 128, 256, True, True),     # segments of 512 rows
    (1200, 3, 256, 128, False, True),    # segments of 400 rows: ragged last block in each
    (384, 1, 128, 128, True, True),      # one segment: the plain loop
    (1200, 3, 128, 256, True, False),    # without rotation: no streaming pass
])
def test_segmented_matches_oracle(L, S, dk, dv, with_in, rotate):
    """ret_chunkwise_segmented: all segments of every sequence at once, each
    from the state the scan gives it, against the oracle's uncut run
    (outputs of every head and the final state)."""
    B, H = 1, 3
    g = [0.96875, 0.99, 0.999]
    Q, K, V = _qkv(B, H, L, dk, dv, 130)
    S0 = random_tensor((B, H, dk, dv), 135, 0.1) if with_in else None
    O_ref, S_ref = orc.recurrent(Q, K, V, g, rotate=rotate, pos_offset=77, state_in=S0)
    O = torch.empty(B, H, L, dv, device="cuda", dtype=torch.bfloat16)
    St = torch.empty(B, H, dk, dv, device="cuda")
    n0 = R.ret_kernel_launches()
    R.ret_chunkwise_segmented(Q.cuda(), K.cuda(), V.cuda(), g, 128, S, O=O,
                              state_in=None if S0 is None else S0.cuda(), state_out=St,
                              rotate=rotate, pos_offset=77)
    # the streaming pass, the segment states, the scan, the chunk loop
    assert R.ret_kernel_launches() - n0 == 4
    torch.cuda.synchronize()
    for h in range(H):
        assert rel_l2(O[0, h], O_ref[0, h]) <= TOL_BF16, h
        assert rel_l2(St[0, h], S_ref[0, h]) <= TOL_BF16, h


@pytest.mark.parametrize("L,dk,dv,rotate,segs", [
    (2048, 128, 128, True, 4),     # 2 heads x 1 value tile: 4 segments of 512 rows
    (2048, 64, 64, False, 4),      # msr_small's head shape, without rotation
    (1536, 256, 256, True, 2),     # 1536 = 3 x 512: two segments of 768 rows
])
def test_chunkwise_takes_segments_for_few_heads(L, dk, dv, rotate, segs):
    """ret_chunkwise with ret_chunkwise_fast_size bytes of workspace on few
    heads: every sequence cut into segments that run at once, the fused
    GroupNorm + gate on each segment's own rows, O and the final state from
    a carried state; against the oracle's uncut run, and against the plain
    loop (no workspace) up to rounding."""
    B, H = 1, 2
    g = [0.96875, 0.999]
    Q, K, V = _qkv(B, H, L, dk, dv, 150)
    G = random_tensor((B, L, H * dv), 155).bfloat16()
    S0 = random_tensor((B, H, dk, dv), 156, 0.1)
    O_ref, S_ref = orc.recurrent(Q, K, V, g, rotate=rotate, pos_offset=9, state_in=S0)
    Y_ref = orc.gate_groupnorm(O_ref, G)
    desc = R.make_desc(B, H, L, dk, dv, R.RET_BF16, R.RET_BF16, g, rotate, 10000.0, 9)
    lib = R.load_library()
    # (at least the segments' bytes: the one-launch path's block sums may
    # need more, but a call with a carried state takes the segments)
    assert lib.ret_chunkwise_fast_size(ctypes.byref(desc), 128) >= \
        lib.ret_chunkwise_segmented_workspace_size(ctypes.byref(desc), 128, segs)
    Qd, Kd, Vd, Gd, S0d = Q.cuda(), K.cuda(), V.cuda(), G.cuda(), S0.cuda()
    O = torch.empty(B, H, L, dv, device="cuda", dtype=torch.bfloat16)
    Y = torch.empty(B, L, H * dv, device="cuda", dtype=torch.bfloat16)
    St = torch.empty(B, H, dk, dv, device="cuda")
    n0 = R.ret_kernel_launches()
    R.ret_chunkwise(Qd, Kd, Vd, g, 128, O=O, state_in=S0d, state_out=St, G=Gd, Y=Y,
                    rotate=rotate, pos_offset=9)
    # the streaming pass, the segment states, the scan, the chunk loop
    assert R.ret_kernel_launches() - n0 == 4
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    for h in range(H):
        assert rel_l2(O[0, h], O_ref[0, h]) <= TOL_BF16, h
        assert rel_l2(Y[0, :, h * dv:(h + 1) * dv], Y_ref[0, :, h * dv:(h + 1) * dv]) <= TOL_BF16, h
        assert rel_l2(St[0, h], S_ref[0, h]) <= TOL_BF16, h
    # the plain loop on the same call, without the workspace
    O2, Y2, S2 = torch.empty_like(O), torch.empty_like(Y), torch.empty_like(St)
    R.ret_chunkwise(Qd, Kd, Vd, g, 128, O=O2, state_in=S0d, state_out=S2, G=Gd, Y=Y2,
                    rotate=rotate, pos_offset=9, prep=False)
    torch.cuda.synchronize()
    assert rel_l2(O2, O) <= TOL_BF16 and rel_l2(Y2, Y) <= TOL_BF16 and rel_l2(S2, St) <= TOL_BF16
