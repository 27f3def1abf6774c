"""The one-launch chunkwise path (few heads, no rotation, no carried state:
every block of 128 rows of every head at once, each block's entering state
formed from the key-value sums its predecessors publish) against the fp64
oracle: a single block, ragged lengths, the largest block count, both d_k
and d_v sizes, O and Y in both output dtypes, gamma = 1 and the smallest
gamma the path takes.  The launch count shows which path ran."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from parity import rel_l2, TOL_BF16
from retentive_network_scale_b200 import retention as R
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


def _inputs(B, H, L, dk, dv, seed):
    Q = random_tensor((B, H, L, dk), seed, dk ** -0.5).bfloat16()
    K = random_tensor((B, H, L, dk), seed + 1, dk ** -0.5).bfloat16()
    V = random_tensor((B, H, L, dv), seed + 2).bfloat16()
    G = random_tensor((B, L, H * dv), seed + 3).bfloat16()
    return Q, K, V, G


@pytest.mark.parametrize("B,H,L,dk,dv,gam,out", [
    (1, 1, 100, 128, 64, [0.96875], torch.bfloat16),          # one short block
    (1, 3, 300, 128, 128, [0.96875, 0.999, 1.0], torch.bfloat16),  # ragged, gamma = 1
    (2, 2, 4096, 64, 128, [0.75, 0.9921875], torch.float32),   # 32 blocks, small gamma
    (2, 3, 1000, 64, 64, [0.9, 0.99, 0.999], torch.bfloat16),
])
def test_onepass_matches_oracle(B, H, L, dk, dv, gam, out):
    Q, K, V, G = _inputs(B, H, L, dk, dv, 1200 + L)
    O_ref, _ = orc.recurrent(Q, K, V, gam, rotate=False)
    Y_ref = orc.gate_groupnorm(O_ref, G)
    Qd, Kd, Vd, Gd = Q.cuda(), K.cuda(), V.cuda(), G.cuda()
    O = torch.empty(B, H, L, dv, device="cuda", dtype=out)
    Y = torch.empty(B, L, H * dv, device="cuda", dtype=out)
    n0 = R.ret_kernel_launches()
    R.ret_chunkwise(Qd, Kd, Vd, gam, 64, O=O, G=Gd, Y=Y)
    assert R.ret_kernel_launches() - n0 == 1
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    for b in range(B):
        for h in range(H):
            assert rel_l2(O[b, h], O_ref[b, h]) <= TOL_BF16, (b, h)
            assert rel_l2(Y[b, :, h * dv:(h + 1) * dv], Y_ref[b, :, h * dv:(h + 1) * dv]) <= TOL_BF16, (b, h)
    # Y alone, and O alone, through the same launch
    Y2 = torch.empty_like(Y)
    R.ret_chunkwise(Qd, Kd, Vd, gam, 64, G=Gd, Y=Y2)
    O2 = torch.empty_like(O)
    R.ret_chunkwise(Qd, Kd, Vd, gam, 64, O=O2)
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    assert torch.equal(Y2, Y) and torch.equal(O2, O)


def test_onepass_leaves_states_and_rotation_to_the_other_paths():
    B, H, L, dk, dv = 1, 2, 600, 64, 64
    gam = [0.9, 0.99]
    Q, K, V, G = _inputs(B, H, L, dk, dv, 1300)
    S0 = random_tensor((B, H, dk, dv), 1304, 0.1)
    Qd, Kd, Vd, Gd = Q.cuda(), K.cuda(), V.cuda(), G.cuda()
    Y = torch.empty(B, L, H * dv, device="cuda", dtype=torch.bfloat16)
    St = torch.empty(B, H, dk, dv, device="cuda")
    R.ret_chunkwise(Qd, Kd, Vd, gam, 64, G=Gd, Y=Y, state_in=S0.cuda(), state_out=St)
    O_ref, S_ref = orc.recurrent(Q, K, V, gam, rotate=False, state_in=S0)
    Y_ref = orc.gate_groupnorm(O_ref, G)
    torch.cuda.synchronize()
    for h in range(H):
        assert rel_l2(Y[0, :, h * dv:(h + 1) * dv], Y_ref[0, :, h * dv:(h + 1) * dv]) <= TOL_BF16
        assert rel_l2(St[0, h], S_ref[0, h]) <= TOL_BF16
    # with rotation
    Yr = torch.empty_like(Y)
    R.ret_chunkwise(Qd, Kd, Vd, gam, 64, G=Gd, Y=Yr, rotate=True, pos_offset=3)
    Or_ref, _ = orc.recurrent(Q, K, V, gam, rotate=True, pos_offset=3)
    Yr_ref = orc.gate_groupnorm(Or_ref, G)
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    for h in range(H):
        assert rel_l2(Yr[0, :, h * dv:(h + 1) * dv], Yr_ref[0, :, h * dv:(h + 1) * dv]) <= TOL_BF16
