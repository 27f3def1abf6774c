"""Several tokens per ret_recurrent_step call (1 < T <= RET_MAX_DECODE_STEPS):
outputs and the in-place state against the oracle's recurrent form run on
from the same state, for the three column layouts of the kernels (d_v a
multiple of 128, of 32, neither), fp32 and bf16, with rotation at a large
offset;
T-token calls chained, and agreement with T single-token calls."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from parity import normwise, rel_l2, TOL_BF16, TOL_F32
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


def _case(B, H, T, dk, dv, dtype, seed):
    q = random_tensor((B, H, T, dk), seed, dk ** -0.5).to(dtype)
    k = random_tensor((B, H, T, dk), seed + 1, dk ** -0.5).to(dtype)
    v = random_tensor((B, H, T, dv), seed + 2).to(dtype)
    s0 = random_tensor((B, H, dk, dv), seed + 3, 0.2)
    return q, k, v, s0


@pytest.mark.parametrize("T", [2, 5, 8, 16])
@pytest.mark.parametrize("dtype,dv", [(torch.float32, 96), (torch.bfloat16, 36),
                                      (torch.float32, 256), (torch.bfloat16, 128)])
def test_multi_token_step_matches_oracle(T, dtype, dv):
    B, H, dk, p0 = 2, 3, 64, 1000
    q, k, v, s0 = _case(B, H, T, dk, dv, dtype, 40 + T)
    g = [0.9, 0.99, 1.0]
    O_ref, S_ref = orc.recurrent(q, k, v, g, rotate=True, pos_offset=p0, state_in=s0)
    state = s0.cuda()
    o = torch.empty(B, H, T, dv, device="cuda", dtype=dtype)
    n0 = R.ret_kernel_launches()
    R.ret_recurrent_step(q.cuda(), k.cuda(), v.cuda(), state, o, g, pos=p0, rotate=True)
    assert R.ret_kernel_launches() - n0 == 1            # one pass over the state
    torch.cuda.synchronize()
    if dtype == torch.float32:
        assert normwise(o, O_ref) <= TOL_F32
        assert normwise(state, S_ref) <= TOL_F32
    else:
        assert rel_l2(o, O_ref) <= TOL_BF16
        assert rel_l2(state, S_ref) <= TOL_BF16


def test_multi_token_chained_and_single_steps():
    """T=3 then T=5 from a state equals 8 single-token steps and the oracle."""
    B, H, dk, dv, p0 = 1, 2, 128, 256, 77
    q, k, v, s0 = _case(B, H, 8, dk, dv, torch.float32, 90)
    g = [0.96875, 0.999]
    O_ref, S_ref = orc.recurrent(q, k, v, g, rotate=True, pos_offset=p0, state_in=s0)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    st = s0.cuda()
    o = torch.empty(B, H, 8, dv, device="cuda")
    o1 = torch.empty(B, H, 3, dv, device="cuda")
    o2 = torch.empty(B, H, 5, dv, device="cuda")
    R.ret_recurrent_step(qd[:, :, :3].contiguous(), kd[:, :, :3].contiguous(), vd[:, :, :3].contiguous(),
                         st, o1, g, pos=p0, rotate=True)
    R.ret_recurrent_step(qd[:, :, 3:].contiguous(), kd[:, :, 3:].contiguous(), vd[:, :, 3:].contiguous(),
                         st, o2, g, pos=p0 + 3, rotate=True)
    st1 = s0.cuda()
    o_single = torch.empty(B, H, 8, dv, device="cuda")
    for t in range(8):
        ot = torch.empty(B, H, dv, device="cuda")
        R.ret_recurrent_step(qd[:, :, t].contiguous(), kd[:, :, t].contiguous(), vd[:, :, t].contiguous(),
                             st1, ot, g, pos=p0 + t, rotate=True)
        o_single[:, :, t] = ot
    torch.cuda.synchronize()
    got = torch.cat([o1, o2], 2)
    assert normwise(got, O_ref) <= TOL_F32
    assert normwise(st, S_ref) <= TOL_F32
    assert normwise(got, o_single.cpu().double().numpy()) <= TOL_F32
    assert normwise(st, st1.cpu().double().numpy()) <= TOL_F32


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_multi_token_fast_decays_take_the_direct_form(dtype):
    """Heads with gamma^T below 2^-60 (gamma 0 and 0.01 at T = 16) run the
    direct update in the same call as a slow head on the rescaled one; all
    three match the oracle."""
    B, H, T, dk, dv, p0 = 2, 3, 16, 64, 128, 500
    q, k, v, s0 = _case(B, H, T, dk, dv, dtype, 77)
    g = [0.0, 0.01, 0.9]
    O_ref, S_ref = orc.recurrent(q, k, v, g, rotate=True, pos_offset=p0, state_in=s0)
    state = s0.cuda()
    o = torch.empty(B, H, T, dv, device="cuda", dtype=dtype)
    R.ret_recurrent_step(q.cuda(), k.cuda(), v.cuda(), state, o, g, pos=p0, rotate=True)
    torch.cuda.synchronize()
    if dtype == torch.float32:
        assert normwise(o, O_ref) <= TOL_F32
        assert normwise(state, S_ref) <= TOL_F32
    else:
        assert rel_l2(o, O_ref) <= TOL_BF16
        assert rel_l2(state, S_ref) <= TOL_BF16
