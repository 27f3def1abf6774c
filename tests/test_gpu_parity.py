"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle on
the same seeded inputs, element by element at small sizes and on sampled
(b, h) slices at the full workload sizes."""
import numpy as np
import pytest
import torch

from oracle import oracle as orc
from parity import (oracle_gate_slices, oracle_slices, rel_l2, normwise, to64, within,
                    y_slices, TOL_BF16, TOL_F32)
from retentive_network_scale_b200 import retention as R
from retentive_network_scale_b200.synth import WORKLOADS, make_inputs, make_decode_inputs, random_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from retentive_network_scale_b200 import build
    build.build()
    R.load_library()
    torch.cuda.init()
    yield
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0


def dev(d):
    return {k: v.cuda() for k, v in d.items()}


# ------------------------------------------------------------------ tiny fp32
def test_tiny_fp32_all_forms():
    w = WORKLOADS["tiny_fp32"]
    x = make_inputs(w)
    g = R.msr_gammas(w.H)
    ref = orc.parallel(x["Q"], x["K"], x["V"], orc.gammas(w.H), rotate=True)
    _, S_ref = orc.recurrent(x["Q"], x["K"], x["V"], orc.gammas(w.H), rotate=True)
    d = dev(x)
    O = torch.empty(w.B, w.H, w.L, w.d_v, device="cuda")
    R.ret_parallel(d["Q"], d["K"], d["V"], O, g, rotate=True)
    assert normwise(O, ref) <= TOL_F32
    O2 = torch.empty_like(O)
    S = torch.empty(w.B, w.H, w.d_k, w.d_v, device="cuda")
    R.ret_chunkwise(d["Q"], d["K"], d["V"], g, w.chunk, O=O2, state_out=S, rotate=True)
    assert normwise(O2, ref) <= TOL_F32
    assert normwise(S, S_ref) <= TOL_F32
    # recurrent: L steps of the decode entry point from a zero state
    st = torch.zeros(w.B, w.H, w.d_k, w.d_v, device="cuda")
    o = torch.empty(w.B, w.H, w.d_v, device="cuda")
    outs = []
    for t in range(w.L):
        R.ret_recurrent_step(d["Q"][:, :, t].contiguous(), d["K"][:, :, t].contiguous(),
                             d["V"][:, :, t].contiguous(), st, o, g, pos=t, rotate=True)
        outs.append(o.clone())
    assert normwise(torch.stack(outs, 2), ref) <= TOL_F32
    assert normwise(st, S_ref) <= TOL_F32


# ------------------------------------------------------------------ edge cases
@pytest.mark.parametrize("L,C", [(37, 16), (100, 1), (100, 5), (100, 32), (100, 1000), (1, 7)])
def test_chunk_sizes_and_ragged_tails(L, C):
    B, H, dk, dv = 2, 3, 8, 12
    Q = random_tensor((B, H, L, dk), 11, 0.5)
    K = random_tensor((B, H, L, dk), 12, 0.5)
    V = random_tensor((B, H, L, dv), 13)
    g = [0.0, 0.9, 1.0]
    ref = orc.parallel(Q, K, V, g, rotate=True, pos_offset=3)
    _, S_ref = orc.recurrent(Q, K, V, g, rotate=True, pos_offset=3)
    O = torch.empty(B, H, L, dv, device="cuda")
    S = torch.empty(B, H, dk, dv, device="cuda")
    R.ret_chunkwise(Q.cuda(), K.cuda(), V.cuda(), g, C, O=O, state_out=S, rotate=True, pos_offset=3)
    assert normwise(O, ref) <= TOL_F32
    assert normwise(S, S_ref) <= TOL_F32
    O2 = torch.empty_like(O)
    R.ret_parallel(Q.cuda(), K.cuda(), V.cuda(), O2, g, rotate=True, pos_offset=3)
    assert normwise(O2, ref) <= TOL_F32


def test_empty_and_passthrough():
    B, H, dk, dv = 2, 2, 8, 8
    Q = torch.zeros(B, H, 0, dk, device="cuda")
    V = torch.zeros(B, H, 0, dv, device="cuda")
    S_in = random_tensor((B, H, dk, dv), 3).cuda()
    S_out = torch.full_like(S_in, 7.0)
    R.ret_chunkwise(Q, Q, V, [0.5, 0.6], 4, O=torch.zeros(B, H, 0, dv, device="cuda"),
                    state_in=S_in, state_out=S_out)
    torch.cuda.synchronize()
    assert torch.equal(S_in, S_out)
    R.ret_chunkwise(Q, Q, V, [0.5, 0.6], 4, O=torch.zeros(B, H, 0, dv, device="cuda"),
                    state_out=S_out)
    torch.cuda.synchronize()
    assert S_out.abs().max().item() == 0.0
    O = torch.zeros(B, H, 0, dv, device="cuda")
    R.ret_parallel(Q, Q, V, O, [0.5, 0.6])


def test_state_handoff_and_alias():
    """chunkwise(L1) -> state -> chunkwise(L2) in place -> recurrent steps
    equals one oracle run over the whole sequence."""
    B, H, dk, dv, L1, L2, T = 1, 2, 16, 8, 45, 30, 5
    L = L1 + L2 + T
    Q = random_tensor((B, H, L, dk), 21, 0.25)
    K = random_tensor((B, H, L, dk), 22, 0.25)
    V = random_tensor((B, H, L, dv), 23)
    g = [0.95, 0.999]
    ref, S_ref = orc.recurrent(Q, K, V, g, rotate=True, pos_offset=1000)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    S = torch.empty(B, H, dk, dv, device="cuda")
    O1 = torch.empty(B, H, L1, dv, device="cuda")
    R.ret_chunkwise(Qd[:, :, :L1].contiguous(), Kd[:, :, :L1].contiguous(), Vd[:, :, :L1].contiguous(),
                    g, 16, O=O1, state_out=S, rotate=True, pos_offset=1000)
    O2 = torch.empty(B, H, L2, dv, device="cuda")
    sl = slice(L1, L1 + L2)
    R.ret_chunkwise(Qd[:, :, sl].contiguous(), Kd[:, :, sl].contiguous(), Vd[:, :, sl].contiguous(),
                    g, 16, O=O2, state_in=S, state_out=S, rotate=True, pos_offset=1000 + L1)
    outs = []
    o = torch.empty(B, H, dv, device="cuda")
    for t in range(L1 + L2, L):
        R.ret_recurrent_step(Qd[:, :, t].contiguous(), Kd[:, :, t].contiguous(), Vd[:, :, t].contiguous(),
                             S, o, g, pos=1000 + t, rotate=True)
        outs.append(o.clone())
    got = torch.cat([O1, O2, torch.stack(outs, 2)], 2)
    assert normwise(got, ref) <= TOL_F32
    assert normwise(S, S_ref) <= TOL_F32


def test_large_positions():
    """Rotation angles near 10^5 rad keep fp32 accuracy."""
    B, H, L, dk, dv = 1, 2, 50, 32, 8
    Q = random_tensor((B, H, L, dk), 31, 0.2)
    K = random_tensor((B, H, L, dk), 32, 0.2)
    V = random_tensor((B, H, L, dv), 33)
    g = [0.9, 0.99]
    ref = orc.parallel(Q, K, V, g, rotate=True, pos_offset=100000)
    O = torch.empty(B, H, L, dv, device="cuda")
    R.ret_chunkwise(Q.cuda(), K.cuda(), V.cuda(), g, 16, O=O, rotate=True, pos_offset=100000)
    assert normwise(O, ref) <= TOL_F32


def test_limits_max_dims_and_heads():
    B, H, L, dk, dv = 1, 2, 40, 256, 512
    Q = random_tensor((B, H, L, dk), 41, 1 / 16)
    K = random_tensor((B, H, L, dk), 42, 1 / 16)
    V = random_tensor((B, H, L, dv), 43)
    g = [0.96875, 0.999]
    ref, S_ref = orc.recurrent(Q, K, V, g, rotate=True)
    O = torch.empty(B, H, L, dv, device="cuda")
    S = torch.empty(B, H, dk, dv, device="cuda")
    R.ret_chunkwise(Q.cuda(), K.cuda(), V.cuda(), g, 16, O=O, state_out=S, rotate=True)
    assert normwise(O, ref) <= TOL_F32 and normwise(S, S_ref) <= TOL_F32
    # many heads, small dims
    H = R.RET_MAX_HEADS
    Q = random_tensor((1, H, 9, 4), 44)
    V = random_tensor((1, H, 9, 4), 45)
    g = R.msr_gammas(H)
    g = [min(x, 1.0) for x in g]
    ref = orc.parallel(Q, Q, V, g)
    O = torch.empty(1, H, 9, 4, device="cuda")
    R.ret_parallel(Q.cuda(), Q.cuda(), V.cuda(), O, g)
    assert normwise(O, ref) <= TOL_F32


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dv", [64, 20, 512])
def test_gate_norm_standalone(dtype, dv):
    B, H, L = 2, 3, 33
    O = (random_tensor((B, H, L, dv), 51) * 2 + 0.5).to(dtype)
    G = random_tensor((B, L, H * dv), 52).to(dtype)
    ref = orc.gate_groupnorm(O, G, 1e-5)
    Y = torch.empty(B, L, H * dv, device="cuda", dtype=dtype)
    R.ret_gate_norm(O.cuda(), G.cuda(), Y, 1e-5)
    ok, err = within(Y, ref, dtype)
    assert ok, err


def test_gate_norm_large_mean():
    """Rows far from zero mean (around 300, spread 0.5): the shifted sums
    keep the variance."""
    B, H, L, dv = 1, 2, 9, 128
    O = random_tensor((B, H, L, dv), 53) * 0.5 + 300.0
    G = random_tensor((B, L, H * dv), 54)
    Y = torch.empty(B, L, H * dv, device="cuda")
    R.ret_gate_norm(O.cuda(), G.cuda(), Y, 1e-5)
    assert normwise(Y, orc.gate_groupnorm(O, G, 1e-5)) <= TOL_F32


@pytest.mark.parametrize("o_dtype,g_dtype", [(torch.float32, torch.float32),
                                             (torch.bfloat16, torch.bfloat16),
                                             (torch.float32, torch.bfloat16)])
@pytest.mark.parametrize("dv", [64, 20, 512])
def test_gate_norm_backward(o_dtype, g_dtype, dv):
    """dO and dG of the GroupNorm + swish gate against the fp64 oracle's
    chain rule, with a ragged row count, d_v below, across and at the
    kernel's 512-channel limit."""
    B, H, L = 2, 3, 37
    O = (random_tensor((B, H, L, dv), 71) * 2 + 0.5).to(o_dtype)
    G = (random_tensor((B, L, H * dv), 72) * 1.5).to(g_dtype)
    dY = random_tensor((B, L, H * dv), 73).to(g_dtype)
    dO_ref, dG_ref = orc.gate_groupnorm_backward(O, G, dY, 1e-5)
    dO = torch.full((B, H, L, dv), float("nan"), device="cuda", dtype=o_dtype)
    dG = torch.full((B, L, H * dv), float("nan"), device="cuda", dtype=g_dtype)
    n0 = R.ret_kernel_launches()
    R.ret_gate_norm_backward(O.cuda(), G.cuda(), dY.cuda(), dO, dG, 1e-5)
    assert R.ret_kernel_launches() - n0 == 1
    ok, err = within(dO, dO_ref, o_dtype)
    assert ok, ("dO", err)
    ok, err = within(dG, dG_ref, g_dtype)
    assert ok, ("dG", err)


def test_gate_norm_backward_large_mean():
    """Rows whose mean is far above their spread (O around 300 with a
    spread of 0.5): the statistics must not lose the variance to the mean."""
    B, H, L, dv = 1, 2, 9, 128
    O = random_tensor((B, H, L, dv), 74) * 0.5 + 300.0
    G = random_tensor((B, L, H * dv), 75)
    dY = random_tensor((B, L, H * dv), 76)
    dO_ref, dG_ref = orc.gate_groupnorm_backward(O, G, dY, 1e-5)
    dO = torch.empty(B, H, L, dv, device="cuda")
    dG = torch.empty(B, L, H * dv, device="cuda")
    R.ret_gate_norm_backward(O.cuda(), G.cuda(), dY.cuda(), dO, dG, 1e-5)
    assert normwise(dO, dO_ref) <= TOL_F32
    assert normwise(dG, dG_ref) <= TOL_F32


def test_gate_norm_backward_full_size_sampled():
    """At the msr_1p3b size the bench times (B=8 H=8 L=4096 d_v=512, bf16
    O, G and dY): rows sampled across the batch, the sequence and the tail
    are checked against the oracle (rows are independent), and every row of
    dO sums to zero up to bf16 rounding."""
    w = WORKLOADS["msr_1p3b"]
    B, H, L, dv = w.B, w.H, w.L, w.d_v
    gen = torch.Generator(device="cuda")
    gen.manual_seed(77)
    O = torch.randn(B, H, L, dv, device="cuda", generator=gen).bfloat16()
    G = torch.randn(B, L, H * dv, device="cuda", generator=gen).bfloat16()
    dY = torch.randn(B, L, H * dv, device="cuda", generator=gen).bfloat16()
    dO = torch.empty_like(O)
    dG = torch.empty_like(G)
    R.ret_gate_norm_backward(O, G, dY, dO, dG, 1e-5)
    torch.cuda.synchronize()
    rows = [(0, 0), (0, 1), (3, 2047), (5, 100), (7, L - 2), (7, L - 1)]
    for b, t in rows:
        o = O[b, :, t:t + 1, :].unsqueeze(0).cpu()
        g = G[b, t:t + 1, :].unsqueeze(0).cpu()
        dy = dY[b, t:t + 1, :].unsqueeze(0).cpu()
        dO_ref, dG_ref = orc.gate_groupnorm_backward(o, g, dy, 1e-5)
        assert rel_l2(dO[b, :, t:t + 1, :].unsqueeze(0), dO_ref) <= TOL_BF16, (b, t)
        assert rel_l2(dG[b, t:t + 1, :].unsqueeze(0), dG_ref) <= TOL_BF16, (b, t)
    # bf16 rounding leaves each row sum about 2^-9/sqrt(3) of the row's norm
    f = dO.float()
    assert bool((f.sum(-1).abs() <= 0.02 * f.norm(dim=-1) + 1e-6).all())


# ------------------------------------------------------------------ workloads
def test_msr_small_bf16():
    """B=4 H=8 L=2048 d=64, chunk 64, GroupNorm + swish gate: every output."""
    w = WORKLOADS["msr_small"]
    x = make_inputs(w)
    d = dev(x)
    g = R.msr_gammas(w.H)
    pairs = [(b, h) for b in range(w.B) for h in range(w.H)]
    O_ref, S_ref = oracle_slices(x["Q"], x["K"], x["V"], pairs, orc.gammas(w.H), w.rotate)
    Y_ref = oracle_gate_slices(O_ref, x["G"], pairs)
    O = torch.empty(w.B, w.H, w.L, w.d_v, device="cuda", dtype=torch.bfloat16)
    Y = torch.empty(w.B, w.L, w.H * w.d_v, device="cuda", dtype=torch.bfloat16)
    S = torch.empty(w.B, w.H, w.d_k, w.d_v, device="cuda")
    # the tensor-core path: no workspace for Y alone, and one launch of the
    # loop when called without a workspace (the CUDA-core path would need an
    # fp32 O to normalise and a second launch for the gate)
    assert R.ret_workspace_size(w.B, w.H, w.L, w.d_k, w.d_v, R.RET_BF16, R.RET_BF16, g, w.chunk,
                                want_O=False, want_Y=True, rotate=w.rotate) == 0
    n0 = R.ret_kernel_launches()
    R.ret_chunkwise(d["Q"], d["K"], d["V"], g, w.chunk, O=O, state_out=S, G=d["G"], Y=Y,
                    rotate=w.rotate, prep=False)
    assert R.ret_kernel_launches() - n0 == 1
    assert rel_l2(O.reshape(-1, w.L, w.d_v), O_ref) <= TOL_BF16
    assert rel_l2(S.reshape(-1, w.d_k, w.d_v), S_ref) <= TOL_BF16
    assert rel_l2(y_slices(Y, pairs, w.d_v), Y_ref) <= TOL_BF16
    # Y alone (the benchmarked call, with ret_chunkwise_fast_size bytes: all
    # 512 blocks of 128 rows of the 32 heads in one launch, each block taking
    # its entering state from its predecessors' key-value sums)
    Y2 = torch.empty_like(Y)
    n0 = R.ret_kernel_launches()
    R.ret_chunkwise(d["Q"], d["K"], d["V"], g, w.chunk, G=d["G"], Y=Y2, rotate=w.rotate)
    assert R.ret_kernel_launches() - n0 == 1
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    assert rel_l2(y_slices(Y2, pairs, w.d_v), Y_ref) <= TOL_BF16
    # parallel form
    Op = torch.empty_like(O)
    R.ret_parallel(d["Q"], d["K"], d["V"], Op, g, rotate=w.rotate)
    assert rel_l2(Op.reshape(-1, w.L, w.d_v), O_ref) <= TOL_BF16


MSR_PAIRS = [(0, 0), (3, 4), (7, 7)]


def test_msr_1p3b_bf16_sampled():
    """RetNet-1.3B-shaped MSR, full size (B=8 H=8 L=4096 dk=256 dv=512,
    chunk 128, xPos): Y alone as benchmarked, then O, Y and the state, on
    three sampled (b, h) slices."""
    w = WORKLOADS["msr_1p3b"]
    x = make_inputs(w)
    d = dev(x)
    g = R.msr_gammas(w.H)
    O_ref, S_ref = oracle_slices(x["Q"], x["K"], x["V"], MSR_PAIRS, orc.gammas(w.H), w.rotate)
    Y_ref = oracle_gate_slices(O_ref, x["G"], MSR_PAIRS)
    Y = torch.empty(w.B, w.L, w.H * w.d_v, device="cuda", dtype=torch.bfloat16)
    R.ret_chunkwise(d["Q"], d["K"], d["V"], g, w.chunk, G=d["G"], Y=Y, rotate=w.rotate)
    assert rel_l2(y_slices(Y, MSR_PAIRS, w.d_v), Y_ref) <= TOL_BF16
    O = torch.empty(w.B, w.H, w.L, w.d_v, device="cuda", dtype=torch.bfloat16)
    S = torch.empty(w.B, w.H, w.d_k, w.d_v, device="cuda")
    Y.zero_()
    R.ret_chunkwise(d["Q"], d["K"], d["V"], g, w.chunk, O=O, state_out=S, G=d["G"], Y=Y,
                    rotate=w.rotate)
    for i, (b, h) in enumerate(MSR_PAIRS):
        assert rel_l2(O[b, h], O_ref[i]) <= TOL_BF16, (b, h)
        assert rel_l2(S[b, h], S_ref[i]) <= TOL_BF16, (b, h)
    assert rel_l2(y_slices(Y, MSR_PAIRS, w.d_v), Y_ref) <= TOL_BF16


def test_long_ctx_sampled():
    """Long context at full size (B=1 H=16 L=65536 d_k=128 d_v=256, chunk
    256, xPos): the outputs over all 65536 positions and the final state of
    the fastest- and slowest-decaying heads against the oracle's recurrent
    form."""
    w = WORKLOADS["long_ctx"]
    x = make_inputs(w)
    d = dev(x)
    pairs = [(0, 0), (0, w.H - 1)]
    O_ref, S_ref = oracle_slices(x["Q"], x["K"], x["V"], pairs, orc.gammas(w.H), w.rotate)
    O = torch.empty(w.B, w.H, w.L, w.d_v, device="cuda", dtype=torch.bfloat16)
    S = torch.empty(w.B, w.H, w.d_k, w.d_v, device="cuda")
    R.ret_chunkwise(d["Q"], d["K"], d["V"], R.msr_gammas(w.H), w.chunk, O=O, state_out=S,
                    rotate=w.rotate)
    for i, (b, h) in enumerate(pairs):
        assert rel_l2(O[b, h], O_ref[i]) <= TOL_BF16, (b, h)
        assert rel_l2(O[b, h, :4096], O_ref[i, :4096]) <= TOL_BF16, (b, h)
        assert rel_l2(S[b, h], S_ref[i]) <= TOL_BF16, (b, h)
    # the same with the sequence cut into 8 segments that run at once
    O8 = torch.empty_like(O)
    S8 = torch.empty_like(S)
    R.ret_chunkwise_segmented(d["Q"], d["K"], d["V"], R.msr_gammas(w.H), w.chunk, 8, O=O8,
                              state_out=S8, rotate=w.rotate)
    for i, (b, h) in enumerate(pairs):
        assert rel_l2(O8[b, h], O_ref[i]) <= TOL_BF16, (b, h)
        assert rel_l2(O8[b, h, :4096], O_ref[i, :4096]) <= TOL_BF16, (b, h)
        assert rel_l2(S8[b, h], S_ref[i]) <= TOL_BF16, (b, h)


def test_msr_1p3b_parallel_sampled():
    w = WORKLOADS["msr_1p3b"]
    x = make_inputs(w)
    d = dev(x)
    O_ref, _ = oracle_slices(x["Q"], x["K"], x["V"], MSR_PAIRS, orc.gammas(w.H), w.rotate)
    O = torch.empty(w.B, w.H, w.L, w.d_v, device="cuda", dtype=torch.bfloat16)
    R.ret_parallel(d["Q"], d["K"], d["V"], O, R.msr_gammas(w.H), rotate=w.rotate)
    for i, (b, h) in enumerate(MSR_PAIRS):
        assert rel_l2(O[b, h], O_ref[i]) <= TOL_BF16, (b, h)


def test_decode_after_prefill_sampled():
    """Recurrent decode at full size (B=64 H=16 dk=256 dv=512): chunkwise
    prefill of 8192 tokens builds the fp32 state, then single-token steps;
    two sampled sequences against the oracle over all 8192 + steps tokens."""
    w = WORKLOADS["decode"]
    steps = 4
    x = make_inputs(w, device="cuda")
    s = make_decode_inputs(w, steps=steps, device="cuda")
    g = R.msr_gammas(w.H)
    S = torch.empty(w.B, w.H, w.d_k, w.d_v, device="cuda")
    O = torch.empty(w.B, w.H, w.L, w.d_v, device="cuda", dtype=torch.bfloat16)
    R.ret_chunkwise(x["Q"], x["K"], x["V"], g, w.chunk, O=O, state_out=S, rotate=w.rotate)
    o = torch.empty(w.B, w.H, w.d_v, device="cuda", dtype=torch.float32)
    outs = []
    for t in range(steps):
        R.ret_recurrent_step(s["q"][t], s["k"][t], s["v"][t], S, o, g, pos=w.L + t, rotate=w.rotate)
        outs.append(o.clone())
    pairs = [(0, 0), (37, 15)]
    for i, (b, h) in enumerate(pairs):
        qq = torch.cat([x["Q"][b, h], s["q"][:, b, h]], 0)[None, None]
        kk = torch.cat([x["K"][b, h], s["k"][:, b, h]], 0)[None, None]
        vv = torch.cat([x["V"][b, h], s["v"][:, b, h]], 0)[None, None]
        O_ref, S_ref = orc.recurrent(qq, kk, vv, [orc.gammas(w.H)[h]], rotate=w.rotate)
        got = torch.stack([oo[b, h] for oo in outs])
        assert rel_l2(got, O_ref[0, 0, w.L:]) <= TOL_BF16
        assert rel_l2(O[b, h], O_ref[0, 0, :w.L]) <= TOL_BF16
        assert rel_l2(S[b, h], S_ref[0, 0]) <= TOL_BF16
