"""Parity of the tensor-core chunkwise path (bf16 inputs, chunk 128, d_k 128
or 256, d_v a multiple of 128, gamma^128 >= 2^-60) against the fp64 oracle:
ragged tails, a single row, state in/out (aliased), rotation at large
positions, gamma = 1 heads, fp32 and bf16 outputs, and the fused GroupNorm +
swish gate epilogue at cluster sizes 1, 2 and 4.  Each case runs with the
operands prepared ahead by the streaming pass (`prep`, two launches) and
with the kernel preparing them itself (one launch)."""
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
    return Q, K, V


@pytest.mark.parametrize("prep", [True, False])
@pytest.mark.parametrize("B,H,L,dk,dv,out", [
    (1, 2, 128, 128, 128, torch.float32),
    (1, 2, 300, 128, 128, torch.float32),
    (2, 1, 1, 256, 128, torch.float32),
    (1, 3, 257, 256, 256, torch.bfloat16),
    (2, 2, 640, 256, 512, torch.bfloat16),
])
def test_tc_chunkwise_matches_oracle(B, H, L, dk, dv, out, prep):
    Q, K, V = _inputs(B, H, L, dk, dv, 100 + L)
    g = ([0.75, 0.96875, 1.0] * 2)[:H] if H > 1 else [0.96875]
    O_ref, S_ref = orc.recurrent(Q, K, V, g, rotate=True, pos_offset=5)
    O = torch.empty(B, H, L, dv, device="cuda", dtype=out)
    S = torch.empty(B, H, dk, dv, device="cuda")
    R.ret_chunkwise(Q.cuda(), K.cuda(), V.cuda(), g, 128, O=O, state_out=S, rotate=True,
                    pos_offset=5, prep=prep)
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    for b in range(B):
        for h in range(H):
            assert rel_l2(O[b, h], O_ref[b, h]) <= TOL_BF16, (b, h)
            assert rel_l2(S[b, h], S_ref[b, h]) <= TOL_BF16, (b, h)


@pytest.mark.parametrize("prep", [True, False])
def test_tc_chunk_multiple_of_128(prep):
    """Chunks of 256 and 384 rows run on the tensor cores as blocks of 128
    rows; outputs, the fused gate and the state match the oracle."""
    B, H, L, dk, dv = 1, 2, 700, 128, 256
    Q, K, V = _inputs(B, H, L, dk, dv, 77)
    G = random_tensor((B, L, H * dv), 78).bfloat16()
    g = [0.96875, 0.999]
    O_ref, S_ref = orc.recurrent(Q, K, V, g, rotate=True, pos_offset=3)
    Y_ref = orc.gate_groupnorm(O_ref, G)
    for chunk in (256, 384):
        O = torch.empty(B, H, L, dv, device="cuda", dtype=torch.bfloat16)
        Y = torch.empty(B, L, H * dv, device="cuda", dtype=torch.bfloat16)
        S = torch.empty(B, H, dk, dv, device="cuda")
        n0 = R.ret_kernel_launches()
        R.ret_chunkwise(Q.cuda(), K.cuda(), V.cuda(), g, chunk, O=O, G=G.cuda(), Y=Y, state_out=S,
                        rotate=True, pos_offset=3, prep=prep)
        assert R.ret_kernel_launches() - n0 == (2 if prep else 1)   # no CUDA-core fallback
        torch.cuda.synchronize()
        assert R.ret_last_device_status() == 0
        for h in range(H):
            assert rel_l2(O[0, h], O_ref[0, h]) <= TOL_BF16, (chunk, h)
            assert rel_l2(S[0, h], S_ref[0, h]) <= TOL_BF16, (chunk, h)
        assert rel_l2(Y, Y_ref) <= TOL_BF16, chunk


@pytest.mark.parametrize("prep", [True, False])
def test_tc_state_chaining_and_large_positions(prep):
    """Two calls joined through an aliased state equal one oracle run; the
    second starts near position 60000."""
    B, H, L1, L2, dk, dv = 1, 2, 200, 190, 128, 128
    Q, K, V = _inputs(B, H, L1 + L2, dk, dv, 7)
    g = [0.96875, 0.999]
    p0 = 60000
    O_ref, S_ref = orc.recurrent(Q, K, V, g, rotate=True, pos_offset=p0)
    Qd, Kd, Vd = Q.cuda(), K.cuda(), V.cuda()
    S = torch.empty(B, H, dk, dv, device="cuda")
    O1 = torch.empty(B, H, L1, dv, device="cuda")
    O2 = torch.empty(B, H, L2, dv, device="cuda")
    R.ret_chunkwise(Qd[:, :, :L1].contiguous(), Kd[:, :, :L1].contiguous(), Vd[:, :, :L1].contiguous(),
                    g, 128, O=O1, state_out=S, rotate=True, pos_offset=p0, prep=prep)
    R.ret_chunkwise(Qd[:, :, L1:].contiguous(), Kd[:, :, L1:].contiguous(), Vd[:, :, L1:].contiguous(),
                    g, 128, O=O2, state_in=S, state_out=S, rotate=True, pos_offset=p0 + L1,
                    prep=prep)
    got = torch.cat([O1, O2], 2)
    for h in range(H):
        assert rel_l2(got[0, h], O_ref[0, h]) <= TOL_BF16
        assert rel_l2(S[0, h], S_ref[0, h]) <= TOL_BF16


@pytest.mark.parametrize("prep", [True, False])
@pytest.mark.parametrize("dk,dv,rotate,with_O,with_state", [
    (256, 256, False, False, False),
    (256, 512, True, True, False),
    (128, 128, True, False, True),
    (128, 384, False, True, True),
])
def test_tc_fused_gate_groupnorm(dk, dv, rotate, with_O, with_state, prep):
    """Y = swish(G) (.) GroupNorm_h(O) from the one fused launch (after the
    preparing pass when `prep`)."""
    B, H, L = 2, 2, 300
    Q, K, V = _inputs(B, H, L, dk, dv, 21 + dv)
    G = random_tensor((B, L, H * dv), 24).bfloat16()
    S0 = random_tensor((B, H, dk, dv), 25, 0.3) if with_state else None
    g = [0.9, 0.995]
    O_ref, S_ref = orc.recurrent(Q, K, V, g, rotate=rotate, pos_offset=17, state_in=S0)
    Y_ref = orc.gate_groupnorm(O_ref, G)
    Y = torch.empty(B, L, H * dv, device="cuda", dtype=torch.bfloat16)
    O = torch.empty(B, H, L, dv, device="cuda", dtype=torch.bfloat16) if with_O else None
    S = torch.empty(B, H, dk, dv, device="cuda")
    n0 = R.ret_kernel_launches()
    R.ret_chunkwise(Q.cuda(), K.cuda(), V.cuda(), g, 128, O=O, G=G.cuda(), Y=Y, rotate=rotate,
                    pos_offset=17, state_in=None if S0 is None else S0.cuda(), state_out=S,
                    prep=prep)
    assert R.ret_kernel_launches() - n0 == (2 if prep else 1)
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    for b in range(B):
        for h in range(H):
            assert rel_l2(Y[b, :, h * dv:(h + 1) * dv], Y_ref[b, :, h * dv:(h + 1) * dv]) <= TOL_BF16
            assert rel_l2(S[b, h], S_ref[b, h]) <= TOL_BF16
            if with_O:
                assert rel_l2(O[b, h], O_ref[b, h]) <= TOL_BF16


def test_small_gamma_uses_cuda_core_path():
    """gamma below the tensor-core range (gamma^128 < 2^-60) still matches."""
    B, H, L, dk, dv = 1, 2, 200, 128, 128
    Q, K, V = _inputs(B, H, L, dk, dv, 31)
    g = [0.0, 0.5]
    O_ref, _ = orc.recurrent(Q, K, V, g, rotate=True)
    O = torch.empty(B, H, L, dv, device="cuda")
    R.ret_chunkwise(Q.cuda(), K.cuda(), V.cuda(), g, 128, O=O, rotate=True)
    assert rel_l2(O, O_ref) <= TOL_BF16


@pytest.mark.parametrize("B,H,L,dk,dv,rotate,out", [
    (1, 3, 300, 128, 128, True, torch.float32),
    (2, 2, 640, 256, 256, True, torch.bfloat16),
    (1, 3, 1100, 256, 512, False, torch.bfloat16),
    (1, 1, 1, 128, 256, True, torch.float32),
])
def test_tc_parallel_matches_oracle(B, H, L, dk, dv, rotate, out):
    """Parallel form on the tensor cores (rotation pre-pass into the
    workspace, decay as a rank-1 scaling, underflowed key tiles skipped)."""
    Q, K, V = _inputs(B, H, L, dk, dv, 300 + L)
    g = ([0.75, 0.96875, 1.0] * 2)[:H]
    O_ref, _ = orc.recurrent(Q, K, V, g, rotate=rotate, pos_offset=9)
    O = torch.empty(B, H, L, dv, device="cuda", dtype=out)
    R.ret_parallel(Q.cuda(), K.cuda(), V.cuda(), O, g, rotate=rotate, pos_offset=9)
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    for b in range(B):
        for h in range(H):
            assert rel_l2(O[b, h], O_ref[b, h]) <= TOL_BF16, (b, h)


@pytest.mark.parametrize("rotate", [True, False])
def test_prepare_pass_matches_oracle(rotate):
    """The streaming pass alone: Q^ = Theta_t Q_t and K~ = gamma^{n-1-j}
    Theta_t K_t (bf16) for row t at offset j of its chunk of n rows (ragged
    last chunk), against the oracle's fp64 rotation, row by row."""
    B, H, L, dk, p0 = 2, 3, 300, 256, 70000
    Q, K, _ = _inputs(B, H, L, dk, 128, 41)
    g = [0.9, 0.96875, 0.999]
    size = R.ret_chunkwise_prep_size(B, H, L, dk, 128, R.RET_BF16, R.RET_BF16, g, 128,
                                     rotate=rotate, pos_offset=p0)
    assert size == (2 if rotate else 1) * B * H * L * dk * 2
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")
    qh, kt = R.ret_chunkwise_prepare(Q.cuda(), K.cuda(), g, 128, ws, rotate=rotate, pos_offset=p0)
    torch.cuda.synchronize()
    t = np.arange(L)
    j = t % 128
    n = np.minimum(128, L - (t - j))
    for b in range(B):
        for h in range(H):
            for name, X, got, weighted in (("Q", Q, qh, False), ("K", K, kt, True)):
                if got is None:
                    continue
                x = X[b, h].double().numpy()
                ref = np.stack([orc.xpos_rotate(x[r], p0 + r) for r in range(L)]) if rotate else x
                if weighted:
                    ref = ref * (g[h] ** (n - 1 - j))[:, None]
                out = got[b, h].float().cpu().double().numpy()
                err = np.abs(out - ref)
                assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-6 * np.abs(ref).max()), (name, b, h)


def test_batch_slices_and_prepared_loop_are_exact():
    """Two waves of CTAs (B=3 x H=16 x d_v/128=4 = 192 > 148 SMs): the call
    cuts the batch into two uneven slices (1 and 2 batch elements, one wave
    each) and overlaps the streaming pass of one with the loop of the other.
    Every (b, h) is independent, so the result is bitwise that of one call
    per batch element (64 CTAs, no slices) and of the loop alone on rows
    prepared by ret_chunkwise_prepare; and it matches the oracle on sampled
    slices."""
    B, H, L, dk, dv = 3, 16, 300, 128, 512
    Q, K, V = _inputs(B, H, L, dk, dv, 61)
    G = random_tensor((B, L, H * dv), 62).bfloat16()
    S0 = random_tensor((B, H, dk, dv), 63, 0.1)
    g = [1 - 2.0 ** (-5 - (h % 8)) for h in range(H)]
    Qd, Kd, Vd, Gd, S0d = Q.cuda(), K.cuda(), V.cuda(), G.cuda(), S0.cuda()
    mk = lambda: (torch.empty(B, H, L, dv, device="cuda", dtype=torch.bfloat16),  # noqa: E731
                  torch.empty(B, L, H * dv, device="cuda", dtype=torch.bfloat16),
                  torch.empty(B, H, dk, dv, device="cuda"))
    O1, Y1, S1 = mk()
    n0 = R.ret_kernel_launches()
    R.ret_chunkwise(Qd, Kd, Vd, g, 128, O=O1, G=Gd, Y=Y1, state_in=S0d, state_out=S1, rotate=True,
                    pos_offset=9)
    assert R.ret_kernel_launches() - n0 == 4          # two slices: pass + loop each
    O2, Y2, S2 = mk()
    for b in range(B):
        R.ret_chunkwise(Qd[b:b + 1], Kd[b:b + 1], Vd[b:b + 1], g, 128, O=O2[b:b + 1], G=Gd[b:b + 1],
                        Y=Y2[b:b + 1], state_in=S0d[b:b + 1], state_out=S2[b:b + 1], rotate=True,
                        pos_offset=9)
    size = R.ret_chunkwise_prep_size(B, H, L, dk, dv, R.RET_BF16, R.RET_BF16, g, 128, rotate=True,
                                     pos_offset=9)
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")
    qh, kt = R.ret_chunkwise_prepare(Qd, Kd, g, 128, ws, rotate=True, pos_offset=9)
    O3, Y3, S3 = mk()
    R.ret_chunkwise_prepared(qh, kt, Vd, g, 128, O=O3, G=Gd, Y=Y3, state_in=S0d, state_out=S3,
                             rotate=True, pos_offset=9)
    torch.cuda.synchronize()
    for a, b in ((O1, O2), (Y1, Y2), (S1, S2), (O1, O3), (Y1, Y3), (S1, S3)):
        assert torch.equal(a, b)
    pairs = [(0, 0), (1, 7), (2, 15)]
    pick = lambda X: np.stack([X[b, h].double().numpy() for b, h in pairs])[None]  # noqa: E731
    O_ref, S_ref = orc.recurrent(pick(Q), pick(K), pick(V), [g[h] for _, h in pairs], rotate=True,
                                 pos_offset=9, state_in=pick(S0))
    for i, (b, h) in enumerate(pairs):
        assert rel_l2(O1[b, h], O_ref[0, i]) <= TOL_BF16, (b, h)
        assert rel_l2(S1[b, h], S_ref[0, i]) <= TOL_BF16, (b, h)


@pytest.mark.parametrize("dk,dv,chunk,rotate,prep", [
    (64, 64, 64, True, True),      # the small MSR head (rotated: prepared rows)
    (64, 64, 64, False, False),    # value rows weighted inside the loop
    (64, 256, 128, True, True),    # d_k 64 with two CTAs of columns per head
    (128, 64, 64, False, True),    # d_v 64 under a wider d_k
])
def test_tc_small_heads(dk, dv, chunk, rotate, prep):
    """d_k 64 and d_v 64 on the tensor cores (a CTA with 64 value columns,
    the rest of its tile zero), chunks of 64 rows (two per block of 128):
    O, Y and the state against the oracle, ragged tail, with a state in."""
    B, H, L = 2, 3, 333
    Q, K, V = _inputs(B, H, L, dk, dv, 500 + dk + dv)
    G = random_tensor((B, L, H * dv), 520).bfloat16()
    S0 = random_tensor((B, H, dk, dv), 521, 0.2)
    g = [0.96875, 0.99, 0.999]
    O_ref, S_ref = orc.recurrent(Q, K, V, g, rotate=rotate, pos_offset=11, state_in=S0)
    Y_ref = orc.gate_groupnorm(O_ref, G)
    O = torch.empty(B, H, L, dv, device="cuda", dtype=torch.bfloat16)
    Y = torch.empty(B, L, H * dv, device="cuda", dtype=torch.bfloat16)
    S = torch.empty(B, H, dk, dv, device="cuda")
    n0 = R.ret_kernel_launches()
    R.ret_chunkwise(Q.cuda(), K.cuda(), V.cuda(), g, chunk, O=O, G=G.cuda(), Y=Y, rotate=rotate,
                    pos_offset=11, state_in=S0.cuda(), state_out=S, prep=prep)
    assert R.ret_kernel_launches() - n0 == (2 if prep else 1)   # no CUDA-core fallback
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    for b in range(B):
        for h in range(H):
            assert rel_l2(O[b, h], O_ref[b, h]) <= TOL_BF16, (b, h)
            assert rel_l2(S[b, h], S_ref[b, h]) <= TOL_BF16, (b, h)
            assert rel_l2(Y[b, :, h * dv:(h + 1) * dv], Y_ref[b, :, h * dv:(h + 1) * dv]) <= TOL_BF16


@pytest.mark.parametrize("B,H,L,dk,dv,rotate,out", [
    (2, 3, 333, 64, 64, True, torch.bfloat16),
    (1, 2, 500, 64, 256, False, torch.float32),
    (1, 2, 300, 128, 64, True, torch.bfloat16),
])
def test_tc_parallel_small_heads(B, H, L, dk, dv, rotate, out):
    """The parallel form on the tensor cores at d_k 64 and d_v 64 (value
    slices of 64 columns): against the oracle, and on the tensor-core path
    (with rotation it needs the workspace for the turned rows and launches
    the two turning passes and the product)."""
    Q, K, V = _inputs(B, H, L, dk, dv, 700 + L)
    g = ([0.75, 0.96875, 1.0] * 2)[:H]
    O_ref, _ = orc.recurrent(Q, K, V, g, rotate=rotate, pos_offset=3)
    O = torch.empty(B, H, L, dv, device="cuda", dtype=out)
    n0 = R.ret_kernel_launches()
    R.ret_parallel(Q.cuda(), K.cuda(), V.cuda(), O, g, rotate=rotate, pos_offset=3)
    if rotate:
        assert R.ret_kernel_launches() - n0 == 3
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    for b in range(B):
        for h in range(H):
            assert rel_l2(O[b, h], O_ref[b, h]) <= TOL_BF16, (b, h)
