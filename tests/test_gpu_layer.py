"""ret_msr_layer (projections, retention with the fused GroupNorm + gate,
output projection) against the fp64 layer oracle; the projection's epilogue
writes the turned / decay-weighted Q and K per head and the chunk loop reads
V and G from the projection in place (strided tensor maps), so small cases
with two or three heads, ragged lengths (blocks of 128 rows cut short, rows
of one tile spanning two sequences) and both tensor-core d_k check that
plumbing; plus argument refusals."""
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


@pytest.mark.parametrize("dk,dv,rotate,H", [(128, 128, True, 2), (256, 256, False, 2),
                                            (128, 384, True, 2), (128, 128, True, 3),
                                            (256, 128, True, 1)])
def test_msr_layer_matches_oracle(dk, dv, rotate, H):
    B, L, dm = 2, 300, 256
    g = [0.96875, 0.999, 0.9921875][:H]
    n_proj = H * (2 * dk + 2 * dv)
    X = random_tensor((B, L, dm), 700).bfloat16()
    W = random_tensor((dm, n_proj), 701, dm ** -0.5).bfloat16()
    Wo = random_tensor((H * dv, dm), 702, (H * dv) ** -0.5).bfloat16()
    ref = orc.msr_layer(X, W, Wo, g, dk, dv, rotate=rotate, pos_offset=5)
    n0 = R.ret_kernel_launches()
    out = R.ret_msr_layer(X.cuda(), W.cuda(), Wo.cuda(), g, 128, dk, dv, rotate=rotate,
                          pos_offset=5)
    assert R.ret_kernel_launches() - n0 == 3          # projection (+ turn), chunk loop, W_o
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    assert rel_l2(out, ref) <= TOL_BF16


def test_msr_layer_refusals():
    X = torch.zeros(1, 128, 64, device="cuda", dtype=torch.bfloat16)
    W = torch.zeros(64, 2 * (2 * 128 + 2 * 128), device="cuda", dtype=torch.bfloat16)
    Wo = torch.zeros(2 * 128, 64, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(R.RetentionError, match="RET_ERR_SHAPE"):   # chunk 96: CUDA-core path
        R.ret_msr_layer(X, W, Wo, [0.9, 0.99], 96, 128, 128)
    with pytest.raises(R.RetentionError, match="RET_ERR_SHAPE"):   # gamma^128 below 2^-60
        R.ret_msr_layer(X, W, Wo, [0.5, 0.99], 128, 128, 128)


def test_msr_layer_full_size_sampled():
    """The RetNet-1.3B layer at full size (B=8 L=4096 d_model=2048 H=8
    d_k=256 d_v=512, chunk 128, xPos: the benchmarked shapes, 128 x 48 tiles
    of the projection GEMM, positions up to 4095 in its turn epilogue); batch
    element 0, every row and column, against the fp64 layer oracle on that
    element alone (a row of the layer depends only on its own sequence)."""
    from retentive_network_scale_b200.synth import WORKLOADS
    w = WORKLOADS["msr_1p3b"]
    dm = w.H * w.d_k
    n_proj = w.H * (2 * w.d_k + 2 * w.d_v)
    X = random_tensor((w.B, w.L, dm), 710).bfloat16()
    W = random_tensor((dm, n_proj), 711, dm ** -0.5).bfloat16()
    Wo = random_tensor((w.H * w.d_v, dm), 712, (w.H * w.d_v) ** -0.5).bfloat16()
    out = R.ret_msr_layer(X.cuda(), W.cuda(), Wo.cuda(), R.msr_gammas(w.H), w.chunk, w.d_k, w.d_v,
                          rotate=True)
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    ref = orc.msr_layer(X[:1], W, Wo, orc.gammas(w.H), w.d_k, w.d_v, rotate=True)
    assert rel_l2(out[0], ref[0]) <= TOL_BF16
