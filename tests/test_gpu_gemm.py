"""ret_gemm_bf16, the tensor-core product behind the layer's projections,
against the fp64 product of the same bf16 operands on the CPU: ragged M, N
and K (tails of every tile dimension and of the 64-wide k blocks), strided
rows, more tiles than SMs (each persistent CTA then reuses both tensor
memory accumulators and every pipeline stage several times), and the
argument refusals."""
import pytest
import torch

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


def check(A, B, C):
    """Every element within the bf16 rounding of the exact product plus an
    fp32 accumulation allowance."""
    ref = A.double().cpu() @ B.double().cpu()
    mag = A.double().abs().cpu() @ B.double().abs().cpu()
    err = (C.double().cpu() - ref).abs()
    bound = 2.0 ** -8 * ref.abs() + 1e-5 * mag + 1e-30
    assert bool((err <= bound).all()), float((err / bound).max())


@pytest.mark.parametrize("M,N,K", [(1, 8, 8), (128, 256, 64), (300, 264, 200), (257, 520, 1000),
                                   (4096, 4096, 128), (2048, 2560, 320)])
def test_gemm_matches_fp64_product(M, N, K):
    A = random_tensor((M, K), 900 + M).bfloat16().cuda()
    B = random_tensor((K, N), 901 + N, K ** -0.5).bfloat16().cuda()
    C = R.ret_gemm_bf16(A, B)
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    check(A, B, C)


def test_gemm_strided_rows():
    # A and C as column windows of wider matrices (leading dimensions above
    # the row length), B a window of a wider weight matrix
    Aw = random_tensor((200, 328), 910).bfloat16().cuda()
    Bw = random_tensor((136, 1040), 911, 0.1).bfloat16().cuda()
    Cw = torch.zeros(200, 800, device="cuda", dtype=torch.bfloat16)
    A, B, C = Aw[:, 8:144], Bw[:, 16:528], Cw[:, 40:552]
    R.ret_gemm_bf16(A, B, C)
    torch.cuda.synchronize()
    check(A, B, C)
    # nothing outside the window was written
    assert bool((Cw[:, :40] == 0).all()) and bool((Cw[:, 552:] == 0).all())


def test_gemm_refusals():
    A = torch.zeros(16, 16, device="cuda", dtype=torch.bfloat16)
    B = torch.zeros(16, 12, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(R.RetentionError, match="RET_ERR_SHAPE"):   # N not a multiple of 8
        R.ret_gemm_bf16(A, B)
    B0 = torch.zeros(0, 16, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(R.RetentionError, match="RET_ERR_SHAPE"):   # K = 0
        R.ret_gemm_bf16(torch.zeros(16, 0, device="cuda", dtype=torch.bfloat16), B0)
    buf = torch.zeros(16 * 16 + 1, device="cuda", dtype=torch.bfloat16)
    Am = buf[1:].view(16, 16)                                        # 2-byte offset
    with pytest.raises(R.RetentionError, match="RET_ERR_ALIGN"):
        R.ret_gemm_bf16(Am, torch.zeros(16, 16, device="cuda", dtype=torch.bfloat16))
    C = R.ret_gemm_bf16(torch.zeros(0, 16, device="cuda", dtype=torch.bfloat16),
                        torch.zeros(16, 16, device="cuda", dtype=torch.bfloat16))
    assert C.shape == (0, 16)
