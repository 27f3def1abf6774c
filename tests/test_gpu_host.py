"""ret_chunkwise_host: the chunkwise forward from host buffers to host
buffers through the batch-slice pipeline matches ret_chunkwise on device
buffers exactly (the same kernels run on every (b, h)), for every slice
count, on the tensor-core path with the fused gate and on the CUDA-core
path, with page-locked and with pageable host memory; and it matches the
oracle."""
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


def _inputs(B, H, L, dk, dv, dtype, seed, gate=True):
    Q = random_tensor((B, H, L, dk), seed, dk ** -0.5).to(dtype)
    K = random_tensor((B, H, L, dk), seed + 1, dk ** -0.5).to(dtype)
    V = random_tensor((B, H, L, dv), seed + 2).to(dtype)
    G = random_tensor((B, L, H * dv), seed + 3).to(dtype) if gate else None
    return Q, K, V, G


@pytest.mark.parametrize("slices", [1, 2, 3, 5])
def test_host_pipeline_tc_gate(slices):
    B, H, L, dk, dv = 5, 2, 300, 128, 256
    Q, K, V, G = _inputs(B, H, L, dk, dv, torch.bfloat16, 500)
    g = [0.96875, 0.999]
    Y_dev = torch.empty(B, L, H * dv, device="cuda", dtype=torch.bfloat16)
    R.ret_chunkwise(Q.cuda(), K.cuda(), V.cuda(), g, 128, G=G.cuda(), Y=Y_dev, rotate=True,
                    pos_offset=11)
    pin = lambda t: t.pin_memory()
    Y = torch.full((B, L, H * dv), float("nan"), dtype=torch.bfloat16).pin_memory()
    R.ret_chunkwise_host(pin(Q), pin(K), pin(V), g, 128, G=pin(G), Y=Y, rotate=True,
                         pos_offset=11, slices=slices)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y_dev.cpu())
    if slices == 2:
        O_ref, _ = orc.recurrent(Q, K, V, g, rotate=True, pos_offset=11)
        assert rel_l2(Y, orc.gate_groupnorm(O_ref, G)) <= TOL_BF16


@pytest.mark.parametrize("pinned", [True, False])
def test_host_pipeline_cuda_core_outputs(pinned):
    """fp32 inputs (CUDA-core kernel), O and Y together, pageable or
    page-locked host memory, a ragged last slice."""
    B, H, L, dk, dv = 3, 2, 100, 32, 32
    Q, K, V, G = _inputs(B, H, L, dk, dv, torch.float32, 600)
    g = [0.9, 0.99]
    O_dev = torch.empty(B, H, L, dv, device="cuda")
    Y_dev = torch.empty(B, L, H * dv, device="cuda")
    R.ret_chunkwise(Q.cuda(), K.cuda(), V.cuda(), g, 16, O=O_dev, G=G.cuda(), Y=Y_dev, rotate=True)
    hold = (lambda t: t.pin_memory()) if pinned else (lambda t: t.clone())
    O = hold(torch.zeros(B, H, L, dv))
    Y = hold(torch.zeros(B, L, H * dv))
    R.ret_chunkwise_host(hold(Q), hold(K), hold(V), g, 16, O=O, G=hold(G), Y=Y, rotate=True,
                         slices=2)
    torch.cuda.synchronize()
    assert torch.equal(O, O_dev.cpu())
    assert torch.equal(Y, Y_dev.cpu())
