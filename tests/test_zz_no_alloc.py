"""ret_chunkwise_gate_static: the chunkwise forward with the fused
GroupNorm + swish gate for callers that may not allocate device memory
(memory reserved up front by a host framework, or a fixed budget once
serving starts).  Its scratch is the library's fixed device array, so the
test checks, through the C ABI, that two calls in a row match the
allocating entry point ret_chunkwise on the same inputs, and that a problem
too large for the array is refused.  It sits in a file of its own, collected
last, and must pass alone in a fresh process as well."""
import ctypes

import pytest
import torch

from parity import normwise, rel_l2, TOL_BF16, TOL_F32
from retentive_network_scale_b200 import build
from retentive_network_scale_b200 import retention as R
from retentive_network_scale_b200.synth import random_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    build.build()
    return R.load_library()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_static(lib, Q, K, V, G, Y, g, chunk, rotate):
    B, H, L, dk = Q.shape
    dv = V.shape[-1]
    code = R.RET_F32 if Q.dtype == torch.float32 else R.RET_BF16
    d = R.make_desc(B, H, L, dk, dv, code, code, g, rotate)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.ret_chunkwise_gate_static(ctypes.byref(d), chunk, _ptr(Q), _ptr(K), _ptr(V), None,
                                         None, _ptr(G), ctypes.c_float(1e-5), _ptr(Y), stream)


@pytest.mark.parametrize("dtype,dk,dv,rotate", [
    (torch.float32, 32, 48, True),
    (torch.bfloat16, 64, 64, False),
])
def test_static_scratch_matches_allocating_entry(lib, dtype, dk, dv, rotate):
    B, H, L, chunk = 2, 3, 150, 32
    Q = random_tensor((B, H, L, dk), 61, dk ** -0.5).to(dtype).cuda()
    K = random_tensor((B, H, L, dk), 62, dk ** -0.5).to(dtype).cuda()
    V = random_tensor((B, H, L, dv), 63).to(dtype).cuda()
    G = random_tensor((B, L, H * dv), 64).to(dtype).cuda()
    g = [0.9, 0.96875, 0.999]
    # this shape needs scratch in ret_chunkwise (the CUDA-core path)
    assert R.ret_workspace_size(B, H, L, dk, dv, R._dtype_code(Q), R._dtype_code(Q), g, chunk,
                                want_O=False, want_Y=True, rotate=rotate) > 0
    Y_ref = torch.empty(B, L, H * dv, device="cuda", dtype=dtype)
    R.ret_chunkwise(Q, K, V, g, chunk, G=G, Y=Y_ref, rotate=rotate)
    for _ in range(2):  # two calls in a row share the scratch
        Y = torch.full((B, L, H * dv), float("nan"), device="cuda", dtype=dtype)
        assert _call_static(lib, Q, K, V, G, Y, g, chunk, rotate) == 0
        torch.cuda.synchronize()
        assert R.ret_last_device_status() == 0
        if dtype == torch.float32:
            assert normwise(Y, Y_ref) <= TOL_F32
        else:
            assert rel_l2(Y, Y_ref) <= TOL_BF16


def test_static_scratch_refuses_oversized_problem(lib):
    # B*H*L*d_v floats beyond the fixed array: refused before anything runs
    B, H, dk, dv = 1, 1, 16, 64
    L = R.RET_STATIC_SCRATCH_FLOATS // dv + 1
    Q = torch.zeros(1, device="cuda")
    d = R.make_desc(B, H, L, dk, dv, R.RET_F32, R.RET_F32, [0.9])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.ret_chunkwise_gate_static(ctypes.byref(d), 16, _ptr(Q), _ptr(Q), _ptr(Q), None, None,
                                       _ptr(Q), ctypes.c_float(1e-5), _ptr(Q), stream)
    assert rc == R.STATUS_NAMES.index("RET_ERR_WORKSPACE")
